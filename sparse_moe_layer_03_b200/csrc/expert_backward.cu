// Memory-bound pieces of the expert MLPs' backward ("Scaling Diffusion Transformers
// to 16 Billion Parameters", "MOE 回顾" eq. MoE(x) and "MOE-DIT" eq. MLP: the
// models are trained, so every weight, the input and the gates need gradients).
// The GEMMs run on the CTA-pair tensor-core kernel; here:
//
//   gather  : dY rows into the expert-contiguous order of the forward, twice: as
//             given (dY_perm, for dH = dY W2 and the gates' gradient) and scaled by
//             the row's gate (dZ_perm = g dY, for dW2 and db2).  Padding rows get 0.
//   colsum  : bias gradients, column sums over each expert's rows (or all T rows):
//             partial sums of 256-row chunks, then each segment's chunks in order.
//             Fixed order throughout: bit-reproducible.
//   dgate   : dJ/dg for every selected (token, expert) slot, <dY_t, e_i(x_t)>:
//             the GELU-backward GEMM leaves sum_h (dY W2)[r,h] gelu(u)[r,h] per
//             column tile; this adds the tiles in order and <dY_t, b2_i>.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kEbThreads = 256;
constexpr int kColChunk = 256;          // rows per partial sum (a segment of the permuted layout holds whole chunks)

template <typename S>
__global__ void __launch_bounds__(kEbThreads) bwd_gather_kernel(ExpertBwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int nvec = a.D / 8;                            // 16-byte vectors of a 16-bit row
  const long long r = (long long)blockIdx.x * (kEbThreads / 32) + (threadIdx.x >> 5);
  if (r >= a.rows) return;
  const int t = a.row_token[r];
  uint4* dp = reinterpret_cast<uint4*>(a.dout_perm) + r * nvec;
  uint4* dz = reinterpret_cast<uint4*>(a.dz_perm) + r * nvec;
  if (t < 0 || t >= a.T) {
    for (int v = lane; v < nvec; v += 32) {
      dp[v] = make_uint4(0u, 0u, 0u, 0u);
      dz[v] = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }
  const float g = a.row_gate[r];
  const uint4* src = reinterpret_cast<const uint4*>(a.dout) + (long long)t * nvec;
  for (int v = lane; v < nvec; v += 32) {
    const uint4 q = __ldg(src + v);
    dp[v] = q;
    float f[8];
    S::x8_to_f32(q, f);
    dz[v] = make_uint4(S::pack2(g * f[0], g * f[1]), S::pack2(g * f[2], g * f[3]), S::pack2(g * f[4], g * f[5]),
                       S::pack2(g * f[6], g * f[7]));
  }
}

// partial[chunk, c] = sum of rows [chunk * 256, ...) of X[:, c], in row order; each thread takes
// two adjacent columns
template <typename S>
__global__ void __launch_bounds__(kEbThreads) colsum_partial_kernel(const void* X, long long nrows, int C,
                                                                    float* partial) {
  const int chunk = blockIdx.x;
  const int c = (blockIdx.y * kEbThreads + threadIdx.x) * 2;
  if (c >= C) return;
  const long long r0 = (long long)chunk * kColChunk;
  const long long r1 = r0 + kColChunk < nrows ? r0 + kColChunk : nrows;
  const uint16_t* x = reinterpret_cast<const uint16_t*>(X);
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
  for (long long r = r0; r < r1; ++r) {
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(x + r * C + c));
    float f[8];
    S::x8_to_f32(make_uint4(v, 0u, 0u, 0u), f);
    s0 += f[0];
    s1 += f[1];
  }
  partial[(long long)chunk * C + c] = s0;
  partial[(long long)chunk * C + c + 1] = s1;
}

// out[seg, c] (repeated nrep times, rows seg * nrep + j) = sum over the segment's chunks in
// order.  Segments: the experts' padded segments (offsets != null) or every chunk (one segment).
__global__ void __launch_bounds__(kEbThreads) colsum_reduce_kernel(const float* partial, int nchunks, int C,
                                                                   const int32_t* offsets, int E, int nrep,
                                                                   float* out) {
  const int nseg = offsets ? E : 1;
  const long long n = (long long)nseg * C;
  for (long long i = (long long)blockIdx.x * kEbThreads + threadIdx.x; i < n; i += (long long)gridDim.x * kEbThreads) {
    const int seg = (int)(i / C), c = (int)(i % C);
    int k0 = 0, k1 = nchunks;
    if (offsets) {
      long long p = 0;
      for (int j = 0; j < seg; ++j) p += (offsets[j + 1] - offsets[j] + kSegAlign - 1) / kSegAlign * kSegAlign;
      const int cnt = offsets[seg + 1] - offsets[seg];
      k0 = (int)(p / kColChunk);
      k1 = k0 + (cnt + kColChunk - 1) / kColChunk;
      if (k1 > nchunks) k1 = nchunks;
    }
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    int k = k0;
    for (; k + 4 <= k1; k += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) s[u] += __ldcg(partial + (long long)(k + u) * C + c);
    }
    for (int u = 0; k < k1; ++k, ++u) s[u] += __ldcg(partial + (long long)k * C + c);
    const float v = (s[0] + s[1]) + (s[2] + s[3]);
    for (int j = 0; j < nrep; ++j) out[((long long)seg * nrep + j) * C + c] = v;
  }
}

// dgate[t, k] for the token's selected slots (0 on unused ones): the column tiles' row dots of
// the slot's row, in order, plus <dY_t, b2_i> (one warp per token)
template <typename S>
__global__ void __launch_bounds__(kEbThreads) dgate_kernel(ExpertBwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kEbThreads / 32) + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int ns = a.n_sel ? a.n_sel[t] : a.K;
  const int nvec = a.D / 8;
  for (int k = 0; k < a.Kmax; ++k) {
    float v = 0.f;
    const int r = k < ns ? a.pos[(long long)t * a.Kmax + k] : -1;
    const int e = k < ns ? a.topk_idx[(long long)t * a.Kmax + k] : -1;
    if (r >= 0 && r < a.rows && e >= 0 && e < a.E) {
      float bsum = 0.f;
      if (a.b2) {
        const uint4* dy = reinterpret_cast<const uint4*>(a.dout) + (long long)t * nvec;
        const uint4* bv = reinterpret_cast<const uint4*>(a.b2) + (long long)e * nvec;
        for (int q = lane; q < nvec; q += 32) {
          float f[8], g[8];
          S::x8_to_f32(__ldg(dy + q), f);
          S::x8_to_f32(__ldg(bv + q), g);
#pragma unroll
          for (int j = 0; j < 8; ++j) bsum = fmaf(f[j], g[j], bsum);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
      }
      float d = 0.f;
      for (int j = 0; j < a.dg_stride; ++j) d += __ldcg(a.dg + (long long)r * a.dg_stride + j);
      v = d + bsum;
    }
    if (lane == 0) a.dgate[(long long)t * a.Kmax + k] = v;
  }
}

int colsum_chunks(long long nrows) { return (int)((nrows + kColChunk - 1) / kColChunk); }

cudaError_t launch_bwd_gather(const ExpertBwdArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)((a.rows + kEbThreads / 32 - 1) / (kEbThreads / 32));
  if (a.f16) bwd_gather_kernel<StoreF16><<<grid, kEbThreads, 0, s>>>(a);
  else bwd_gather_kernel<StoreBF16><<<grid, kEbThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const void* X, long long nrows, int C, const int32_t* offsets, int E, int nrep,
                          float* partial, float* out, int f16, cudaStream_t s) {
  const int nch = colsum_chunks(nrows);
  if (nch > 0) {
    const dim3 g1((unsigned)nch, (unsigned)((C / 2 + kEbThreads - 1) / kEbThreads));
    if (f16) colsum_partial_kernel<StoreF16><<<g1, kEbThreads, 0, s>>>(X, nrows, C, partial);
    else colsum_partial_kernel<StoreBF16><<<g1, kEbThreads, 0, s>>>(X, nrows, C, partial);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const long long n = (long long)(offsets ? E : 1) * C;
  const unsigned g2 = (unsigned)((n + kEbThreads - 1) / kEbThreads);
  colsum_reduce_kernel<<<g2, kEbThreads, 0, s>>>(partial, nch, C, offsets, E, nrep, out);
  return cudaGetLastError();
}

cudaError_t launch_dgate(const ExpertBwdArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)((a.T + kEbThreads / 32 - 1) / (kEbThreads / 32));
  if (a.f16) dgate_kernel<StoreF16><<<grid, kEbThreads, 0, s>>>(a);
  else dgate_kernel<StoreBF16><<<grid, kEbThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
