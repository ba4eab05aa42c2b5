// Dispatch: permute tokens into expert-contiguous blocks so that only the
// selected experts are computed ("Scaling Diffusion Transformers to 16 Billion
// Parameters", "MOE 回顾": with a sparse g, unused experts need not be run).
//
// Layout: expert i owns rows [P_i, P_i + counts_i), P_i = sum_{j<i}
// round_up(counts_j, 256), tokens ascending inside a segment.  Positions come
// from integer counts and prefix sums only (no order-dependent atomics), so
// the permutation is deterministic and equals the canonical one bit for bit.
//
//   count kernel  (1 block per chunk of tokens): per-chunk expert counts.
//   gather kernel (1 block per chunk): sums of the chunk counts give the
//                 padded segment starts and the chunk's base in each segment;
//                 ranks inside the chunk by warp ballots; positions; padding
//                 rows marked; 16-byte row copies x -> x_perm.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kGatherThreads = 256;

// per-chunk expert counts, expert-major: cnt[e * nchunks + c]
__global__ void __launch_bounds__(kGatherThreads) dispatch_count_kernel(DispatchArgs a) {
  __shared__ int cc[32];
  const int tid = threadIdx.x, c = blockIdx.x, Kmax = a.Kmax;
  if (tid < 32) cc[tid] = 0;
  __syncthreads();
  const int t0 = c * a.chunk;
  const int n = min(a.chunk, a.T - t0) * Kmax;
  for (int i = tid; i < n; i += kGatherThreads) {
    const int t = t0 + i / Kmax, k = i % Kmax;
    const int ns = a.n_sel ? a.n_sel[t] : a.K;
    if (k >= ns) continue;
    const int e = a.topk_idx[(size_t)t0 * Kmax + i];
    if (e >= 0 && e < a.E) atomicAdd(&cc[e], 1);
  }
  __syncthreads();
  if (tid < a.E) a.chunk_base[(size_t)tid * a.nchunks + c] = cc[tid];
}

template <typename T, int EMAX>
__global__ void __launch_bounds__(kGatherThreads) dispatch_gather_kernel(DispatchArgs a) {
  extern __shared__ int sm[];
  const int Kmax = a.Kmax, E = a.E, CH = a.chunk;
  int* sidx = sm;                     // [CH][Kmax] expert of each slot (-1 unused)
  int* spos = sm + CH * Kmax;         // [CH][Kmax] rank in warp, then row
  __shared__ int wcnt[kGatherThreads / 32][EMAX];
  __shared__ int before_s[EMAX], total_s[EMAX], poff_s[EMAX + 1];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int c = blockIdx.x;
  const int t0 = c * CH;

  // ---- segment starts and this chunk's base: sums over the chunk counts
  for (int e = w; e < E; e += kGatherThreads / 32) {
    const int* row = a.chunk_base + (size_t)e * a.nchunks;
    int before = 0, total = 0;
#pragma unroll 4
    for (int j = lane; j < a.nchunks; j += 32) {
      const int v = row[j];
      total += v;
      before += j < c ? v : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
    }
    if (lane == 0) { total_s[e] = total; before_s[e] = before; }
  }
  __syncthreads();
  if (tid == 0) {
    int p = 0;
    for (int e = 0; e < E; ++e) { poff_s[e] = p; p += (total_s[e] + kSegAlign - 1) / kSegAlign * kSegAlign; }
    poff_s[E] = p;
  }
  __syncthreads();
  if (c == 0 && tid <= E) {
    int u = 0;
    for (int e = 0; e < tid; ++e) u += total_s[e];
    a.offsets[tid] = u;
  }
  // padding rows: segment e's tail (e < E) or the rows after the last segment (e = E)
  for (int e = c; e <= E; e += gridDim.x) {
    const long long lo = e < E ? (long long)poff_s[e] + total_s[e] : poff_s[E];
    const long long hi = e < E ? (long long)poff_s[e + 1] : a.r_max;
    for (long long r = lo + tid; r < hi; r += kGatherThreads) {
      a.row_token[r] = -1;
      a.row_gate[r] = 0.f;
    }
  }

  // ---- slots of this chunk
  for (int i = tid; i < CH * Kmax; i += kGatherThreads) {
    const int l = i / Kmax, k = i % Kmax, t = t0 + l;
    int e = -1;
    if (t < a.T) {
      const int ns = a.n_sel ? a.n_sel[t] : a.K;
      if (k < ns) {
        e = a.topk_idx[(size_t)t * Kmax + k];
        if (e >= E) { set_status(a.status, DEV_BAD_INDEX, 200); e = -1; }
      }
    }
    sidx[i] = e < 0 ? -1 : e;
    spos[i] = -1;
  }
  __syncthreads();
  // ---- rank of each token among the chunk's tokens of the same expert (token order)
  if (w < CH / 32) {
    const int l = w * 32 + lane;
    for (int e = 0; e < E; ++e) {
      int slot = -1;
      for (int k = 0; k < Kmax; ++k)
        if (sidx[l * Kmax + k] == e) slot = k;
      const unsigned mask = __ballot_sync(0xffffffffu, slot >= 0);
      if (slot >= 0) spos[l * Kmax + slot] = __popc(mask & ((1u << lane) - 1u));
      if (lane == 0) wcnt[w][e] = __popc(mask);
    }
  }
  __syncthreads();
  for (int i = tid; i < CH * Kmax; i += kGatherThreads) {
    const int l = i / Kmax, k = i % Kmax, t = t0 + l;
    if (t >= a.T) continue;
    const int e = sidx[i];
    int p = -1;
    if (e >= 0) {
      int base = poff_s[e] + before_s[e];
      for (int ww = 0; ww < l / 32; ++ww) base += wcnt[ww][e];
      p = base + spos[i];
      if (p < 0 || p >= a.r_max) { set_status(a.status, DEV_BAD_INDEX, 201); p = -1; }
      else {
        a.row_token[p] = t;
        a.row_gate[p] = a.topk_w[(size_t)t * Kmax + k];
      }
    }
    a.pos[(size_t)t * Kmax + k] = p;
    spos[i] = p;
  }
  __syncthreads();
  // ---- row copies: one warp per token, 16-byte vectors
  const int nvec = a.D * (int)sizeof(T) / 16;
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  uint4* xp = reinterpret_cast<uint4*>(a.x_perm);
  for (int l = w; l < CH; l += kGatherThreads / 32) {
    const int t = t0 + l;
    if (t >= a.T) break;
    const uint4* src = xv + (size_t)t * nvec;
    for (int v0 = 0; v0 < nvec; v0 += 32 * 4) {
      uint4 buf[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < nvec) buf[u] = src[v];
      }
      for (int k = 0; k < Kmax; ++k) {
        const int p = spos[l * Kmax + k];
        if (p < 0) continue;
        uint4* dst = xp + (size_t)p * nvec;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < nvec) dst[v] = buf[u];
        }
      }
    }
  }
}

template <typename T>
static cudaError_t launch_gather_t(const DispatchArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)2 * a.chunk * a.Kmax * sizeof(int);
  cudaError_t err = cudaSuccess;
  if (a.E <= 8) err = cudaFuncSetAttribute(dispatch_gather_kernel<T, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  else if (a.E <= 16) err = cudaFuncSetAttribute(dispatch_gather_kernel<T, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  else err = cudaFuncSetAttribute(dispatch_gather_kernel<T, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (a.E <= 8) dispatch_gather_kernel<T, 8><<<a.nchunks, kGatherThreads, smem, s>>>(a);
  else if (a.E <= 16) dispatch_gather_kernel<T, 16><<<a.nchunks, kGatherThreads, smem, s>>>(a);
  else dispatch_gather_kernel<T, 32><<<a.nchunks, kGatherThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s) {
  dispatch_count_kernel<<<a.nchunks, kGatherThreads, 0, s>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return a.bf16 ? launch_gather_t<__nv_bfloat16>(a, s) : launch_gather_t<float>(a, s);
}

}  // namespace moe
