// Dispatch: permute tokens into expert-contiguous blocks so that only the
// selected experts are computed ("Scaling Diffusion Transformers to 16 Billion
// Parameters", "MOE 回顾": with a sparse g, unused experts need not be run).
//
// Layout: expert i owns rows [P_i, P_i + counts_i), P_i = sum_{j<i}
// round_up(counts_j, 128), tokens ascending inside a segment.  Positions come
// from integer counts and prefix sums only (no order-dependent atomics), so
// the permutation is deterministic and equals the canonical one bit for bit.
//
//   plan kernel   (1 block): per-chunk expert counts -> prefix over chunks ->
//                 offsets, padded offsets, chunk bases; marks padding rows.
//   gather kernel (1 block per chunk of tokens): ranks inside the chunk by warp
//                 ballots, positions, then 16-byte row copies x -> x_perm.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kPlanThreads = 1024;
constexpr int kGatherThreads = 256;

// exclusive scan of one value per thread over a 1024-thread block
__device__ __forceinline__ int block_excl_scan_1024(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;   // inclusive totals of warps
  }
  __syncthreads();
  const int before = (w ? warp_tot[w - 1] : 0) + x - v;
  total = warp_tot[31];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kPlanThreads) dispatch_plan_kernel(DispatchArgs a) {
  extern __shared__ int cc[];   // [nchunks][E]
  __shared__ int warp_tot[32];
  __shared__ int tot[33], poff[33];
  const int tid = threadIdx.x;
  const int E = a.E, Kmax = a.Kmax;
  for (int i = tid; i < a.nchunks * E; i += kPlanThreads) cc[i] = 0;
  __syncthreads();
  const long long npairs = (long long)a.T * Kmax;
  for (long long i = tid; i < npairs; i += kPlanThreads) {
    const int t = (int)(i / Kmax), k = (int)(i % Kmax);
    const int ns = a.n_sel ? a.n_sel[t] : a.K;
    if (k >= ns) continue;
    const int e = a.topk_idx[i];
    if (e >= 0 && e < E) atomicAdd(&cc[(t / a.chunk) * E + e], 1);
  }
  __syncthreads();
  for (int e = 0; e < E; ++e) {
    const int v = tid < a.nchunks ? cc[tid * E + e] : 0;
    int total;
    const int before = block_excl_scan_1024(v, warp_tot, total);
    if (tid < a.nchunks) cc[tid * E + e] = before;
    if (tid == 0) tot[e] = total;
  }
  __syncthreads();
  if (tid == 0) {
    int u = 0, p = 0;
    for (int e = 0; e < E; ++e) {
      a.offsets[e] = u;
      poff[e] = p;
      u += tot[e];
      p += (tot[e] + 127) / 128 * 128;
    }
    a.offsets[E] = u;
    poff[E] = p;
  }
  __syncthreads();
  for (int i = tid; i < a.nchunks * E; i += kPlanThreads) a.chunk_base[i] = poff[i % E] + cc[i];
  // padding rows: inside each segment after its last token, and after the last segment
  for (int e = 0; e <= E; ++e) {
    const long long lo = e < E ? (long long)poff[e] + tot[e] : poff[E];
    const long long hi = e < E ? (long long)poff[e + 1] : a.r_max;
    for (long long r = lo + tid; r < hi; r += kPlanThreads) {
      a.row_token[r] = -1;
      a.row_gate[r] = 0.f;
    }
  }
}

template <typename T, int EMAX>
__global__ void __launch_bounds__(kGatherThreads) dispatch_gather_kernel(DispatchArgs a) {
  extern __shared__ int sm[];
  const int Kmax = a.Kmax, E = a.E, CH = a.chunk;
  int* sidx = sm;                     // [CH][Kmax] expert of each slot (-1 unused)
  int* spos = sm + CH * Kmax;         // [CH][Kmax] rank in warp, then row
  __shared__ int wcnt[kGatherThreads / 32][EMAX];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int c = blockIdx.x;
  const int t0 = c * CH;

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
      int base = a.chunk_base[(size_t)c * E + e];
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
  // row copies: one warp per token, 16-byte vectors
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
  const size_t smem = (size_t)a.nchunks * a.E * sizeof(int);
  cudaError_t err = cudaFuncSetAttribute(dispatch_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dispatch_plan_kernel<<<1, kPlanThreads, smem, s>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  return a.bf16 ? launch_gather_t<__nv_bfloat16>(a, s) : launch_gather_t<float>(a, s);
}

}  // namespace moe
