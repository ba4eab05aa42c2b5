// Combine: MoE(x_t) = sum_{i in sel_t} g_{t,i} e_i(x_t) + sum_j s_j(x_t)
// ("Scaling Diffusion Transformers to 16 Billion Parameters", "MOE 回顾"
// eq. MoE(x) and "MOE-DIT" shared experts).  The gates were applied in the
// second expert GEMM's epilogue, so this is an un-permute and a sum: fp32 in
// slot order k = 0..n_sel-1, then the shared term, rounded once.
// HBM-bound: one warp per token, 16-byte loads of fp32 rows.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kCombineThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a) {
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (kCombineThreads / 32);
  const int n4 = a.D / 4;
  const float4* yp = reinterpret_cast<const float4*>(a.y_perm);
  const float4* ys = reinterpret_cast<const float4*>(a.y_sh);
  for (int t = blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5); t < a.T; t += nwarps) {
    int ns = a.n_sel ? a.n_sel[t] : a.K;
    ns = ns < 0 ? 0 : (ns > a.Kmax ? a.Kmax : ns);
    int rows[32];
    for (int k = 0; k < ns; ++k) {
      const int p = a.pos[(size_t)t * a.Kmax + k];
      rows[k] = (p >= 0 && p < a.r_max) ? p : -1;
    }
    for (int v = lane; v < n4; v += 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < ns; ++k) {
        if (rows[k] < 0) continue;
        const float4 y = yp[(size_t)rows[k] * n4 + v];
        acc.x += y.x; acc.y += y.y; acc.z += y.z; acc.w += y.w;
      }
      if (ys) {
        const float4 y = ys[(size_t)t * n4 + v];
        acc.x += y.x; acc.y += y.y; acc.z += y.z; acc.w += y.w;
      }
      if constexpr (sizeof(T) == 2) {
        uint2 o;
        o.x = pack_bf16x2(acc.x, acc.y);
        o.y = pack_bf16x2(acc.z, acc.w);
        reinterpret_cast<uint2*>(a.out)[(size_t)t * n4 + v] = o;
      } else {
        reinterpret_cast<float4*>(a.out)[(size_t)t * n4 + v] = acc;
      }
    }
  }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  int grid = (a.T + 7) / 8;
  if (grid > 148 * 16) grid = 148 * 16;
  if (a.bf16) combine_kernel<__nv_bfloat16><<<grid, kCombineThreads, 0, s>>>(a);
  else combine_kernel<float><<<grid, kCombineThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
