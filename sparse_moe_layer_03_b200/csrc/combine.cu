// Combine: MoE(x_t) = sum_{i in sel_t} g_{t,i} e_i(x_t) + sum_j s_j(x_t)
// ("Scaling Diffusion Transformers to 16 Billion Parameters", "MOE 回顾"
// eq. MoE(x) and "MOE-DIT" shared experts).  The gates were applied in the
// second expert GEMM's epilogue, so this is an un-permute and a sum: fp32 in
// slot order k = 0..n_sel-1, then the shared term; with the adaLN-Zero residual
// ("Scalable Diffusion Models with Transformers (DiT)", DiT block details)
// out = x_res + alpha_image * that sum; rounded once.
// HBM-bound: one warp per token, 16-byte loads.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kCombineThreads = 256;

// 8 consecutive elements as fp32
template <typename T> __device__ __forceinline__ void load8(const T* p, size_t i, float* f);
template <> __device__ __forceinline__ void load8<float>(const float* p, size_t i, float* f) {
  const float4 a = reinterpret_cast<const float4*>(p)[2 * i], b = reinterpret_cast<const float4*>(p)[2 * i + 1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, size_t i, float* f) {
  bf16x8_to_f32(reinterpret_cast<const uint4*>(p)[i], f);
}
template <> __device__ __forceinline__ void load8<__half>(const __half* p, size_t i, float* f) {
  f16x8_to_f32(reinterpret_cast<const uint4*>(p)[i], f);
}
__device__ __forceinline__ uint32_t pack2(const __nv_bfloat16*, float lo, float hi) { return pack_bf16x2(lo, hi); }
__device__ __forceinline__ uint32_t pack2(const __half*, float lo, float hi) { return pack_f16x2(lo, hi); }

template <typename T>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a) {
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (kCombineThreads / 32);
  const int n8 = a.D / 8;
  const T* yp = reinterpret_cast<const T*>(a.y_perm);
  const T* ys = reinterpret_cast<const T*>(a.y_sh);
  const T* xr = reinterpret_cast<const T*>(a.x_res);
  const T* al = reinterpret_cast<const T*>(a.alpha);
  for (int t = blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5); t < a.T; t += nwarps) {
    int ns = a.n_sel ? a.n_sel[t] : a.K;
    ns = ns < 0 ? 0 : (ns > a.Kmax ? a.Kmax : ns);
    int rows[32];
    for (int k = 0; k < ns; ++k) {
      const int p = a.pos[(size_t)t * a.Kmax + k];
      rows[k] = (p >= 0 && p < a.r_max) ? p : -1;
    }
    for (int v = lane; v < n8; v += 32) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int k = 0; k < ns; ++k) {
        if (rows[k] < 0) continue;
        float y[8];
        load8<T>(yp, (size_t)rows[k] * n8 + v, y);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += y[q];
      }
      if (ys) {
        float y[8];
        load8<T>(ys, (size_t)t * n8 + v, y);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += y[q];
      }
      if (xr) {   // adaLN-Zero: the residual plus the image's gate times the layer output
        float r[8], g[8];
        load8<T>(xr, (size_t)t * n8 + v, r);
        load8<T>(al, (size_t)(t / a.img_len) * n8 + v, g);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = r[q] + g[q] * acc[q];
      }
      if constexpr (sizeof(T) == 2) {
        const T* tag = nullptr;
        uint4 o;
        o.x = pack2(tag, acc[0], acc[1]);
        o.y = pack2(tag, acc[2], acc[3]);
        o.z = pack2(tag, acc[4], acc[5]);
        o.w = pack2(tag, acc[6], acc[7]);
        reinterpret_cast<uint4*>(a.out)[(size_t)t * n8 + v] = o;
      } else {
        float4* o = reinterpret_cast<float4*>(a.out) + (size_t)t * 2 * n8 + 2 * v;
        o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  int grid = (a.T + 7) / 8;
  if (grid > 148 * 16) grid = 148 * 16;
  if (a.b16 && a.f16) combine_kernel<__half><<<grid, kCombineThreads, 0, s>>>(a);
  else if (a.b16) combine_kernel<__nv_bfloat16><<<grid, kCombineThreads, 0, s>>>(a);
  else combine_kernel<float><<<grid, kCombineThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
