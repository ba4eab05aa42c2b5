// Backward of the expert-level balance loss through the router
// ("Scaling Diffusion Transformers to 16 Billion Parameters", "MOE-DIT",
// eq. L_balance).  L = alpha sum_i f_i p_i with f_i = (E/(K T)) counts_i from
// the discrete selection (no gradient) and p_i = (1/T) sum_t P[t,i], so
// dL/dP[t,i] = alpha f_i / T = c_i for every token, and through the softmax
//     dl[t,i] = P[t,i] (c_i - sum_j P[t,j] c_j).
// The router's linear map l = x Wg^T + b then gives dWg = dl^T x, db = sum_t dl
// and dx = dl Wg.
//
// token kernel (one warp per token, the gate weight in shared memory): the row
//   of x in 16-byte vectors, E partial dot products per lane and a fixed xor
//   tree, softmax and dl (every lane), the dx row, dl written out, and the
//   block's db partial (warps in a fixed order).
// wgrad kernel: blocks over (chunk of kWgTokens tokens, 512 columns); each
//   thread owns 2 columns x E experts and walks its chunk's tokens in order.
// reduce kernel: the chunk partials of dWg and the block partials of db,
//   summed in order.  Every sum has a fixed order: bit-reproducible.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kBwdThreads = 256;
constexpr int kWgTokens = 256;
constexpr int kWgCols = 2 * kBwdThreads;

template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void to_f(const uint4& v, float* f) { bf16x8_to_f32(v, f); }
  static __device__ __forceinline__ uint4 from_f(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
};
template <> struct Vec16<__half> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void to_f(const uint4& v, float* f) { f16x8_to_f32(v, f); }
  static __device__ __forceinline__ uint4 from_f(const float* f) {
    return make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]), pack_f16x2(f[4], f[5]), pack_f16x2(f[6], f[7]));
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void to_f(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y); f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  static __device__ __forceinline__ uint4 from_f(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

template <typename T, int EMAX>
__global__ void __launch_bounds__(kBwdThreads) balance_grad_token_kernel(BalanceGradArgs a) {
  using V = Vec16<T>;
  constexpr int NW = kBwdThreads / 32;
  extern __shared__ __align__(16) uint8_t wsm[];     // gate weight [E, D] act, as given
  __shared__ float c_s[EMAX];
  __shared__ float wdb[NW][EMAX];
  const int D = a.D, E = a.E, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nv = D / V::N;                           // 16-byte vectors per row
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.wg);
    uint4* dst = reinterpret_cast<uint4*>(wsm);
    for (int i = tid; i < E * nv; i += kBwdThreads) dst[i] = __ldg(src + i);
  }
  if (tid < EMAX)
    c_s[tid] = tid < E ? a.scale * a.alpha * ((float)E / ((float)a.K * a.T)) * (float)a.counts[tid] / (float)a.T : 0.f;
  __syncthreads();
  const uint4* wv = reinterpret_cast<const uint4*>(wsm);
  float dbw[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) dbw[e] = 0.f;
  for (int t = blockIdx.x * NW + w; t < a.T; t += gridDim.x * NW) {
    const uint4* xr = reinterpret_cast<const uint4*>(a.x) + (size_t)t * nv;
    float l[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) l[e] = 0.f;
    for (int v = lane; v < nv; v += 32) {
      float xf[V::N];
      V::to_f(__ldg(xr + v), xf);          // default caching: the wgrad kernel reads x next
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          float wf[V::N];
          V::to_f(wv[e * nv + v], wf);
#pragma unroll
          for (int q = 0; q < V::N; ++q) l[e] = fmaf(xf[q], wf[q], l[e]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], o);
    }
    // softmax and dl, the same in every lane
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] += a.bias ? a.bias[e] : 0.f; m = fmaxf(m, l[e]); }
    float z = 0.f;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] = expf(l[e] - m); z += l[e]; }
    const float iz = 1.0f / z;
    float pc = 0.f;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] *= iz; pc += l[e] * c_s[e]; }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      l[e] = e < E ? l[e] * (c_s[e] - pc) : 0.f;      // dl
      dbw[e] += l[e];
    }
    if (lane < E) {
      float v = 0.f;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) v = e == lane ? l[e] : v;
      a.dl[(size_t)t * E + lane] = v;
    }
    if (a.dx) {
      uint4* dxr = reinterpret_cast<uint4*>(a.dx) + (size_t)t * nv;
      for (int v = lane; v < nv; v += 32) {
        float o[V::N];
#pragma unroll
        for (int q = 0; q < V::N; ++q) o[q] = 0.f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
          if (e < E) {
            float wf[V::N];
            V::to_f(wv[e * nv + v], wf);
#pragma unroll
            for (int q = 0; q < V::N; ++q) o[q] = fmaf(l[e], wf[q], o[q]);
          }
        }
        dxr[v] = V::from_f(o);
      }
    }
  }
  // db partial of this block: lane 0's sums (every lane holds the same), warps in order
  if (lane == 0) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e) wdb[w][e] = dbw[e];
  }
  __syncthreads();
  if (tid < E) {
    float s = 0.f;
    for (int k = 0; k < NW; ++k) s += wdb[k][tid];
    a.db_part[(size_t)blockIdx.x * E + tid] = s;
  }
}

// dWg partial of one chunk of tokens: thread (column pair) accumulates E x 2 sums in token order
template <typename T, int EMAX>
__global__ void __launch_bounds__(kBwdThreads) balance_grad_wg_kernel(BalanceGradArgs a) {
  __shared__ float dls[kWgTokens][EMAX];
  const int D = a.D, E = a.E, tid = threadIdx.x;
  const int chunk = blockIdx.x, t0 = chunk * kWgTokens;
  const int nt = min(kWgTokens, a.T - t0);
  for (int i = tid; i < nt * EMAX; i += kBwdThreads) {
    const int t = i / EMAX, e = i % EMAX;
    dls[t][e] = e < E ? a.dl[(size_t)(t0 + t) * E + e] : 0.f;
  }
  __syncthreads();
  const int c = blockIdx.y * kWgCols + 2 * tid;      // this thread's two columns
  if (c >= D) return;
  float acc[EMAX][2];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) { acc[e][0] = 0.f; acc[e][1] = 0.f; }
  const T* x = reinterpret_cast<const T*>(a.x);
#pragma unroll 8
  for (int t = 0; t < nt; ++t) {
    float x0, x1;
    if (sizeof(T) == 2) {   // the column pair as one 4-byte load
      const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(x + (size_t)(t0 + t) * D + c));
      T h[2];
      *reinterpret_cast<uint32_t*>(h) = v;
      x0 = Elem<T>::to_f(h[0]);
      x1 = Elem<T>::to_f(h[1]);
    } else {
      const float2 v = __ldg(reinterpret_cast<const float2*>(x + (size_t)(t0 + t) * D + c));
      x0 = v.x;
      x1 = v.y;
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      acc[e][0] = fmaf(dls[t][e], x0, acc[e][0]);
      acc[e][1] = fmaf(dls[t][e], x1, acc[e][1]);
    }
  }
  float* part = a.partials + (size_t)chunk * E * D;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
      part[(size_t)e * D + c] = acc[e][0];
      part[(size_t)e * D + c + 1] = acc[e][1];
    }
  }
}

// Fixed-order sums of the partials: eight interleaved running sums (partial p goes to sum
// p % 8), added up in order at the end, so eight loads are in flight per thread.
__device__ __forceinline__ float sum_strided(const float* p, int n, size_t stride) {
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int k = 0;
  for (; k + 8 <= n; k += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) s[u] += __ldcg(p + (size_t)(k + u) * stride);
  }
  for (int u = 0; k < n; ++k, ++u) s[u] += __ldcg(p + (size_t)k * stride);
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

__global__ void __launch_bounds__(kBwdThreads) balance_grad_reduce_kernel(BalanceGradArgs a, int nchunks, int nblocks) {
  const int n = a.E * a.D;
  for (int i = blockIdx.x * kBwdThreads + threadIdx.x; i < n + a.E; i += gridDim.x * kBwdThreads) {
    if (i < n) a.dwg[i] = sum_strided(a.partials + i, nchunks, (size_t)n);
    else if (a.dbias) a.dbias[i - n] = sum_strided(a.db_part + (i - n), nblocks, (size_t)a.E);
  }
}

int balance_grad_chunks(int T) { return (T + kWgTokens - 1) / kWgTokens; }

template <typename T, int EM>
static cudaError_t launch_bg(const BalanceGradArgs& a, int blocks, cudaStream_t s) {
  const size_t smem = (size_t)a.E * a.D * (a.dtype == 0 ? 4 : 2);
  cudaError_t e = cudaFuncSetAttribute(balance_grad_token_kernel<T, EM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  balance_grad_token_kernel<T, EM><<<blocks, kBwdThreads, smem, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 g2((unsigned)balance_grad_chunks(a.T), (unsigned)((a.D + kWgCols - 1) / kWgCols));
  balance_grad_wg_kernel<T, EM><<<g2, kBwdThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_bg_t(const BalanceGradArgs& a, int blocks, cudaStream_t s) {
  if (a.E <= 8) return launch_bg<T, 8>(a, blocks, s);
  if (a.E <= 16) return launch_bg<T, 16>(a, blocks, s);
  return launch_bg<T, 32>(a, blocks, s);
}

cudaError_t launch_balance_grad(const BalanceGradArgs& a, int blocks, cudaStream_t s) {
  cudaError_t e = a.dtype == 0 ? launch_bg_t<float>(a, blocks, s)
                  : a.dtype == 2 ? launch_bg_t<__half>(a, blocks, s)
                                 : launch_bg_t<__nv_bfloat16>(a, blocks, s);
  if (e != cudaSuccess) return e;
  const int n = a.E * a.D + a.E;
  balance_grad_reduce_kernel<<<(n + kBwdThreads - 1) / kBwdThreads, kBwdThreads, 0, s>>>(
      a, balance_grad_chunks(a.T), blocks);
  return cudaGetLastError();
}

}  // namespace moe
