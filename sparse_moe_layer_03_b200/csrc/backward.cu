// Backward of the router: the expert-level balance loss ("Scaling Diffusion
// Transformers to 16 Billion Parameters", "MOE-DIT", eq. L_balance) and, for the
// whole layer's backward, the gates' gradient.  L = alpha sum_i f_i p_i with
// f_i = (E/(K T)) counts_i from the discrete selection (no gradient) and
// p_i = (1/T) sum_t P[t,i], so dL/dP[t,i] = alpha f_i / T = c_i for every token;
// the gates g = P on the selected slots add dgate there.  Through the softmax
//     dl[t,i] = P[t,i] (dP[t,i] - sum_j P[t,j] dP[t,j]),
// and the router's linear map l = x Wg^T + b gives dWg = dl^T x, db = sum_t dl
// and dx = dl Wg.
//
// One pass kernel (rows of at most 2048 16-bit or 1024 fp32 values): CTA b owns
// a contiguous range of tokens.  Phase 1, one warp per token (the next token's
// row already loading into registers): logits from the gate weight in shared
// memory, a fixed xor tree, softmax and dl in every lane, the dx row written
// (added to the experts' part when asked), dl kept in shared memory.  Phase 2,
// each thread owns 8 (or 4) columns and adds dl^T x over the CTA's tokens in
// order (x read again, from L2), giving the CTA's partial dWg.
// Wider rows use the older three-kernel path (token kernel, chunked wgrad).
// A reduce kernel sums the partials of dWg and db in order: bit-reproducible.
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
    // dJ/dP: the balance term c_i on every entry, plus the gates' gradient on the selected slots
    float dp[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) dp[e] = c_s[e];
    if (a.dgate) {
      const int ns = a.n_sel ? a.n_sel[t] : a.K;
      for (int k = 0; k < a.Kmax && k < ns; ++k) {
        const int sel = a.topk_idx[(size_t)t * a.Kmax + k];
        const float gk = a.dgate[(size_t)t * a.Kmax + k];
#pragma unroll
        for (int e = 0; e < EMAX; ++e) dp[e] += e == sel ? gk : 0.f;
      }
    }
    float pc = 0.f;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] *= iz; pc += l[e] * dp[e]; }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      l[e] = e < E ? l[e] * (dp[e] - pc) : 0.f;       // dl
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
        if (a.dx_accumulate) V::to_f(dxr[v], o);       // the experts' part of dx, then the router's
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

constexpr int kRbThreads = 256;
constexpr int kRbMaxV = 8;                         // 16-byte vectors per lane and row (D <= 2048 16-bit)

template <typename T, int EMAX>
__global__ void __launch_bounds__(kRbThreads, 2) router_bwd_pass_kernel(BalanceGradArgs a, int tpc) {
  using V = Vec16<T>;
  constexpr int NW = kRbThreads / 32;
  extern __shared__ __align__(16) uint8_t rsm[];    // gate weight [E, D] act, then dl [tpc, EMAX] fp32
  __shared__ float c_s[EMAX];
  __shared__ float wdb[NW][EMAX];
  const int D = a.D, E = a.E, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nv = D / V::N;
  const int t0 = blockIdx.x * tpc, t1 = min(a.T, t0 + tpc);
  float* dls = reinterpret_cast<float*>(rsm + (size_t)E * D * sizeof(T));
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.wg);
    uint4* dst = reinterpret_cast<uint4*>(rsm);
    for (int i = tid; i < E * nv; i += kRbThreads) dst[i] = __ldg(src + i);
  }
  if (tid < EMAX)
    c_s[tid] = tid < E ? a.scale * a.alpha * ((float)E / ((float)a.K * a.T)) * (float)a.counts[tid] / (float)a.T : 0.f;
  __syncthreads();
  const uint4* wv = reinterpret_cast<const uint4*>(rsm);
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  float dbw[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) dbw[e] = 0.f;
  // ---- phase 1: one warp per token
  uint4 cur[kRbMaxV], nxt[kRbMaxV];
  int t = t0 + w;
  if (t < t1) {
#pragma unroll
    for (int k = 0; k < kRbMaxV; ++k) {
      const int v = lane + 32 * k;
      if (v < nv) cur[k] = __ldg(xv + (size_t)t * nv + v);
    }
  }
  for (; t < t1; t += NW) {
    const int tn = t + NW;
    if (tn < t1) {                                   // the next row loads while this one is worked on
#pragma unroll
      for (int k = 0; k < kRbMaxV; ++k) {
        const int v = lane + 32 * k;
        if (v < nv) nxt[k] = __ldg(xv + (size_t)tn * nv + v);
      }
    }
    float l[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) l[e] = 0.f;
#pragma unroll
    for (int k = 0; k < kRbMaxV; ++k) {
      const int v = lane + 32 * k;
      if (v < nv) {
        float xf[V::N];
        V::to_f(cur[k], xf);
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
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], o);
    }
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] += a.bias ? a.bias[e] : 0.f; m = fmaxf(m, l[e]); }
    float z = 0.f;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] = expf(l[e] - m); z += l[e]; }
    const float iz = 1.0f / z;
    float dp[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) dp[e] = c_s[e];
    if (a.dgate) {
      const int ns = a.n_sel ? a.n_sel[t] : a.K;
      for (int k = 0; k < a.Kmax && k < ns; ++k) {
        const int sel = a.topk_idx[(size_t)t * a.Kmax + k];
        const float gk = a.dgate[(size_t)t * a.Kmax + k];
#pragma unroll
        for (int e = 0; e < EMAX; ++e) dp[e] += e == sel ? gk : 0.f;
      }
    }
    float pc = 0.f;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) { l[e] *= iz; pc += l[e] * dp[e]; }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      l[e] = e < E ? l[e] * (dp[e] - pc) : 0.f;       // dl
      dbw[e] += l[e];
    }
    if (lane < EMAX) {
      float v = 0.f;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) v = e == lane ? l[e] : v;
      dls[(size_t)(t - t0) * EMAX + lane] = v;
    }
    if (a.dx) {
      uint4* dxr = reinterpret_cast<uint4*>(a.dx) + (size_t)t * nv;
#pragma unroll
      for (int k = 0; k < kRbMaxV; ++k) {
        const int v = lane + 32 * k;
        if (v < nv) {
          float o[V::N];
#pragma unroll
          for (int q = 0; q < V::N; ++q) o[q] = 0.f;
          if (a.dx_accumulate) V::to_f(dxr[v], o);
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
#pragma unroll
    for (int k = 0; k < kRbMaxV; ++k) cur[k] = nxt[k];
  }
  if (lane == 0) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e) wdb[w][e] = dbw[e];
  }
  __syncthreads();
  if (tid < E) {
    float sdb = 0.f;
    for (int k = 0; k < NW; ++k) sdb += wdb[k][tid];
    a.db_part[(size_t)blockIdx.x * E + tid] = sdb;
  }
  // ---- phase 2: this CTA's dWg partial, column vector v of every expert over the CTA's tokens
  const int ntok = t1 - t0;
  float* part = a.partials + (size_t)blockIdx.x * E * D;
  for (int v = tid; v < nv; v += kRbThreads) {
    for (int e0 = 0; e0 < E; e0 += 8) {
      float acc[8][V::N];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int q = 0; q < V::N; ++q) acc[j][q] = 0.f;
      // eight rows in flight per thread, then their products in token order
      for (int tb = 0; tb < ntok; tb += 8) {
        uint4 xr[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (tb + u < ntok) xr[u] = __ldg(xv + (size_t)(t0 + tb + u) * nv + v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (tb + u < ntok) {
            float xf[V::N];
            V::to_f(xr[u], xf);
            const float* dr = dls + (size_t)(tb + u) * EMAX + e0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float d = dr[j];
#pragma unroll
              for (int q = 0; q < V::N; ++q) acc[j][q] = fmaf(d, xf[q], acc[j][q]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (e0 + j < E) {
#pragma unroll
          for (int q = 0; q < V::N; ++q) part[(size_t)(e0 + j) * D + v * V::N + q] = acc[j][q];
        }
    }
  }
}

// Block b sums elements [32 b, 32 b + 32) of [dWg, db]: lane = element, warp w takes the partials
// p = w, w + 8, ... in order (eight loads in flight per lane), then the eight warp sums are added
// in warp order.  A fixed order throughout.
__global__ void __launch_bounds__(kBwdThreads) balance_grad_reduce_kernel(BalanceGradArgs a, int nchunks, int nblocks) {
  constexpr int NW = kBwdThreads / 32;
  __shared__ float ws[NW][32];
  const int n = a.E * a.D;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (i < n + a.E) {
    const bool wg = i < n;
    const float* p = wg ? a.partials + i : a.db_part + (i - n);
    const size_t stride = wg ? (size_t)n : (size_t)a.E;
    const int cnt = wg ? nchunks : nblocks;
    float r[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int k = w, u = 0;
    for (; k < cnt; k += NW, u = (u + 1) & 7) r[u] += __ldcg(p + (size_t)k * stride);
    s = ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
  }
  ws[w][lane] = s;
  __syncthreads();
  if (w == 0 && i < n + a.E) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < NW; ++k) t += ws[k][lane];
    if (i < n) a.dwg[i] = t;
    else if (a.dbias) a.dbias[i - n] = t;
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

template <typename T, int EM>
static cudaError_t launch_rb(const BalanceGradArgs& a, int grid, int tpc, cudaStream_t s) {
  const size_t smem = (size_t)a.E * a.D * sizeof(T) + (size_t)tpc * EM * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(router_bwd_pass_kernel<T, EM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  router_bwd_pass_kernel<T, EM><<<grid, kRbThreads, smem, s>>>(a, tpc);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_rb_t(const BalanceGradArgs& a, int grid, int tpc, cudaStream_t s) {
  if (a.E <= 8) return launch_rb<T, 8>(a, grid, tpc, s);
  if (a.E <= 16) return launch_rb<T, 16>(a, grid, tpc, s);
  return launch_rb<T, 32>(a, grid, tpc, s);
}

int router_bwd_pass_grid(int T, int sms, int* tpc) {
  int g = 2 * sms;                                 // two CTAs per SM
  if (g > kBwdMaxBlocks) g = kBwdMaxBlocks;
  if (g > T) g = T > 0 ? T : 1;
  const int per = (T + g - 1) / g;
  *tpc = per > 0 ? per : 1;
  return (T + *tpc - 1) / *tpc;
}

bool router_bwd_pass_fits(int D, int E, int dtype, int T, int sms) {
  const int vec = dtype == 0 ? 4 : 8;
  if (D % vec || D / vec > 32 * kRbMaxV) return false;
  int tpc = 0;
  router_bwd_pass_grid(T, sms, &tpc);
  const int em = E <= 8 ? 8 : (E <= 16 ? 16 : 32);
  const size_t smem = (size_t)E * D * (dtype == 0 ? 4 : 2) + (size_t)tpc * em * 4;
  return smem <= 232448 / 2 - 2048;               // two CTAs per SM
}

cudaError_t launch_balance_grad(const BalanceGradArgs& a, int blocks, cudaStream_t s) {
  cudaError_t e;
  int nparts = blocks, nchunks = balance_grad_chunks(a.T);
  if (a.pass_grid > 0) {
    // one pass: partials of dWg and db per CTA
    e = a.dtype == 0 ? launch_rb_t<float>(a, a.pass_grid, a.pass_tpc, s)
        : a.dtype == 2 ? launch_rb_t<__half>(a, a.pass_grid, a.pass_tpc, s)
                       : launch_rb_t<__nv_bfloat16>(a, a.pass_grid, a.pass_tpc, s);
    nparts = nchunks = a.pass_grid;
  } else {
    e = a.dtype == 0 ? launch_bg_t<float>(a, blocks, s)
        : a.dtype == 2 ? launch_bg_t<__half>(a, blocks, s)
                       : launch_bg_t<__nv_bfloat16>(a, blocks, s);
  }
  if (e != cudaSuccess) return e;
  const int n = a.E * a.D + a.E;
  balance_grad_reduce_kernel<<<(n + 31) / 32, kBwdThreads, 0, s>>>(a, nchunks, nparts);
  return cudaGetLastError();
}

}  // namespace moe
