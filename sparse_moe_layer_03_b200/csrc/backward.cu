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

// ---------------------------------------------------------------- bf16: on mma.sync
// Rows of 16 tokens come in by TMA (two half-row boxes per stage, 128-byte swizzle, a ring of
// kRmStages stages refilled as soon as every warp has left the block).  Per block: each of the
// 16 warps takes every 16th k16 step for the partial logits x Wg^T (as the forward router); the
// first 256 threads add the 16 partials in warp order; one thread per (token, expert) computes
// softmax and dl (the token's lanes reduce by shuffles), written to shared memory as two bf16
// parts (dl = hi + lo, about 16 bits of mantissa); then every warp, on its own contiguous slice of the D/8 8-column
// tiles, forms dx = dl Wg (two MMAs, written to global memory; the experts' part, loaded first
// for all of the slice's tiles at once, added when asked) and accumulates dWg += dl^T x in
// registers over all of the CTA's blocks (x read straight from the stage with transposed
// ldmatrix).  Sixteen warps per SM keep enough MMAs and loads in flight: with four, the SM
// waited on single dependences most of the time.  E <= 16 (zero-padded to 16), D <= 1152.
// With E <= 8 the two parts of dl share one MMA's k = 16: dl is held as [hi | lo] per token and
// the gate weight as [Wg; Wg], so dx takes one MMA per tile, and dWg's tile gets the hi part in
// rows 0-7 and the lo part in rows 8-15 (added when the partials are written).
constexpr int kRmWarps = 16;
constexpr int kRmStages = 4;
constexpr int kRmMaxNT = 9;                       // 8-column tiles per warp: ceil(D / 8 / kRmWarps)

struct RmSmem {
  size_t wg, x, dl, lp, ls, db, misc, total;
  int hc, stage_bytes, wg_stride;
};
__host__ __device__ inline RmSmem rm_layout(int D) {
  RmSmem L;
  L.hc = (D / 64 + 1) / 2;
  L.stage_bytes = 16 * 2 * L.hc * 128;
  L.wg_stride = D * 2 + 16;
  L.wg = 0;
  L.x = ((size_t)16 * L.wg_stride + 1023) & ~(size_t)1023;
  L.dl = L.x + (size_t)kRmStages * L.stage_bytes;
  L.lp = L.dl + 2 * 16 * 16 * 2;                   // dl hi and lo, [16 tokens][16 experts] bf16 each
  L.ls = L.lp + (size_t)kRmWarps * 16 * 16 * 4;    // partial logits [warp][token][expert] fp32
  L.db = L.ls + 16 * 16 * 4;                       // logits [token][expert] fp32
  L.misc = L.db + 16 * 16 * 4;                     // db per (token, expert) thread
  L.total = L.misc + 256 + 1024;                   // barriers; 1 KB alignment slack
  return L;
}

bool router_bwd_mma_fits(int D, int E, int dtype) {
  if (dtype != 1 || E > 16 || D % 64 || (D / 8 + kRmWarps - 1) / kRmWarps > kRmMaxNT) return false;
  return rm_layout(D).total <= 232448;
}
size_t router_bwd_mma_smem(int D) { return rm_layout(D).total; }

template <int EMAX>
__global__ void __launch_bounds__(kRmWarps * 32, 1)
router_bwd_mma_kernel(const __grid_constant__ CUtensorMap tmap_x, BalanceGradArgs a) {
  constexpr int NTE = EMAX / 8;                    // expert tiles of the logits
  constexpr bool PACK = EMAX == 8;                 // hi and lo parts of dl in one k16 step
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const RmSmem L = rm_layout(a.D);
  const int D = a.D, E = a.E, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, c = lane & 3, li = lane >> 3, lj = lane & 7;
  const int nks = D / 16, ntiles = D / 8;
  const int tb = w * ntiles / kRmWarps, te = (w + 1) * ntiles / kRmWarps;   // this warp's 8-column tiles
  uint8_t* wg_s = smem + L.wg;
  uint8_t* xs = smem + L.x;
  uint16_t* dlh = reinterpret_cast<uint16_t*>(smem + L.dl);
  uint16_t* dll = dlh + 16 * 16;
  float* lp = reinterpret_cast<float*>(smem + L.lp);
  float* ls = reinterpret_cast<float*>(smem + L.ls);
  float* dbs = reinterpret_cast<float*>(smem + L.db);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.misc);
  __shared__ float c_s[16];
  const int nrb = (a.T + 15) / 16;
  const int my_rb = (nrb - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  auto issue = [&](int j) {                        // thread 0: row block j of this CTA into its stage
    const int st = j % kRmStages;
    const int rb = blockIdx.x + j * gridDim.x;
    const uint32_t bar = smem_u32(&full[st]);
    const uint32_t dst = smem_u32(xs + (size_t)st * L.stage_bytes);
    mbar_arrive_expect_tx(bar, (uint32_t)L.stage_bytes);
    tma_load_3d(dst, &tmap_x, 0, rb * 16, 0, bar);
    tma_load_3d(dst + L.hc * 2048, &tmap_x, 0, rb * 16, L.hc, bar);
  };
  if (tid < 16)
    c_s[tid] = tid < E ? a.scale * a.alpha * ((float)E / ((float)a.K * a.T)) * (float)a.counts[tid] / (float)a.T : 0.f;
  if (tid < 256) dbs[tid] = 0.f;
  // Gate weight rows 0..15 (zero past E; rows 8..15 repeat rows 0..7 when packed), padded stride:
  // bulk copies of whole rows, issued before any x load (loaded by the threads after the x loads,
  // the weight's reads queued behind every CTA's x stream); then the x stages.
  uint64_t* wbar = full + 8;
  if (tid == 0) {
    mbar_init(smem_u32(wbar), 1);
    for (int st = 0; st < kRmStages; ++st) mbar_init(smem_u32(&full[st]), 1);
    fence_barrier_init();
    int nrows = 0;
    for (int e = 0; e < 16; ++e) nrows += (PACK ? (e & 7) : e) < E ? 1 : 0;
    mbar_arrive_expect_tx(smem_u32(wbar), (uint32_t)(nrows * D * 2));
    for (int e = 0; e < 16; ++e) {
      const int src = PACK ? (e & 7) : e;
      if (src < E)
        bulk_load(smem_u32(wg_s + (size_t)e * L.wg_stride), reinterpret_cast<const uint8_t*>(a.wg) + (size_t)src * D * 2,
                  (uint32_t)(D * 2), smem_u32(wbar));
    }
    for (int j = 0; j < kRmStages && j < my_rb; ++j) issue(j);
  }
  {  // the rows of no expert are zero
    const int vpr = D / 8;
    for (int i = tid; i < 16 * vpr; i += blockDim.x) {
      const int e = i / vpr;
      if ((PACK ? (e & 7) : e) >= E) *reinterpret_cast<uint4*>(wg_s + (size_t)e * L.wg_stride + (i % vpr) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();
  mbar_wait(smem_u32(wbar), 0, nullptr, nullptr, 121);
  const uint32_t wg_base = smem_u32(wg_s);
  float acc[kRmMaxNT][4];
#pragma unroll
  for (int i = 0; i < kRmMaxNT; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
  bool ok = true;
  for (int j = 0; j < my_rb; ++j) {
    const int st = j % kRmStages;
    const int rb = blockIdx.x + j * gridDim.x;
    // a wait that ran out once makes every later block skip its work; the barriers still run
    // (no status word here: the router backward's scratch has none; a wait that ran out still ends the kernel)
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), (j / kRmStages) & 1, nullptr, nullptr, 120));
    const uint32_t xb = smem_u32(xs + (size_t)st * L.stage_bytes);
    // ---- partial logits of this warp's k16 steps
    float la[NTE][4];
#pragma unroll
    for (int nt = 0; nt < NTE; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) la[nt][q] = 0.f;
    if (ok) {
      for (int sk = w; sk < nks; sk += kRmWarps) {
        const int ks = sk & 3;
        const uint32_t box = xb + (sk >> 2) * 2048;
        uint32_t bb[NTE][2];
        const int kc = sk * 16 + (li & 1) * 8;
#pragma unroll
        for (int np = 0; np < NTE; np += 2) {
          if (np + 1 < NTE) {
            const int n = (np + (li >> 1)) * 8 + lj;
            ldsm_x4(wg_base + n * L.wg_stride + kc * 2, bb[np][0], bb[np][1], bb[np + 1][0], bb[np + 1][1]);
          } else {
            ldsm_x2(wg_base + (np * 8 + lj) * L.wg_stride + kc * 2, bb[np][0], bb[np][1]);
          }
        }
        const int row = (li & 1) * 8 + lj;
        const int chunk = ks * 2 + (li >> 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(box + row * 128 + ((chunk ^ (row & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NTE; ++nt) mma_16816<false>(la[nt], a0, a1, a2, a3, bb[nt][0], bb[nt][1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTE; ++nt) {
      float* pw = lp + (size_t)w * 256;
      pw[g * 16 + nt * 8 + 2 * c] = la[nt][0];
      pw[g * 16 + nt * 8 + 2 * c + 1] = la[nt][1];
      pw[(g + 8) * 16 + nt * 8 + 2 * c] = la[nt][2];
      pw[(g + 8) * 16 + nt * 8 + 2 * c + 1] = la[nt][3];
    }
    __syncthreads();
    // every warp has left block j - 1: its stage takes block j - 1 + kRmStages
    if (tid == 0 && j >= 1 && j - 1 + kRmStages < my_rb) {
      fence_async_shared();
      issue(j - 1 + kRmStages);
    }
    if (tid < 256) {                               // the logits: the warps' partials in warp order
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < kRmWarps; ++k) v += lp[k * 256 + tid];
      ls[tid] = v;
    }
    __syncthreads();
    // ---- softmax and dl of the block's 16 tokens: thread (token, expert) of the first 16 * EMAX,
    // the token's EMAX lanes reducing by shuffles
    if (tid < 16 * EMAX) {
      const int tl_ = tid / EMAX, e = tid % EMAX;
      const int t = rb * 16 + tl_;
      const bool act = e < E;
      float l = ls[tl_ * 16 + e] + (act && a.bias ? a.bias[e] : 0.f);
      float m = act ? l : -INFINITY;
#pragma unroll
      for (int o = 1; o < EMAX; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float pe = act ? expf(l - m) : 0.f;
      float z = pe;
#pragma unroll
      for (int o = 1; o < EMAX; o <<= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      pe *= 1.0f / z;
      float dp = c_s[e];
      const bool valid = t < a.T && ok;
      if (a.dgate && valid) {
        const int ns = a.n_sel ? a.n_sel[t] : a.K;
        for (int k = 0; k < a.Kmax && k < ns; ++k)
          if (a.topk_idx[(size_t)t * a.Kmax + k] == e) dp += a.dgate[(size_t)t * a.Kmax + k];
      }
      float pc = pe * dp;
#pragma unroll
      for (int o = 1; o < EMAX; o <<= 1) pc += __shfl_xor_sync(0xffffffffu, pc, o);
      const float dl = (act && valid) ? pe * (dp - pc) : 0.f;
      dbs[tid] += dl;
      const __nv_bfloat16 h = __float2bfloat16_rn(dl);
      const __nv_bfloat16 lo = __float2bfloat16_rn(dl - __bfloat162float(h));
      // packed: [hi of experts 0..7 | lo of experts 0..7] in one row; else hi and lo rows apart
      reinterpret_cast<__nv_bfloat16*>(dlh)[tl_ * 16 + e] = h;
      reinterpret_cast<__nv_bfloat16*>(PACK ? dlh + 8 : dll)[tl_ * 16 + e] = lo;
    }
    __syncthreads();
    // ---- dx = dl Wg and dWg += dl^T x on this warp's 8-column tiles
    if (ok) {
      const int t0 = rb * 16 + g, t1 = t0 + 8;
      const bool v0 = t0 < a.T, v1 = t1 < a.T;
      // rows t0 and t1 of dx, as bf16 pairs; this lane's pair of each tile sits at (tile * 8 + 2c) / 2
      uint32_t* dx0 = reinterpret_cast<uint32_t*>(a.dx) + ((size_t)t0 * D + 2 * c) / 2;
      uint32_t* dx1 = dx0 + (size_t)8 * D / 2;
      // the experts' part of dx for every tile of the slice, in flight together
      uint32_t prev[kRmMaxNT][2];
#pragma unroll
      for (int i = 0; i < kRmMaxNT; ++i) {
        prev[i][0] = prev[i][1] = 0u;
        if (a.dx && a.dx_accumulate && tb + i < te) {
          if (v0) prev[i][0] = __ldcg(reinterpret_cast<const unsigned int*>(dx0 + (tb + i) * 4));
          if (v1) prev[i][1] = __ldcg(reinterpret_cast<const unsigned int*>(dx1 + (tb + i) * 4));
        }
      }
      uint32_t ah[4], al[4], th[4], tl[4];
      {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8, cb = (lane >> 4) * 8;   // A = dl [t][e]
        ldsm_x4(smem_u32(dlh + r * 16 + cb), ah[0], ah[1], ah[2], ah[3]);
        const int mi = lane >> 3, tt = (mi >> 1) * 8 + (lane & 7), e0 = (mi & 1) * 8;  // A = dl^T [e][t]
        ldsm_x4_t(smem_u32(dlh + tt * 16 + e0), th[0], th[1], th[2], th[3]);
        if (!PACK) {
          ldsm_x4(smem_u32(dll + r * 16 + cb), al[0], al[1], al[2], al[3]);
          ldsm_x4_t(smem_u32(dll + tt * 16 + e0), tl[0], tl[1], tl[2], tl[3]);
        }
      }
      const int rr = lane & 15;                    // row of the 8x8 tiles this lane addresses
      const uint32_t wrow = wg_base + rr * L.wg_stride;
      const uint32_t xrow = xb + rr * 128;
#pragma unroll
      for (int i = 0; i < kRmMaxNT; ++i) {
        if (tb + i < te) {
          const int tile = tb + i;
          uint32_t b0, b1, x0, x1;
          ldsm_x2_t(wrow + tile * 16, b0, b1);                                    // B = Wg [e][d]
          ldsm_x2_t(xrow + (tile >> 3) * 2048 + (((tile & 7) ^ (rr & 7)) << 4), x0, x1);   // B = x [t][d]
          float d4[4] = {0.f, 0.f, 0.f, 0.f};
          mma_16816<false>(d4, ah[0], ah[1], ah[2], ah[3], b0, b1);
          mma_16816<false>(acc[i], th[0], th[1], th[2], th[3], x0, x1);
          if (!PACK) {
            mma_16816<false>(d4, al[0], al[1], al[2], al[3], b0, b1);
            mma_16816<false>(acc[i], tl[0], tl[1], tl[2], tl[3], x0, x1);
          }
          if (a.dx) {
            if (v0) {
              const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&prev[i][0]));
              const __nv_bfloat162 v = __floats2bfloat162_rn(d4[0] + p.x, d4[1] + p.y);
              dx0[tile * 4] = *reinterpret_cast<const uint32_t*>(&v);
            }
            if (v1) {
              const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&prev[i][1]));
              const __nv_bfloat162 v = __floats2bfloat162_rn(d4[2] + p.x, d4[3] + p.y);
              dx1[tile * 4] = *reinterpret_cast<const uint32_t*>(&v);
            }
          }
        }
      }
    }
  }
  // ---- this CTA's partial dWg (rows e = g, g + 8 of its fragments) and db (tokens in order)
  float* part = a.partials + (size_t)blockIdx.x * E * D;
#pragma unroll
  for (int i = 0; i < kRmMaxNT; ++i) {
    if (tb + i < te) {
      const int col = (tb + i) * 8 + 2 * c;
      if (PACK) {                                  // rows g (hi part) and g + 8 (lo part) of expert g
        if (g < E) {
          part[(size_t)g * D + col] = acc[i][0] + acc[i][2];
          part[(size_t)g * D + col + 1] = acc[i][1] + acc[i][3];
        }
      } else {
        if (g < E) { part[(size_t)g * D + col] = acc[i][0]; part[(size_t)g * D + col + 1] = acc[i][1]; }
        if (g + 8 < E) { part[(size_t)(g + 8) * D + col] = acc[i][2]; part[(size_t)(g + 8) * D + col + 1] = acc[i][3]; }
      }
    }
  }
  __syncthreads();
  if (tid < E) {                                   // thread (token, expert) slots of the expert, in order
    float sdb = 0.f;
    for (int k = 0; k < 16; ++k) sdb += dbs[k * EMAX + tid];
    a.db_part[(size_t)blockIdx.x * E + tid] = sdb;
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
  if (a.mma_grid > 0) {
    // bf16 on mma.sync: partials of dWg and db per CTA
    const size_t smem = router_bwd_mma_smem(a.D);
    if (a.E <= 8) {
      e = cudaFuncSetAttribute(router_bwd_mma_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) router_bwd_mma_kernel<8><<<a.mma_grid, kRmWarps * 32, smem, s>>>(*a.tmap_x, a);
    } else {
      e = cudaFuncSetAttribute(router_bwd_mma_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) router_bwd_mma_kernel<16><<<a.mma_grid, kRmWarps * 32, smem, s>>>(*a.tmap_x, a);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    nparts = nchunks = a.mma_grid;
  } else if (a.pass_grid > 0) {
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
