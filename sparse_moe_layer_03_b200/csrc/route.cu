// Router of the DiT-MoE layer (MoEGate): gate logits x.Wg^T (+ bias), row
// softmax, per-token top-K or the Expert-Race global top-(K*T), per-expert
// counts and the expert-level balance loss.
//
// Sources: "DiT-MoE" hub page, section 1 (MoEGate: weight (E, gating_dim),
// softmax scoring, top_k); "Scaling Diffusion Transformers to 16 Billion
// Parameters", "MOE-DIT" (balance loss eq. L_balance); "Expert Race" abstract
// (tokens and experts compete jointly for the top candidates).
//
// The logits are memory-bound (E FMAs per element of x): x streams through
// shared memory in 128-byte-swizzled column chunks fed by TMA, one or two
// tokens per thread, the gate weight sits in shared memory as fp32 and is read
// by broadcast.  Per-tile partial counts and score sums are reduced in a fixed
// order, so the loss is bit-reproducible.
#include <cuda.h>
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouteThreads = 128;
constexpr int kRouteStages = 3;

size_t route_smem_bytes(int D, int E, int tile_rows, int bf16) {
  (void)bf16;
  size_t wg = (size_t)E * D * sizeof(float);
  wg = (wg + 1023) & ~(size_t)1023;
  // align slack + gate + x stages + barriers (24 B) + counts (<= 128 B) + warp sums (<= 512 B)
  return 1024 + wg + (size_t)kRouteStages * tile_rows * 128 + 1024;
}

template <typename T, int EMAX>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const __grid_constant__ CUtensorMap tmap_x, RouteArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int E = a.E, D = a.D;
  float* wg_s = reinterpret_cast<float*>(smem);
  const size_t wg_bytes = (((size_t)E * D * 4) + 1023) & ~(size_t)1023;
  uint8_t* xs = smem + wg_bytes;
  const int stage_bytes = a.tile_rows * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(xs + (size_t)kRouteStages * stage_bytes);
  int* cnt_s = reinterpret_cast<int*>(full + kRouteStages);          // [EMAX]
  float* wsum_s = reinterpret_cast<float*>(cnt_s + EMAX);             // [4][EMAX]

  constexpr int CC = 128 / (int)sizeof(T);    // columns per 128-byte chunk
  constexpr int VEC = 16 / (int)sizeof(T);    // elements per 16-byte vector
  const int nchunks = D / CC;
  const int tid = threadIdx.x;

  // gate weight -> fp32 shared memory
  const T* wg = reinterpret_cast<const T*>(a.wg);
  for (int i = tid; i < E * D; i += kRouteThreads) wg_s[i] = Elem<T>::to_f(wg[i]);
  if (tid == 0) {
    for (int s = 0; s < kRouteStages; ++s) mbar_init(smem_u32(&full[s]), 1);
    fence_barrier_init();
    prefetch_tmap(&tmap_x);
  }
  __syncthreads();

  const int my_tiles = (a.ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const int items = my_tiles * nchunks;
  auto issue = [&](int item) {
    const int tile = blockIdx.x + (item / nchunks) * gridDim.x;
    const int c = item % nchunks;
    const int s = item % kRouteStages;
    const uint32_t bar = smem_u32(&full[s]);
    mbar_arrive_expect_tx(bar, stage_bytes);
    tma_load_2d(smem_u32(xs + (size_t)s * stage_bytes), &tmap_x, c * CC, tile * a.tile_rows, bar);
  };
  if (tid == 0)
    for (int i = 0; i < kRouteStages && i < items; ++i) issue(i);

  const int r0 = tid, r1 = tid + kRouteThreads;
  const bool has0 = r0 < a.tile_rows, has1 = r1 < a.tile_rows;
  float acc0[EMAX], acc1[EMAX];

  for (int it = 0; it < items; ++it) {
    const int tl = it / nchunks;
    const int c = it % nchunks;
    const int tile = blockIdx.x + tl * gridDim.x;
    if (c == 0) {
#pragma unroll
      for (int e = 0; e < EMAX; ++e) { acc0[e] = 0.f; acc1[e] = 0.f; }
      if (tid < EMAX) cnt_s[tid] = 0;
    }
    const int s = it % kRouteStages;
    const bool ok = mbar_wait(smem_u32(&full[s]), (it / kRouteStages) & 1, nullptr, a.status, 100);
    const uint8_t* st = xs + (size_t)s * stage_bytes;
#pragma unroll 2
    for (int j = 0; j < (ok ? 8 : 0); ++j) {
      float f0[VEC], f1[VEC];
      if (has0) {
        const uint4 v = *reinterpret_cast<const uint4*>(st + r0 * 128 + ((j ^ (r0 & 7)) << 4));
        if constexpr (sizeof(T) == 2) bf16x8_to_f32(v, f0);
        else { f0[0] = __uint_as_float(v.x); f0[1] = __uint_as_float(v.y); f0[2] = __uint_as_float(v.z); f0[3] = __uint_as_float(v.w); }
      }
      if (has1) {
        const uint4 v = *reinterpret_cast<const uint4*>(st + r1 * 128 + ((j ^ (r1 & 7)) << 4));
        if constexpr (sizeof(T) == 2) bf16x8_to_f32(v, f1);
        else { f1[0] = __uint_as_float(v.x); f1[1] = __uint_as_float(v.y); f1[2] = __uint_as_float(v.z); f1[3] = __uint_as_float(v.w); }
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) f1[v] = 0.f;
      }
      const int col = c * CC + j * VEC;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          const float4* wp = reinterpret_cast<const float4*>(wg_s + (size_t)e * D + col);
#pragma unroll
          for (int q = 0; q < VEC / 4; ++q) {
            const float4 w4 = wp[q];
            acc0[e] = fmaf(f0[4 * q + 0], w4.x, acc0[e]);
            acc0[e] = fmaf(f0[4 * q + 1], w4.y, acc0[e]);
            acc0[e] = fmaf(f0[4 * q + 2], w4.z, acc0[e]);
            acc0[e] = fmaf(f0[4 * q + 3], w4.w, acc0[e]);
            acc1[e] = fmaf(f1[4 * q + 0], w4.x, acc1[e]);
            acc1[e] = fmaf(f1[4 * q + 1], w4.y, acc1[e]);
            acc1[e] = fmaf(f1[4 * q + 2], w4.z, acc1[e]);
            acc1[e] = fmaf(f1[4 * q + 3], w4.w, acc1[e]);
          }
        }
      }
    }
    // every thread is done with stage s; a timed-out wait ends the whole block
    if (__syncthreads_or(!ok)) return;
    if (tid == 0 && it + kRouteStages < items) issue(it + kRouteStages);

    if (c == nchunks - 1) {
      // ---- per-token softmax + selection for the (up to) two rows of this thread
      float psum[EMAX];
#pragma unroll
      for (int e = 0; e < EMAX; ++e) psum[e] = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = half ? r1 : r0;
        const bool has = half ? has1 : has0;
        const int tok = tile * a.tile_rows + r;
        if (!has || tok >= a.T) continue;
        float P[EMAX];
        float m = -INFINITY;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
          if (e < E) {
            float l = half ? acc1[e] : acc0[e];
            if (a.bias) l += a.bias[e];
            P[e] = l;
            m = fmaxf(m, l);
          }
        }
        float z = 0.f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e)
          if (e < E) { P[e] = expf(P[e] - m); z += P[e]; }
        const float inv = 1.0f / z;
#pragma unroll
        for (int e = 0; e < EMAX; ++e)
          if (e < E) { P[e] = P[e] * inv; psum[e] += P[e]; }
        if (a.P) {
          float* prow = a.P + (size_t)tok * E;
#pragma unroll
          for (int e = 0; e < EMAX; ++e)
            if (e < E) prow[e] = P[e];
        } else {
          uint32_t taken = 0;
          for (int k = 0; k < a.K; ++k) {
            float bp = -1.f;
            int bi = -1;
#pragma unroll
            for (int e = 0; e < EMAX; ++e)
              if (e < E && !((taken >> e) & 1u) && P[e] > bp) { bp = P[e]; bi = e; }
            if (bi >= 0) { taken |= 1u << bi; atomicAdd(&cnt_s[bi], 1); }
            a.topk_idx[(size_t)tok * a.K + k] = bi;
            a.topk_w[(size_t)tok * a.K + k] = bi >= 0 ? bp : 0.f;
          }
          if (a.n_sel) a.n_sel[tok] = a.K;
        }
      }
      // ---- fixed-order reduction of the score sums: lanes, then warps
      const int w = tid >> 5;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          float v = psum[e];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if ((tid & 31) == 0) wsum_s[w * EMAX + e] = v;
        }
      }
      __syncthreads();
      if (tid < E) {
        const float v = ((wsum_s[tid] + wsum_s[EMAX + tid]) + wsum_s[2 * EMAX + tid]) + wsum_s[3 * EMAX + tid];
        a.tile_psum[(size_t)tile * E + tid] = v;
        if (!a.P) a.tile_counts[(size_t)tile * E + tid] = cnt_s[tid];
      }
      __syncthreads();
    }
  }
}

template <typename T>
static cudaError_t launch_route_t(const RouteArgs& a, const CUtensorMap* tm, cudaStream_t s) {
  const size_t smem = route_smem_bytes(a.D, a.E, a.tile_rows, a.bf16);
  cudaError_t err;
#define MOE_ROUTE_CASE(EM)                                                                     \
  if (a.E <= EM) {                                                                             \
    err = cudaFuncSetAttribute(route_kernel<T, EM>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                               (int)smem);                                                     \
    if (err != cudaSuccess) return err;                                                        \
    route_kernel<T, EM><<<a.grid, kRouteThreads, smem, s>>>(*tm, a);                           \
    return cudaGetLastError();                                                                 \
  }
  MOE_ROUTE_CASE(8)
  MOE_ROUTE_CASE(16)
  MOE_ROUTE_CASE(32)
#undef MOE_ROUTE_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_route(const RouteArgs& a, const CUtensorMap* tm, cudaStream_t s) {
  return a.bf16 ? launch_route_t<__nv_bfloat16>(a, tm, s) : launch_route_t<float>(a, tm, s);
}

// ---------------------------------------------------------------- finalize
// counts_i = sum over tiles; p_i = (1/T) sum over tiles (fp64, fixed order);
// L = alpha * sum_i (E/(K T)) counts_i p_i.
__global__ void __launch_bounds__(256) route_finalize_kernel(FinalizeArgs a) {
  __shared__ double red[256];
  __shared__ double loss_terms[32];
  const int tid = threadIdx.x;
  for (int e = 0; e < a.E; ++e) {
    long long c = 0;
    double p = 0.0;
    for (int t = tid; t < a.ntiles_counts; t += 256) c += a.tile_counts[(size_t)t * a.E + e];
    for (int t = tid; t < a.ntiles_psum; t += 256) p += (double)a.tile_psum[(size_t)t * a.E + e];
    red[tid] = (double)c;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
      if (tid < o) red[tid] += red[tid + o];
      __syncthreads();
    }
    const double cnt = red[0];
    __syncthreads();
    red[tid] = p;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
      if (tid < o) red[tid] += red[tid + o];
      __syncthreads();
    }
    if (tid == 0) {
      a.counts[e] = (int32_t)cnt;
      loss_terms[e] = ((double)a.E / ((double)a.K * a.T)) * cnt * (red[0] / a.T);
    }
    __syncthreads();
  }
  if (tid == 0) {
    double L = 0.0;
    for (int e = 0; e < a.E; ++e) L += loss_terms[e];
    *a.aux_loss = (float)(a.alpha * L);
  }
}

cudaError_t launch_route_finalize(const FinalizeArgs& a, cudaStream_t s) {
  route_finalize_kernel<<<1, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- Expert-Race
// Exact radix select of the S-th largest score over the T x E matrix on the
// fp32 bit patterns (scores are >= 0, so the unsigned order of the bits is the
// numeric order): 12 + 12 + 8 bits.  state[0] = prefix so far, state[1] =
// winners still needed inside the current bin, state[2] = threshold bits,
// state[3] = winners to take among the entries equal to the threshold.
constexpr int kRaceTile = 128;

__global__ void __launch_bounds__(256) race_hist_kernel(const uint32_t* __restrict__ bits, long long n,
                                                       int pass, const uint32_t* __restrict__ state,
                                                       uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[4096];
  for (int i = threadIdx.x; i < 4096; i += 256) h[i] = 0;
  __syncthreads();
  const uint32_t prefix = pass ? state[0] : 0u;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n; i += (long long)gridDim.x * 256) {
    const uint32_t b = bits[i];
    if (pass == 0) atomicAdd(&h[b >> 20], 1u);
    else if (pass == 1) { if ((b >> 20) == prefix) atomicAdd(&h[(b >> 8) & 0xFFFu], 1u); }
    else { if ((b >> 8) == prefix) atomicAdd(&h[b & 0xFFu], 1u); }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 4096; i += 256)
    if (h[i]) atomicAdd(&hist[i], h[i]);
}

// one block of 1024 threads: pick the bin holding the needed rank, from the top
__global__ void __launch_bounds__(1024) race_find_kernel(uint32_t* hist, uint32_t* state, int pass,
                                                         uint32_t S) {
  __shared__ uint32_t part[1024];
  const int nb = pass == 2 ? 256 : 4096;
  const int per = nb / 1024 > 0 ? nb / 1024 : 1;
  const int tid = threadIdx.x;
  const uint32_t need = pass ? state[1] : S;
  // thread i owns bins (from the top) [i*per, i*per+per) when i*per < nb
  uint32_t local = 0;
  if (tid * per < nb)
    for (int j = 0; j < per; ++j) local += hist[nb - 1 - (tid * per + j)];
  part[tid] = local;
  __syncthreads();
  // inclusive scan (Hillis-Steele) over 1024 partial sums
  for (int o = 1; o < 1024; o <<= 1) {
    const uint32_t v = tid >= o ? part[tid - o] : 0u;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  uint32_t above = tid ? part[tid - 1] : 0u;
  if (tid * per < nb) {
    for (int j = 0; j < per; ++j) {
      const int bin = nb - 1 - (tid * per + j);
      const uint32_t h = hist[bin];
      if (above < need && above + h >= need) {
        const uint32_t prefix = pass == 0 ? (uint32_t)bin
                              : pass == 1 ? ((state[0] << 12) | (uint32_t)bin)
                                          : ((state[0] << 8) | (uint32_t)bin);
        state[0] = prefix;
        state[1] = need - above;
        if (pass == 2) { state[2] = prefix; state[3] = need - above; }
      }
      above += h;
    }
  }
  __syncthreads();
  for (int i = tid; i < 4096; i += 1024) hist[i] = 0;   // ready for the next pass
}

// entries equal to the threshold, per tile of 128 tokens
__global__ void __launch_bounds__(kRaceTile) race_count_eq_kernel(const uint32_t* __restrict__ bits,
                                                                 int T, int E, const uint32_t* state,
                                                                 uint32_t* tile_eq) {
  __shared__ uint32_t wsum[kRaceTile / 32];
  const uint32_t thr = state[2];
  const int t = blockIdx.x * kRaceTile + threadIdx.x;
  uint32_t c = 0;
  if (t < T)
    for (int e = 0; e < E; ++e) c += bits[(size_t)t * E + e] == thr;
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t s = 0;
    for (int w = 0; w < kRaceTile / 32; ++w) s += wsum[w];
    tile_eq[blockIdx.x] = s;
  }
}

template <int EMAX>
__global__ void __launch_bounds__(kRaceTile) race_select_kernel(RaceArgs a) {
  __shared__ uint32_t scan[kRaceTile];
  __shared__ int cnt_s[EMAX];
  __shared__ uint32_t base_s;
  const int tid = threadIdx.x;
  const int E = a.E;
  const uint32_t thr = a.state[2], need_eq = a.state[3];
  if (tid < EMAX) cnt_s[tid] = 0;
  if (tid == 0) {
    uint32_t b = 0;
    for (int i = 0; i < (int)blockIdx.x; ++i) b += a.tile_eq[i];
    base_s = b;
  }
  const int t = blockIdx.x * kRaceTile + tid;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(a.P);
  uint32_t v[EMAX];
  uint32_t my_eq = 0;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    v[e] = (t < a.T && e < E) ? bits[(size_t)t * E + e] : 0u;
    my_eq += (t < a.T && e < E && v[e] == thr) ? 1u : 0u;
  }
  scan[tid] = my_eq;
  __syncthreads();
  for (int o = 1; o < kRaceTile; o <<= 1) {
    const uint32_t x = tid >= o ? scan[tid - o] : 0u;
    __syncthreads();
    scan[tid] += x;
    __syncthreads();
  }
  const bool valid = t < a.T;
  if (valid) {
    uint32_t rank = base_s + scan[tid] - my_eq;   // equal entries before this token
    uint32_t chosen = 0;
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        bool sel = v[e] > thr;
        if (v[e] == thr) { sel = rank < need_eq; ++rank; }
        if (sel) chosen |= 1u << e;
      }
    }
    // winners of this token in descending score, ties to the lower expert id
    int n = 0;
    uint32_t left = chosen;
    while (left) {
      uint32_t bv = 0;
      int bi = -1;
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (((left >> e) & 1u) && (bi < 0 || v[e] > bv)) { bv = v[e]; bi = e; }
      left &= ~(1u << bi);
      a.topk_idx[(size_t)t * E + n] = bi;
      a.topk_w[(size_t)t * E + n] = __uint_as_float(bv);
      atomicAdd(&cnt_s[bi], 1);
      ++n;
    }
    for (int k = n; k < E; ++k) {
      a.topk_idx[(size_t)t * E + k] = -1;
      a.topk_w[(size_t)t * E + k] = 0.f;
    }
    a.n_sel[t] = n;
  }
  __syncthreads();
  if (tid < E) a.tile_counts[(size_t)blockIdx.x * E + tid] = cnt_s[tid];
}

cudaError_t launch_race_select(const RaceArgs& a, cudaStream_t s) {
  const long long n = (long long)a.T * a.E;
  const uint32_t S = (uint32_t)((long long)a.K * a.T);
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(a.P);
  int hist_grid = (int)((n + 256 * 8 - 1) / (256 * 8));
  if (hist_grid > 1184) hist_grid = 1184;
  if (hist_grid < 1) hist_grid = 1;
  for (int pass = 0; pass < 3; ++pass) {
    race_hist_kernel<<<hist_grid, 256, 0, s>>>(bits, n, pass, a.state, a.hist);
    race_find_kernel<<<1, 1024, 0, s>>>(a.hist, a.state, pass, S);
  }
  race_count_eq_kernel<<<a.ntiles, kRaceTile, 0, s>>>(bits, a.T, a.E, a.state, a.tile_eq);
  if (a.E <= 8) race_select_kernel<8><<<a.ntiles, kRaceTile, 0, s>>>(a);
  else if (a.E <= 16) race_select_kernel<16><<<a.ntiles, kRaceTile, 0, s>>>(a);
  else race_select_kernel<32><<<a.ntiles, kRaceTile, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
