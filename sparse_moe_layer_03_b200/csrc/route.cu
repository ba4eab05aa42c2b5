// Router of the DiT-MoE layer (MoEGate): gate logits x.Wg^T (+ bias), row
// softmax, per-token top-K or the Expert-Race global top-(K*T), per-expert
// counts and the expert-level balance loss.
//
// Sources: "DiT-MoE" hub page, section 1 (MoEGate: weight (E, gating_dim),
// softmax scoring, top_k); "Scaling Diffusion Transformers to 16 Billion
// Parameters", "MOE-DIT" (balance loss eq. L_balance); "Expert Race" abstract
// (tokens and experts compete jointly for the top candidates).
//
// The logits are HBM-bound: x streams through shared memory once, in
// 128-byte-swizzled column chunks fed by TMA.  bf16 inputs take their E dot
// products on mma.sync (the FP32 pipe alone cannot keep up with HBM at E = 16);
// fp32 inputs use FFMA.  Per-tile partial counts and score sums are reduced in
// a fixed order, so the loss is bit-reproducible.
#include <cuda.h>
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouteThreads = 128;     // FFMA kernel (fp32 inputs)
constexpr int kRouteStages = 4;

__host__ __device__ inline int route_emax(int E) { return E <= 8 ? 8 : (E <= 16 ? 16 : 32); }
__host__ __device__ inline size_t align1k(size_t v) { return (v + 1023) & ~(size_t)1023; }

// Shared-memory layout of both router kernels (bytes from the 1024-aligned base):
//   gate weight | x stages (tile_rows x 128 B each) | logits (mma only) | barriers, counts, sums
struct RouteSmem {
  size_t wg, x, logits, misc, total;
};
__host__ __device__ inline RouteSmem route_layout(int D, int E, int tile_rows, int bf16) {
  RouteSmem L;
  const int em = route_emax(E);
  L.wg = 0;
  const size_t wg_bytes = bf16 ? (size_t)em * (D * 2 + 16) : (size_t)E * D * 4;
  L.x = align1k(wg_bytes);
  // the x stages double as the finalize scratch (2 x 32 x 33 x 8 bytes) at the end
  const size_t xb = (size_t)kRouteStages * tile_rows * 128;
  L.logits = L.x + (xb > 16896 ? xb : 16896);
  L.misc = L.logits + (bf16 ? (size_t)tile_rows * em * 4 : 0);
  // barriers (4 x 8 B) + counts (<= 32 x 4 B) + warp sums (8 x 32 x 4 B)
  L.total = 1024 /*alignment slack*/ + L.misc + 2048;
  return L;
}

size_t route_smem_bytes(int D, int E, int tile_rows, int bf16) {
  return route_layout(D, E, tile_rows, bf16).total;
}

// Per token: bias, softmax, then top-K selection (or the score row for
// Expert-Race); score sums and counts accumulate for the balance loss.
template <int EMAX>
__device__ __forceinline__ void token_select(const float* logit, int tok, const RouteArgs& a, int* cnt_s,
                                             float* psum) {
  const int E = a.E;
  float P[EMAX];
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
      float l = logit[e];
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
    return;
  }
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

// Fixed-order reduction of the per-thread score sums (lanes, then warps) and
// the tile's partial outputs.  Every thread of the block calls it.
template <int EMAX>
__device__ __forceinline__ void tile_partials(const float* psum, int tile, const RouteArgs& a, const int* cnt_s,
                                              float* wsum_s) {
  const int tid = threadIdx.x, w = tid >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < a.E) {
      float v = psum[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((tid & 31) == 0) wsum_s[w * EMAX + e] = v;
    }
  }
  __syncthreads();
  if (tid < a.E) {
    float v = 0.f;
    for (int k = 0; k < nw; ++k) v += wsum_s[k * EMAX + tid];
    a.tile_psum[(size_t)tile * a.E + tid] = v;
    if (!a.P) a.tile_counts[(size_t)tile * a.E + tid] = cnt_s[tid];
  }
  __syncthreads();
}

// ---------------------------------------------------------------- bf16: tensor-core logits
// Work unit = a block of 16 consecutive tokens: their full rows (16 x D bf16,
// one contiguous stretch of HBM, so DRAM pages are read whole) land in one
// pair of shared-memory stages (one per half of the row, each one 3-D TMA box of
// 64-column blocks x 16 rows, 128-byte swizzle).  Each warp owns two stages,
// takes every NC-th row block and issues its own loads: wait for a half,
// compute its part of the 16 x E logits with mma.sync m16n8k16 (A via ldmatrix
// from the swizzled stage, B = gate weight in shared memory with rows padded by
// 16 bytes), refill that stage with the next row block's half (the load
// overlaps the other half's MMAs and the epilogue), then run softmax and
// selection (one lane per token).  No block-wide barrier inside the loop and no
// warp waits on another warp's progress.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kMmaRB = 16;        // tokens per row block
constexpr int kMmaMaxConsumers = 6;

// A row block is loaded as two halves (column blocks [0, hc) and [hc, 2hc), hc =
// ceil(D/128)), each into its own stage; warp c owns stages 2c and 2c+1, issues
// their loads itself and waits on their phases strictly in order.  As many warps
// (<= 6) as the shared memory allows.
struct MmaSmem {
  size_t wg, x, logits, misc, total;
  int consumers, hc;
};
__host__ __device__ inline MmaSmem mma_layout(int D, int E) {
  MmaSmem L;
  const int em = route_emax(E);
  L.hc = (D / 64 + 1) / 2;
  L.wg = 0;
  L.x = align1k((size_t)em * (D * 2 + 16));
  const size_t stage = (size_t)kMmaRB * L.hc * 128;
  L.consumers = 0;
  for (int nc = kMmaMaxConsumers; nc >= 1; --nc) {
    const size_t xb = 2 * nc * stage;
    const size_t total = L.x + (xb > 16896 ? xb : 16896) + (size_t)nc * kMmaRB * em * 4 + 2048 + 1024;
    if (total + 1024 <= 232448) { L.consumers = nc; break; }
  }
  const int nc = L.consumers > 0 ? L.consumers : 1;
  const size_t xb = 2 * nc * stage;
  L.logits = L.x + (xb > 16896 ? xb : 16896);   // x stages double as the finalize scratch
  L.misc = L.logits + (size_t)nc * kMmaRB * em * 4;
  L.total = L.misc + 2048 + 1024;
  return L;
}

// The last block to finish turns the per-block partials into counts and the loss.
// Every thread loads its tiles' partials for all experts at once (no chain of
// dependent loads), then fixed-order shuffle trees and a fixed warp order make
// the result bit-reproducible.  scratch: 2 x 32 x 32 x 8 bytes of shared memory.
constexpr int kFinalizeScratch = 2 * 32 * 32 * 8;
template <int EMAX>
__device__ void finalize_counts_loss(const FinalizeArgs& a, uint8_t* scratch) {
  auto wc = reinterpret_cast<long long(*)[32]>(scratch);
  auto wp = reinterpret_cast<double(*)[32]>(scratch + 32 * 32 * 8);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  const int E = a.E;
  long long c[EMAX];
  double p[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) { c[e] = 0; p[e] = 0.0; }
  const int nt = a.ntiles_counts > a.ntiles_psum ? a.ntiles_counts : a.ntiles_psum;
  for (int t = tid; t < nt; t += blockDim.x) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        if (t < a.ntiles_counts) c[e] += __ldcg(a.tile_counts + (size_t)t * E + e);
        if (t < a.ntiles_psum) p[e] += (double)__ldcg(a.tile_psum + (size_t)t * E + e);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        c[e] += __shfl_xor_sync(0xffffffffu, c[e], o);
        p[e] += __shfl_xor_sync(0xffffffffu, p[e], o);
      }
      if (lane == 0) { wc[w][e] = c[e]; wp[w][e] = p[e]; }
    }
  }
  __syncthreads();
  if (tid < 32) {
    long long cc = 0;
    double pp = 0.0;
    if (tid < E)
      for (int k = 0; k < nw; ++k) { cc += wc[k][tid]; pp += wp[k][tid]; }
    double term = 0.0;
    if (tid < E) {
      a.counts[tid] = (int32_t)cc;
      term = ((double)E / ((double)a.K * a.T)) * (double)cc * (pp / a.T);
    }
    for (int o = 16; o > 0; o >>= 1) term += __shfl_down_sync(0xffffffffu, term, o);
    if (tid == 0) *a.aux_loss = (float)(a.alpha * term);
  }
}

// Count this block as done; true for the block that finishes last (which then
// also resets the counter for the next call).
__device__ bool last_block_done(unsigned int* ctr) {
  __shared__ bool last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int prev = atomicAdd(ctr, 1u);
    last = prev == gridDim.x - 1;
    if (last) *ctr = 0u;
  }
  __syncthreads();
  if (last) __threadfence();
  return last;
}

template <int EMAX>
__global__ void __launch_bounds__(kMmaMaxConsumers * 32, 1)
route_kernel_mma(const __grid_constant__ CUtensorMap tmap_x, RouteArgs a, FinalizeArgs fin) {
  constexpr int NT = EMAX / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const MmaSmem L = mma_layout(a.D, a.E);
  const int NC = L.consumers, hc = L.hc;
  const int E = a.E, D = a.D, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int wg_stride = D * 2 + 16;
  const int nchunks = D / 64;
  const int stage_bytes = kMmaRB * hc * 128;
  uint8_t* wg_s = smem + L.wg;
  uint8_t* xs = smem + L.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.misc);
  int* cnt_s = reinterpret_cast<int*>(full + 2 * kMmaMaxConsumers);
  float* wsum_s = reinterpret_cast<float*>(cnt_s + 32);

  const int nrb = (a.T + kMmaRB - 1) / kMmaRB;
  const int my_rb = (nrb - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  // lane 0 of warp w: half h of this CTA's j-th row block into the warp's stage 2w + h
  auto issue = [&](int j, int h) {
    const int rb = blockIdx.x + j * gridDim.x;
    const int st = 2 * w + h;
    const int z0 = h * hc;
    const int nb = (nchunks - z0) < hc ? (nchunks - z0) : hc;     // blocks inside D
    const uint32_t bar = smem_u32(&full[st]);
    const uint32_t dst = smem_u32(xs + (size_t)st * stage_bytes);
    if (a.tmap3d) {
      // one box of hc blocks; blocks past D come back zero-filled and count as bytes
      mbar_arrive_expect_tx(bar, stage_bytes);
      tma_load_3d(dst, &tmap_x, 0, rb * kMmaRB, z0, bar);
    } else {
      mbar_arrive_expect_tx(bar, (uint32_t)nb * kMmaRB * 128);
      for (int c = 0; c < nb; ++c) tma_load_2d(dst + c * (kMmaRB * 128), &tmap_x, (z0 + c) * 64, rb * kMmaRB, bar);
    }
  };
  if (lane == 0) {
    mbar_init(smem_u32(&full[2 * w]), 1);
    mbar_init(smem_u32(&full[2 * w + 1]), 1);
    fence_barrier_init();
    if (w < my_rb) { issue(w, 0); issue(w, 1); }   // x streams in while the gate weight loads
  }
  if (tid < 32) cnt_s[tid] = 0;
  {  // gate weight (bf16) -> padded rows; rows E..EMAX-1 are zero
    const int vpr = D / 8;
    const uint4* wv = reinterpret_cast<const uint4*>(a.wg);
#pragma unroll 4
    for (int i = tid; i < EMAX * vpr; i += blockDim.x) {
      const int e = i / vpr, v = i % vpr;
      const uint4 val = e < E ? __ldg(wv + (size_t)e * vpr + v) : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(wg_s + (size_t)e * wg_stride + v * 16) = val;
    }
  }
  __syncthreads();

  float psum[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) psum[e] = 0.f;
  bool ok = true;
  float* logit_w = reinterpret_cast<float*>(smem + L.logits) + (size_t)w * kMmaRB * EMAX;
  const uint32_t wg_base = smem_u32(wg_s);
  const int li = lane >> 3, lj = lane & 7;
  for (int j = w, k = 0; j < my_rb; j += NC, ++k) {
    const int rb = blockIdx.x + j * gridDim.x;
    // four independent accumulator chains (one per k16 step of a 64-column block)
    float acc4[4][NT][4];
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc4[g][nt][q] = 0.f;
    for (int h = 0; h < 2; ++h) {
      const int st = 2 * w + h;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), k & 1, nullptr, a.status, 100));
      if (!ok) break;
      const uint32_t buf = smem_u32(xs + (size_t)st * stage_bytes);
      const int z0 = h * hc;
      const int nb = (nchunks - z0) < hc ? (nchunks - z0) : hc;
      for (int cb = 0; cb < nb; ++cb) {
        const int c = z0 + cb;                       // global 64-column block
        const uint32_t box = buf + cb * (kMmaRB * 128);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t b[NT][2];
          const int kc = c * 64 + ks * 16 + (li & 1) * 8;
#pragma unroll
          for (int np = 0; np < NT; np += 2) {
            if (np + 1 < NT) {
              const int n = (np + (li >> 1)) * 8 + lj;
              ldsm_x4(wg_base + n * wg_stride + kc * 2, b[np][0], b[np][1], b[np + 1][0], b[np + 1][1]);
            } else {
              ldsm_x2(wg_base + (np * 8 + lj) * wg_stride + kc * 2, b[np][0], b[np][1]);
            }
          }
          const int row = (li & 1) * 8 + lj;
          const int chunk = ks * 2 + (li >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(box + row * 128 + ((chunk ^ (row & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816(acc4[ks][nt], a0, a1, a2, a3, b[nt][0], b[nt][1]);
        }
      }
      __syncwarp();                                  // every lane is done reading the stage
      if (lane == 0 && j + NC < my_rb) {             // refill it with the next row block's half
        fence_async_shared();
        issue(j + NC, h);
      }
    }
    if (!ok) break;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[nt][q] = (acc4[0][nt][q] + acc4[1][nt][q]) + (acc4[2][nt][q] + acc4[3][nt][q]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = lane >> 2, col = nt * 8 + (lane & 3) * 2;
      logit_w[row * EMAX + col] = acc[nt][0];
      logit_w[row * EMAX + col + 1] = acc[nt][1];
      logit_w[(row + 8) * EMAX + col] = acc[nt][2];
      logit_w[(row + 8) * EMAX + col + 1] = acc[nt][3];
    }
    __syncwarp();
    if (lane < kMmaRB) {
      const int tok = rb * kMmaRB + lane;
      if (tok < a.T) {
        float l[EMAX];
#pragma unroll
        for (int e = 0; e < EMAX; ++e) l[e] = logit_w[lane * EMAX + e];
        token_select<EMAX>(l, tok, a, cnt_s, psum);
      }
    }
    __syncwarp();
  }
  __syncthreads();
  tile_partials<EMAX>(psum, blockIdx.x, a, cnt_s, wsum_s);
  if (!ok) set_status(a.status, DEV_TIMEOUT, 102);
  if (fin.counts != nullptr && last_block_done(fin.ctr)) finalize_counts_loss<EMAX>(fin, xs);
}

// ---------------------------------------------------------------- fp32: FFMA logits
// fp32 inputs keep true fp32 products (a 1e-5 bound rules out tf32 tensor
// cores): one or two tokens per thread, the gate weight as fp32 in shared
// memory read by broadcast.
template <int EMAX>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel_ffma(const __grid_constant__ CUtensorMap tmap_x, RouteArgs a, FinalizeArgs fin) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const RouteSmem L = route_layout(a.D, a.E, a.tile_rows, 0);
  const int E = a.E, D = a.D, tid = threadIdx.x;
  constexpr int CC = 32;     // fp32 columns per 128-byte chunk
  const int nchunks = D / CC;
  float* wg_s = reinterpret_cast<float*>(smem + L.wg);
  uint8_t* xs = smem + L.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.misc);
  int* cnt_s = reinterpret_cast<int*>(full + kRouteStages);
  float* wsum_s = reinterpret_cast<float*>(cnt_s + 32);
  const int stage_bytes = a.tile_rows * 128;
  {
    const float4* wv = reinterpret_cast<const float4*>(a.wg);
#pragma unroll 4
    for (int i = tid; i < E * D / 4; i += kRouteThreads) reinterpret_cast<float4*>(wg_s)[i] = __ldg(wv + i);
  }
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
    const int c = it % nchunks;
    const int tile = blockIdx.x + (it / nchunks) * gridDim.x;
    if (c == 0) {
#pragma unroll
      for (int e = 0; e < EMAX; ++e) { acc0[e] = 0.f; acc1[e] = 0.f; }
      if (tid < 32) cnt_s[tid] = 0;
    }
    const int s = it % kRouteStages;
    const bool ok = mbar_wait(smem_u32(&full[s]), (it / kRouteStages) & 1, nullptr, a.status, 101);
    const uint8_t* st = xs + (size_t)s * stage_bytes;
    for (int j = 0; j < (ok ? 8 : 0); ++j) {
      float f0[4] = {0.f, 0.f, 0.f, 0.f}, f1[4] = {0.f, 0.f, 0.f, 0.f};
      if (has0) {
        const float4 v = *reinterpret_cast<const float4*>(st + r0 * 128 + ((j ^ (r0 & 7)) << 4));
        f0[0] = v.x; f0[1] = v.y; f0[2] = v.z; f0[3] = v.w;
      }
      if (has1) {
        const float4 v = *reinterpret_cast<const float4*>(st + r1 * 128 + ((j ^ (r1 & 7)) << 4));
        f1[0] = v.x; f1[1] = v.y; f1[2] = v.z; f1[3] = v.w;
      }
      const int col = c * CC + j * 4;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          const float4 w4 = *reinterpret_cast<const float4*>(wg_s + (size_t)e * D + col);
          acc0[e] = fmaf(f0[0], w4.x, fmaf(f0[1], w4.y, fmaf(f0[2], w4.z, fmaf(f0[3], w4.w, 0.f)))) + acc0[e];
          acc1[e] = fmaf(f1[0], w4.x, fmaf(f1[1], w4.y, fmaf(f1[2], w4.z, fmaf(f1[3], w4.w, 0.f)))) + acc1[e];
        }
      }
    }
    if (__syncthreads_or(!ok)) { set_status(a.status, DEV_TIMEOUT, 103); break; }
    if (tid == 0 && it + kRouteStages < items) issue(it + kRouteStages);
    if (c == nchunks - 1) {
      float psum[EMAX];
#pragma unroll
      for (int e = 0; e < EMAX; ++e) psum[e] = 0.f;
      const int tok0 = tile * a.tile_rows + r0, tok1 = tile * a.tile_rows + r1;
      if (has0 && tok0 < a.T) token_select<EMAX>(acc0, tok0, a, cnt_s, psum);
      if (has1 && tok1 < a.T) token_select<EMAX>(acc1, tok1, a, cnt_s, psum);
      tile_partials<EMAX>(psum, tile, a, cnt_s, wsum_s);
    }
  }
  if (fin.counts != nullptr && last_block_done(fin.ctr)) finalize_counts_loss<EMAX>(fin, xs);
}

void route_plan(int T, int D, int E, int bf16, int sms, int* tile_rows, int* threads) {
  if (bf16) {
    *tile_rows = kMmaRB;
    *threads = mma_layout(D, E).consumers * 32;
  } else {
    int tile = (T + sms - 1) / sms;
    tile = (tile + 31) / 32 * 32;
    tile = tile < 32 ? 32 : (tile > 256 ? 256 : tile);
    while (tile > 32 && route_smem_bytes(D, E, tile, 0) > 232448) tile -= 32;
    *tile_rows = tile;
    *threads = kRouteThreads;
  }
}

size_t route_smem_total(int D, int E, int tile_rows, int bf16) {
  return bf16 ? mma_layout(D, E).total : route_smem_bytes(D, E, tile_rows, 0);
}

int route_mma_stages(int D, int E) { return mma_layout(D, E).consumers; }

cudaError_t launch_route(const RouteArgs& a, const FinalizeArgs& fin, const CUtensorMap* tm, cudaStream_t s) {
  const size_t smem = route_smem_total(a.D, a.E, a.tile_rows, a.bf16);
  cudaError_t err;
  if (a.bf16) {
#define MOE_ROUTE_MMA(EM)                                                                               \
  if (a.E <= EM) {                                                                                      \
    err = cudaFuncSetAttribute(route_kernel_mma<EM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (err != cudaSuccess) return err;                                                                 \
    route_kernel_mma<EM><<<a.grid, mma_layout(a.D, a.E).consumers * 32, smem, s>>>(*tm, a, fin);          \
    return cudaGetLastError();                                                                          \
  }
    MOE_ROUTE_MMA(8)
    MOE_ROUTE_MMA(16)
    MOE_ROUTE_MMA(32)
#undef MOE_ROUTE_MMA
  } else {
#define MOE_ROUTE_FFMA(EM)                                                                              \
  if (a.E <= EM) {                                                                                      \
    err = cudaFuncSetAttribute(route_kernel_ffma<EM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (err != cudaSuccess) return err;                                                                 \
    route_kernel_ffma<EM><<<a.grid, kRouteThreads, smem, s>>>(*tm, a, fin);                             \
    return cudaGetLastError();                                                                          \
  }
    MOE_ROUTE_FFMA(8)
    MOE_ROUTE_FFMA(16)
    MOE_ROUTE_FFMA(32)
#undef MOE_ROUTE_FFMA
  }
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- finalize (race path)
template <int EMAX>
__global__ void __launch_bounds__(256) route_finalize_kernel(FinalizeArgs a) {
  __shared__ __align__(16) uint8_t scratch[kFinalizeScratch];
  finalize_counts_loss<EMAX>(a, scratch);
}

cudaError_t launch_route_finalize(const FinalizeArgs& a, cudaStream_t s) {
  if (a.E <= 8) route_finalize_kernel<8><<<1, 256, 0, s>>>(a);
  else if (a.E <= 16) route_finalize_kernel<16><<<1, 256, 0, s>>>(a);
  else route_finalize_kernel<32><<<1, 256, 0, s>>>(a);
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
