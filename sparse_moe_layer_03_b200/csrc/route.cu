// Router of the DiT-MoE layer (MoEGate): gate logits x.Wg^T (+ bias), row
// softmax, per-token top-K or the Expert-Race global top-(K*T), per-expert
// counts and the expert-level balance loss.
//
// Sources: "DiT-MoE" hub page, section 1 (MoEGate: weight (E, gating_dim),
// softmax scoring, top_k); "Scaling Diffusion Transformers to 16 Billion
// Parameters", "MOE-DIT" (balance loss eq. L_balance); "Expert Race" abstract
// (tokens and experts compete jointly for the top candidates).
//
// The logits are HBM-bound: x streams through shared memory once, in blocks of
// 16 whole rows brought by TMA (3-D boxes of 64-column blocks, 128-byte swizzle).
// bf16 and fp16 inputs take their E dot products on mma.sync (the FP32 pipe
// alone cannot keep up with HBM at E = 16); fp32 inputs use FFMA.  Per-tile
// partial counts and score sums are reduced in a fixed order, so the loss is
// bit-reproducible.  Also here: the adaLN modulation of the rows in shared
// memory before the logits, the per-image balance loss, and the Expert-Race
// selection (one cooperative kernel after the router).
#include <cuda.h>
#include <type_traits>
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
__host__ __device__ inline RouteSmem route_layout(int D, int E, int tile_rows, int b16) {
  RouteSmem L;
  const int em = route_emax(E);
  L.wg = 0;
  const size_t wg_bytes = b16 ? (size_t)em * (D * 2 + 16) : (size_t)E * D * 4;
  L.x = align1k(wg_bytes);
  // the x stages double as the finalize scratch (2 x 32 x 33 x 8 bytes) at the end
  const size_t xb = (size_t)kRouteStages * tile_rows * 128;
  L.logits = L.x + (xb > 16896 ? xb : 16896);
  L.misc = L.logits + (b16 ? (size_t)tile_rows * em * 4 : 0);
  // barriers (4 x 8 B) + counts (<= 32 x 4 B) + warp sums (8 x 32 x 4 B)
  L.total = 1024 /*alignment slack*/ + L.misc + 2048;
  return L;
}

size_t route_smem_bytes(int D, int E, int tile_rows, int b16) {
  return route_layout(D, E, tile_rows, b16).total;
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
  if (a.P) {      // score row: Expert-Race selects from it; per-image losses read it
    float* prow = a.P + (size_t)tok * E;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) prow[e] = P[e];
    if (a.race) return;
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
    if (!a.race) a.tile_counts[(size_t)tile * a.E + tid] = cnt_s[tid];
  }
  __syncthreads();
}

// ---------------------------------------------------------------- 16-bit: tensor-core logits
// Work unit = a block of 16 consecutive tokens: their full rows (16 x D 16-bit,
// one contiguous stretch of HBM, so DRAM pages are read whole) arrive in P parts,
// each one 3-D TMA box of 64-column blocks x 16 rows (128-byte swizzle) into one
// of the warp's two stages.  Each warp takes every NC-th row block and issues its
// own loads: wait for a part, compute its share of the 16 x E logits with
// mma.sync m16n8k16 (A via ldmatrix from the swizzled stage, B = gate weight in
// shared memory with rows padded by 16 bytes), refill that stage with the part
// after next (the load overlaps the other stage's MMAs and the epilogue), then
// run softmax and selection (one lane per token).  No block-wide barrier inside
// the loop and no warp waits on another warp's progress.
constexpr int kMmaRB = 16;        // tokens per row block
constexpr int kMmaMaxConsumers = 8;

// A row block is loaded in P parts of cpq = ceil(D/64 / P) column blocks (one 3-D TMA box each);
// warp c owns stages 2c and 2c+1, which take the parts of its row blocks in turn (part n of the
// warp's sequence goes to stage n mod 2), issues their loads itself and waits on their phases
// strictly in order.  P is chosen for the most consumer warps (<= 8) that shared memory holds:
// more warps leave fewer row blocks per warp (at XL, 8 warps with P = 3 give each warp at most
// 2 of the 2048 blocks, where 5 warps with halves gave most warps 3).  The adaLN modulation needs
// the whole row in the warp's two stages: P = 2.
struct MmaSmem {
  size_t wg, x, logits, misc, total;
  int consumers, parts, cpq;
};
__host__ __device__ inline MmaSmem mma_layout(int D, int E, bool modulate) {
  MmaSmem best{};
  const int em = route_emax(E);
  const int nchunks = D / 64;
  for (int parts = 2; parts <= (modulate ? 2 : 4); ++parts) {
    if (parts > 2 && parts > nchunks) break;
    MmaSmem L;
    L.parts = parts;
    L.cpq = (nchunks + parts - 1) / parts;
    if (parts > 2 && (parts - 1) * L.cpq >= nchunks) continue;   // no part without columns
    L.wg = 0;
    L.x = align1k((size_t)em * (D * 2 + 16));
    const size_t stage = (size_t)kMmaRB * L.cpq * 128;
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
    if (parts == 2 || L.consumers > best.consumers) best = L;
  }
  return best;
}

// adaLN modulation of one row block held in a warp's two stages, in place:
// m = gamma_b * (x - mean) / sqrt(var + eps) + beta_b for token t of image
// b = t / img_len ("Diffusion Transformer (DiT) 技术全景解析" 2.2.3, AdaLN: a
// plain layer_norm over the features, then the per-sample scale and shift).
// Lane l takes row l % 16 of half l / 16 (two lanes per row).  The statistics
// take one pass over shared memory: sums of x - x0 and its square, shifted by
// the row's first value x0 (so the variance does not cancel when the mean is
// large).  The rewrite applies m = x * a_c + (beta_c - a_c * mean) with
// a_c = gamma_c * rstd, reading each chunk's logical columns through the
// 128-byte swizzle.  Lane (r, p) starts at 16-byte chunk r + 4p of its row, so
// the 32 lanes spread over the 8 chunk positions (4 wavefronts per access).
template <bool F16>
__device__ __forceinline__ void route_modulate(const RouteArgs& a, uint8_t* xs, int stage_bytes, int w, int hc,
                                               int nchunks, int rb, int lane) {   // hc: blocks per half (P = 2)
  using S = typename std::conditional<F16, StoreF16, StoreBF16>::type;
  const int r = lane & 15, p = lane >> 4;
  const int z0 = p * hc;
  const int nb = (nchunks - z0) < hc ? (nchunks - z0) : hc;
  const uint32_t base = smem_u32(xs + (size_t)(2 * w + p) * stage_bytes) + r * 128;
  const int rot = (r + 4 * p) & 7;
  const int D = a.D;
  // the row's first value (logical column 0 lives in half 0, block 0, physical chunk r % 8)
  float x0;
  {
    uint32_t v0;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v0)
                 : "r"(smem_u32(xs + (size_t)(2 * w) * stage_bytes) + r * 128 + ((0 ^ (r & 7)) << 4)));
    const uint4 q = make_uint4(v0, 0u, 0u, 0u);
    float f[8];
    S::x8_to_f32(q, f);
    x0 = f[0];
  }
  float s1 = 0.f, s2 = 0.f;
  for (int cb = 0; cb < nb; ++cb) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int pj = (q + rot) & 7;
      uint4 v;
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(base + cb * (kMmaRB * 128) + pj * 16));
      float f[8];
      S::x8_to_f32(v, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = f[e] - x0;
        s1 += d;
        s2 = fmaf(d, d, s2);
      }
    }
  }
  s1 += __shfl_xor_sync(0xffffffffu, s1, 16);
  s2 += __shfl_xor_sync(0xffffffffu, s2, 16);
  const float inv_d = 1.0f / (float)D;
  const float dm = s1 * inv_d;                                   // mean - x0
  const float var = fmaxf(s2 * inv_d - dm * dm, 0.f);
  const float mu = x0 + dm;
  const float rstd = rsqrtf(var + a.eps);
  const int tok = rb * kMmaRB + r;
  if (tok >= a.T) return;                           // rows past T stay zero (the store clips them)
  const int img = tok / a.img_len;
  const uint4* gp = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.gamma) + (size_t)img * D);
  const uint4* bp = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.beta) + (size_t)img * D);
  for (int cb = 0; cb < nb; ++cb) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int pj = (q + rot) & 7;
      const uint32_t addr = base + cb * (kMmaRB * 128) + pj * 16;
      const int c8 = (z0 + cb) * 8 + (pj ^ (r & 7));   // logical 8-column chunk of this row
      uint4 v;
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(addr));
      float f[8], g[8], b[8];
      S::x8_to_f32(v, f);
      S::x8_to_f32(__ldg(gp + c8), g);
      S::x8_to_f32(__ldg(bp + c8), b);
      float m[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float ac = g[e] * rstd;
        m[e] = fmaf(f[e], ac, fmaf(-ac, mu, b[e]));
      }
      uint4 o;
      o.x = S::pack2(m[0], m[1]);
      o.y = S::pack2(m[2], m[3]);
      o.z = S::pack2(m[4], m[5]);
      o.w = S::pack2(m[6], m[7]);
      asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w)
                   : "memory");
    }
  }
}

// The last block to finish turns the per-block partials into counts and the loss
// (and, where asked, leaves the per-expert score sums for cross-call statistics).
// Thread (chunk, expert) of the first nch * E sums tiles chunk, chunk + nch, ... of
// its expert (all of its loads independent, so the block's loads are in flight
// together: one round trip instead of one per expert); then thread e adds the
// chunks' sums in chunk order, and a fixed tree over the experts gives the loss.
// Bit-reproducible.  scratch: 16 bytes per (chunk, expert), at most blockDim of them.
constexpr int kFinalizeScratch = 2 * 32 * 32 * 8;
template <int EMAX>
__device__ void finalize_counts_loss(const FinalizeArgs& a, uint8_t* scratch) {
  const int tid = threadIdx.x;
  const int E = a.E;
  const int nch = (int)blockDim.x / E;               // E <= 32 <= blockDim
  long long* cc = reinterpret_cast<long long*>(scratch);
  double* pp = reinterpret_cast<double*>(scratch + (size_t)nch * E * sizeof(long long));
  if (tid < nch * E) {
    const int e = tid % E, ch = tid / E;
    const int nt = a.ntiles_counts > a.ntiles_psum ? a.ntiles_counts : a.ntiles_psum;
    long long c = 0;
    double p = 0.0;
#pragma unroll 8
    for (int t = ch; t < nt; t += nch) {
      if (t < a.ntiles_counts) c += __ldcg(a.tile_counts + (size_t)t * E + e);
      if (t < a.ntiles_psum) p += (double)__ldcg(a.tile_psum + (size_t)t * E + e);
    }
    cc[ch * E + e] = c;
    pp[ch * E + e] = p;
  }
  __syncthreads();
  if (tid < 32) {
    double term = 0.0;
    if (tid < E) {
      long long c = 0;
      double p = 0.0;
      for (int ch = 0; ch < nch; ++ch) {
        c += cc[ch * E + tid];
        p += pp[ch * E + tid];
      }
      a.counts[tid] = (int32_t)c;
      if (a.score_sum) a.score_sum[tid] = p;
      term = ((double)E / ((double)a.K * a.T)) * (double)c * (p / a.T);
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

template <int EMAX, bool F16>
__global__ void __launch_bounds__(kMmaMaxConsumers * 32, 1)
route_kernel_mma(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_m, RouteArgs a,
                 FinalizeArgs fin) {
  constexpr int NT = EMAX / 8;
  launch_dependents();                              // the dispatch count kernel may get resident
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const bool modulate = a.gamma != nullptr;
  const MmaSmem L = mma_layout(a.D, a.E, modulate);
  const int NC = L.consumers, P = L.parts, hc = L.cpq;
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
  const uint64_t pol_x = policy_evict_last();
  // lane 0 of warp w: part h of this CTA's j-th row block into stage st (2w or 2w + 1)
  auto issue = [&](int j, int h, int st) {
    const int rb = blockIdx.x + j * gridDim.x;
    const int z0 = h * hc;
    const int nb = (nchunks - z0) < hc ? (nchunks - z0) : hc;     // blocks inside D
    const uint32_t bar = smem_u32(&full[st]);
    const uint32_t dst = smem_u32(xs + (size_t)st * stage_bytes);
    if (a.tmap3d) {
      // one box of hc blocks; blocks past D come back zero-filled and count as bytes
      mbar_arrive_expect_tx(bar, stage_bytes);
      // x stays in L2 for the dispatch gather, which reads it again right after (75 MB at XL)
      tma_load_3d_hint(dst, &tmap_x, 0, rb * kMmaRB, z0, bar, pol_x);
    } else {
      mbar_arrive_expect_tx(bar, (uint32_t)nb * kMmaRB * 128);
      for (int c = 0; c < nb; ++c) tma_load_2d(dst + c * (kMmaRB * 128), &tmap_x, (z0 + c) * 64, rb * kMmaRB, bar);
    }
  };
  // The gate weight's rows come in by bulk copies issued before any x load, so that they are not
  // queued behind every CTA's x stream (loaded by the threads after the x loads were issued,
  // setup took about 8 us at XL, measured with a timer probe); the x loads follow at once.
  uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + L.misc + 1536);
  if (tid == 0) {
    mbar_init(smem_u32(wbar), 1);
    for (int i = 0; i < 2 * NC; ++i) mbar_init(smem_u32(&full[i]), 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(smem_u32(wbar), (uint32_t)(E * D * 2));
    for (int e = 0; e < E; ++e)
      bulk_load(smem_u32(wg_s + (size_t)e * wg_stride), reinterpret_cast<const uint8_t*>(a.wg) + (size_t)e * D * 2,
                (uint32_t)(D * 2), smem_u32(wbar));
  }
  __syncthreads();
  if (lane == 0 && w < my_rb) { issue(w, 0, 2 * w); issue(w, 1, 2 * w + 1); }
  if (tid < 32) cnt_s[tid] = 0;
  if (blockIdx.x == 0 && a.zero)
    for (int i = tid; i < a.nzero; i += blockDim.x) a.zero[i] = 0u;
  {  // rows E..EMAX-1 of the padded gate weight are zero
    const int vpr = D / 8;
    for (int i = E * vpr + tid; i < EMAX * vpr; i += blockDim.x)
      *reinterpret_cast<uint4*>(wg_s + (size_t)(i / vpr) * wg_stride + (i % vpr) * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  if (!mbar_wait(smem_u32(wbar), 0, nullptr, a.status, 104)) set_status(a.status, DEV_TIMEOUT, 104);

  float psum[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) psum[e] = 0.f;
  bool ok = true;
  float* logit_w = reinterpret_cast<float*>(smem + L.logits) + (size_t)w * kMmaRB * EMAX;
  const uint32_t wg_base = smem_u32(wg_s);
  const int li = lane >> 3, lj = lane & 7;
  int n = 0;                                        // this warp's part count: part n uses stage 2w + n % 2
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
    if (modulate) {
      // both halves of the row block, then m in place; m goes out to x_mod while the MMAs read it
      for (int h = 0; h < 2 && ok; ++h)
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[2 * w + h]), k & 1, nullptr, a.status, 103));
      if (!ok) break;
      route_modulate<F16>(a, xs, stage_bytes, w, hc, nchunks, rb, lane);
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        for (int h = 0; h < 2; ++h) {
          const uint32_t src = smem_u32(xs + (size_t)(2 * w + h) * stage_bytes);
          if (a.tmap3d) {
            tma_store_3d(&tmap_m, src, 0, rb * kMmaRB, h * hc);
          } else {
            const int nbh = (nchunks - h * hc) < hc ? (nchunks - h * hc) : hc;
            for (int c = 0; c < nbh; ++c) tma_store_2d(&tmap_m, src + c * (kMmaRB * 128), (h * hc + c) * 64, rb * kMmaRB);
          }
        }
        bulk_commit();
      }
    }
    for (int h = 0; h < P; ++h, ++n) {
      const int st = 2 * w + (n & 1);
      if (!modulate) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), (n >> 1) & 1, nullptr, a.status, 100));
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
          for (int nt = 0; nt < NT; ++nt) mma_16816<F16>(acc4[ks][nt], a0, a1, a2, a3, b[nt][0], b[nt][1]);
        }
      }
      __syncwarp();                                  // every lane is done reading the stage
      const int n2 = n + 2, j2 = w + (n2 / P) * NC;  // the stage's next part: this warp's part n + 2
      if (lane == 0 && j2 < my_rb) {
        if (modulate) bulk_wait_read_all();          // the x_mod store has read the stage
        fence_async_shared();
        issue(j2, n2 % P, st);
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
  if (modulate && lane == 0) bulk_wait_all();       // x_mod stores complete before the stages are reused
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
  if (blockIdx.x == 0 && a.zero)
    for (int i = tid; i < a.nzero; i += blockDim.x) a.zero[i] = 0u;
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

void route_plan(int T, int D, int E, int b16, int modulate, int sms, int* tile_rows, int* threads) {
  if (b16) {
    *tile_rows = kMmaRB;
    *threads = mma_layout(D, E, modulate != 0).consumers * 32;
  } else {
    int tile = (T + sms - 1) / sms;
    tile = (tile + 31) / 32 * 32;
    tile = tile < 32 ? 32 : (tile > 256 ? 256 : tile);
    while (tile > 32 && route_smem_bytes(D, E, tile, 0) > 232448) tile -= 32;
    *tile_rows = tile;
    *threads = kRouteThreads;
  }
}

size_t route_smem_total(int D, int E, int tile_rows, int b16, int modulate) {
  return b16 ? mma_layout(D, E, modulate != 0).total : route_smem_bytes(D, E, tile_rows, 0);
}

int route_mma_stages(int D, int E, int modulate) { return mma_layout(D, E, modulate != 0).consumers; }

int route_box_blocks(int D, int E, int modulate) { return mma_layout(D, E, modulate != 0).cpq; }

cudaError_t launch_route(const RouteArgs& a, const FinalizeArgs& fin, const CUtensorMap* tm, const CUtensorMap* tmm,
                         cudaStream_t s) {
  const bool modulate = a.gamma != nullptr;
  const size_t smem = route_smem_total(a.D, a.E, a.tile_rows, a.b16, modulate);
  cudaError_t err;
  if (a.b16) {
#define MOE_ROUTE_MMA(EM, F)                                                                            \
  if (a.E <= EM && (a.f16 != 0) == F) {                                                                 \
    err = cudaFuncSetAttribute(route_kernel_mma<EM, F>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (err != cudaSuccess) return err;                                                                 \
    route_kernel_mma<EM, F><<<a.grid, mma_layout(a.D, a.E, modulate).consumers * 32, smem, s>>>(*tm, *tmm, a, fin); \
    return cudaGetLastError();                                                                          \
  }
    MOE_ROUTE_MMA(8, false)
    MOE_ROUTE_MMA(16, false)
    MOE_ROUTE_MMA(32, false)
    MOE_ROUTE_MMA(8, true)
    MOE_ROUTE_MMA(16, true)
    MOE_ROUTE_MMA(32, true)
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

// ---------------------------------------------------------------- per-image balance loss
// Block b takes image b's tokens [b*L, (b+1)*L): the counts of their selected
// experts and their score sums per expert (fp64, fixed reduction order), then
// the image's L_balance with T = L.  The last block averages the images'
// losses, in a fixed order.
constexpr int kSeqThreads = 256;

template <int EMAX>
__global__ void __launch_bounds__(kSeqThreads) seq_loss_kernel(SeqLossArgs a) {
  __shared__ double wp[kSeqThreads / 32][EMAX];
  __shared__ int cnt_s[EMAX];
  __shared__ bool last;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, E = a.E, L = a.L;
  const int b = blockIdx.x;
  if (tid < EMAX) cnt_s[tid] = 0;
  __syncthreads();
  double p[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) p[e] = 0.0;
  for (int t = b * L + tid; t < (b + 1) * L; t += kSeqThreads) {
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) p[e] += (double)__ldcg(a.P + (size_t)t * E + e);
    const int ns = a.n_sel ? a.n_sel[t] : a.K;
    for (int k = 0; k < a.Kmax && k < ns; ++k) {
      const int e = a.topk_idx[(size_t)t * a.Kmax + k];
      if (e >= 0 && e < E) atomicAdd(&cnt_s[e], 1);
    }
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
      double v = p[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) wp[w][e] = v;
    }
  }
  __syncthreads();
  if (tid < 32) {
    double term = 0.0;
    if (tid < E) {
      double ps = 0.0;
      for (int k = 0; k < kSeqThreads / 32; ++k) ps += wp[k][tid];
      term = ((double)E / ((double)a.K * L)) * (double)cnt_s[tid] * (ps / L);
    }
    for (int o = 16; o > 0; o >>= 1) term += __shfl_down_sync(0xffffffffu, term, o);
    if (tid == 0) a.seq_loss[b] = a.alpha * term;
  }
  // the last block: mean over images
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(a.ctr, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const int nseq = gridDim.x;
  double s = 0.0;
  for (int i = tid; i < nseq; i += kSeqThreads) s += __ldcg(a.seq_loss + i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) wp[w][0] = s;
  __syncthreads();
  if (tid == 0) {
    double tot = 0.0;
    for (int k = 0; k < kSeqThreads / 32; ++k) tot += wp[k][0];
    *a.aux_loss = (float)(tot / nseq);
    *a.ctr = 0u;
  }
}

cudaError_t launch_seq_loss(const SeqLossArgs& a, cudaStream_t s) {
  const int nseq = a.T / a.L;
  if (a.E <= 8) seq_loss_kernel<8><<<nseq, kSeqThreads, 0, s>>>(a);
  else if (a.E <= 16) seq_loss_kernel<16><<<nseq, kSeqThreads, 0, s>>>(a);
  else seq_loss_kernel<32><<<nseq, kSeqThreads, 0, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- Expert-Race
// Exact radix select of the S-th largest score of the T x E matrix on the fp32
// bit patterns (scores are >= 0, so the unsigned order of the bits is the
// numeric order), digits of 12, 12 and 8 bits, followed by the selection, all in
// one cooperative launch with one CTA per SM.  CTA r owns a contiguous range of
// tokens, hence of flat indices t*E+i.  Per digit: a shared-memory histogram of
// the CTA's range, added into a global one; a grid barrier; then every CTA
// finds the bin that holds the needed rank on its own (the same integers
// everywhere give the same answer), so one barrier per digit suffices.  The
// last digit's histogram of CTA r is also stored: its threshold bin counts the
// CTA's entries equal to the threshold, which gives every CTA the number of
// equal entries before its range (ties go to the lower flat index) without a
// fourth barrier.  Each token's score row for the selection is loaded before
// the last barrier.
constexpr int kRaceThreads = 512;

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier over all CTAs of a cooperative launch: arrive on a counter that only
// grows during the launch, then wait until it reaches `target`.  The wait is
// bounded (`limit_ns`): on expiry the status word records `where` and the CTA
// goes on (its outputs are then invalid, which the status reports).
__device__ void grid_barrier(uint32_t* ctr, uint32_t target, int* status, int where, uint64_t limit_ns) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    const uint64_t t0 = global_ns();
    while (ld_acquire_gpu(ctr) < target) {
      if (global_ns() - t0 > limit_ns) {
        set_status(status, DEV_TIMEOUT, where);
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
  }
  __syncthreads();
}

// Exclusive prefix sum of v over the block (kRaceThreads threads); *total gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  constexpr int NW = kRaceThreads / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    uint32_t y = lane < NW ? wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    if (lane < NW) wsum[lane] = y;
  }
  __syncthreads();
  const uint32_t before = (w ? wsum[w - 1] : 0u) + x - v;
  *total = wsum[NW - 1];
  __syncthreads();
  return before;
}

// The bin of the merged histogram h[nb] (global, counted from the top) that
// holds rank `need`, and the rank inside it: out[0], out[1] for every thread.
__device__ void race_find_bin(const uint32_t* h, int nb, uint32_t need, uint32_t* wsum, uint32_t* out) {
  const int per = nb / kRaceThreads > 0 ? nb / kRaceThreads : 1;    // 8 (4096 bins) or 1 (256)
  const int tid = threadIdx.x;
  if (tid == 0) { out[0] = 0u; out[1] = need; }
  uint32_t c[8];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = tid * per + j;
    c[j] = (j < per && i < nb) ? __ldcg(h + nb - 1 - i) : 0u;
    local += c[j];
  }
  uint32_t total;
  uint32_t above = block_excl_scan(local, wsum, &total);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < per) {
      if (above < need && above + c[j] >= need) { out[0] = (uint32_t)(nb - 1 - (tid * per + j)); out[1] = need - above; }
      above += c[j];
    }
  }
  __syncthreads();
}

template <int DIGIT>
__device__ __forceinline__ void race_count(uint32_t* h, uint32_t b, uint32_t prefix) {
  if (DIGIT == 0) atomicAdd(&h[b >> 20], 1u);
  else if (DIGIT == 1) { if ((b >> 20) == prefix) atomicAdd(&h[(b >> 8) & 0xFFFu], 1u); }
  else { if ((b >> 8) == prefix) atomicAdd(&h[b & 0xFFu], 1u); }
}

// shared-memory histogram of digit DIGIT over bits[e0, e1) (e0 a multiple of 4)
template <int DIGIT>
__device__ void race_local_hist(const uint32_t* bits, long long e0, long long e1, uint32_t prefix, uint32_t* h) {
  const long long n4 = (e1 - e0) >> 2;
  const uint4* v4 = reinterpret_cast<const uint4*>(bits + e0);
  for (long long i = threadIdx.x; i < n4; i += kRaceThreads) {
    const uint4 q = __ldcg(v4 + i);
    race_count<DIGIT>(h, q.x, prefix);
    race_count<DIGIT>(h, q.y, prefix);
    race_count<DIGIT>(h, q.z, prefix);
    race_count<DIGIT>(h, q.w, prefix);
  }
  for (long long i = e0 + n4 * 4 + threadIdx.x; i < e1; i += kRaceThreads) race_count<DIGIT>(h, __ldcg(bits + i), prefix);
}

// Winners of token t among its scores v[] against the threshold (`valid` false:
// no token, but the lane still takes part in the warp's ballots); `rank` counts
// the entries equal to the threshold before them in flat order.  The token's
// row (winners in descending score, ties to the lower expert id, then -1 / 0
// padding) is built in registers and written with 16-byte stores when E is a
// multiple of 4 and at most 16.
template <int EMAX>
__device__ __forceinline__ void race_emit(const RaceArgs& a, int t, bool valid, const uint32_t* v, uint32_t thr,
                                          uint32_t need_eq, uint32_t rank, int* cnt_s) {
  const int E = a.E;
  uint32_t win = 0;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (valid && e < E) {
      bool sel = v[e] > thr;
      if (v[e] == thr) { sel = rank < need_eq; ++rank; }
      if (sel) win |= 1u << e;
    }
  }
  // per-expert counts: one shared atomic per warp and expert
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
      const int c = __popc(__ballot_sync(0xffffffffu, (win >> e) & 1u));
      if (lane == 0 && c) atomicAdd(&cnt_s[e], c);
    }
  }
  if (!valid) return;
  const int n = __popc(win);
  int32_t* ri = a.topk_idx + (size_t)t * E;
  float* rw = a.topk_w + (size_t)t * E;
  if (EMAX <= 16 && (E & 3) == 0) {
    // the row in registers (constant indices only), then 16-byte stores
    int oi[EMAX];
    uint32_t ow[EMAX];
#pragma unroll
    for (int k = 0; k < EMAX; ++k) { oi[k] = -1; ow[k] = 0u; }
    uint32_t left = win;
    for (int m = 0; left; ++m) {
      uint32_t bv = 0;
      int bi = -1;
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (((left >> e) & 1u) && (bi < 0 || v[e] > bv)) { bv = v[e]; bi = e; }
      left &= ~(1u << bi);
#pragma unroll
      for (int k = 0; k < EMAX; ++k)
        if (k == m) { oi[k] = bi; ow[k] = bv; }
    }
#pragma unroll
    for (int k = 0; k < EMAX; k += 4) {
      if (k < E) {
        *reinterpret_cast<int4*>(ri + k) = make_int4(oi[k], oi[k + 1], oi[k + 2], oi[k + 3]);
        *reinterpret_cast<uint4*>(rw + k) = make_uint4(ow[k], ow[k + 1], ow[k + 2], ow[k + 3]);
      }
    }
  } else {
    int m = 0;
    uint32_t left = win;
    while (left) {
      uint32_t bv = 0;
      int bi = -1;
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (((left >> e) & 1u) && (bi < 0 || v[e] > bv)) { bv = v[e]; bi = e; }
      left &= ~(1u << bi);
      ri[m] = bi;
      rw[m] = __uint_as_float(bv);
      ++m;
    }
    for (int k = m; k < E; ++k) {
      ri[k] = -1;
      rw[k] = 0.f;
    }
  }
  a.n_sel[t] = n;
}

template <int EMAX>
__global__ void __launch_bounds__(kRaceThreads, 1) race_select_kernel(RaceArgs a, FinalizeArgs fin) {
  __shared__ __align__(16) uint32_t h[4096];     // also the finalize scratch (16 KB) at the end
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t found[2];
  __shared__ int cnt_s[EMAX];
  const int tid = threadIdx.x, r = blockIdx.x, E = a.E;
  const uint32_t G = gridDim.x;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(a.P);
  uint32_t* g0 = a.sync;
  uint32_t* g1 = a.sync + 4096;
  uint32_t* g2 = a.sync + 8192;
  uint32_t* bar = a.sync + 8448;
  const int t0 = min(a.T, r * a.tpc), t1 = min(a.T, t0 + a.tpc);
  const long long e0 = (long long)t0 * E, e1 = (long long)t1 * E;
  const uint32_t S = (uint32_t)a.K * (uint32_t)a.T;
  // test words (host-written, zero in normal use): bit 1 of word 0 makes every barrier wait for
  // one arrival more than the launch makes; word 1 shortens the barrier waits to microseconds
  const uint32_t tflags = a.test ? __ldcg(a.test) : 0u;
  const uint32_t tlimit_us = a.test ? __ldcg(a.test + 1) : 0u;
  const uint32_t extra = (tflags >> 1) & 1u;
  const uint64_t limit = tlimit_us ? (uint64_t)tlimit_us * 1000ull : kWaitLimitNs;

  // digit 1: bits 31..20
  for (int i = tid; i < 4096; i += kRaceThreads) h[i] = 0u;
  if (tid < EMAX) cnt_s[tid] = 0;
  __syncthreads();
  race_local_hist<0>(bits, e0, e1, 0u, h);
  __syncthreads();
  for (int i = tid; i < 4096; i += kRaceThreads)
    if (h[i]) atomicAdd(&g0[i], h[i]);
  grid_barrier(bar, G + extra, a.status, 300, limit);
  race_find_bin(g0, 4096, S, wsum, found);
  uint32_t prefix = found[0], need = found[1];

  // digit 2: bits 19..8 among the entries whose top 12 bits equal the prefix
  for (int i = tid; i < 4096; i += kRaceThreads) h[i] = 0u;
  __syncthreads();
  race_local_hist<1>(bits, e0, e1, prefix, h);
  __syncthreads();
  for (int i = tid; i < 4096; i += kRaceThreads)
    if (h[i]) atomicAdd(&g1[i], h[i]);
  grid_barrier(bar, 2 * G + extra, a.status, 301, limit);
  race_find_bin(g1, 4096, need, wsum, found);
  prefix = (prefix << 12) | found[0];
  need = found[1];

  // digit 3: bits 7..0; this CTA's histogram is also kept for the tie ranks
  for (int i = tid; i < 256; i += kRaceThreads) h[i] = 0u;
  __syncthreads();
  race_local_hist<2>(bits, e0, e1, prefix, h);
  __syncthreads();
  for (int i = tid; i < 256; i += kRaceThreads) {
    a.loc[(size_t)r * 256 + i] = h[i];
    if (h[i]) atomicAdd(&g2[i], h[i]);
  }
  // the score rows of this CTA's first round of tokens load across the barrier
  uint32_t v[EMAX];
  {
    const int t = t0 + tid;
#pragma unroll
    for (int e = 0; e < EMAX; ++e) v[e] = (t < t1 && e < E) ? __ldcg(bits + (size_t)t * E + e) : 0u;
  }
  grid_barrier(bar, 3 * G + extra, a.status, 302, limit);
  race_find_bin(g2, 256, need, wsum, found);
  const uint32_t thr = (prefix << 8) | found[0];   // the S-th largest score's bits
  const uint32_t need_eq = found[1];                // entries equal to it that are selected

  // entries equal to the threshold in the ranges of CTAs 0..r-1
  uint32_t carry;
  {
    uint32_t c = 0;
    for (int q = tid; q < r; q += kRaceThreads) c += __ldcg(a.loc + (size_t)q * 256 + (thr & 0xFFu));
    block_excl_scan(c, wsum, &carry);
  }

  // selection, kRaceThreads tokens at a time (one per thread), in token order
  for (int tb = t0; tb < t1; tb += kRaceThreads) {
    const int t = tb + tid;
    const bool valid = t < t1;
    if (tb != t0) {
#pragma unroll
      for (int e = 0; e < EMAX; ++e) v[e] = (valid && e < E) ? __ldcg(bits + (size_t)t * E + e) : 0u;
    }
    uint32_t my_eq = 0;
#pragma unroll
    for (int e = 0; e < EMAX; ++e) my_eq += (valid && e < E && v[e] == thr) ? 1u : 0u;
    uint32_t round_eq;
    const uint32_t rank = carry + block_excl_scan(my_eq, wsum, &round_eq);
    carry += round_eq;
    race_emit<EMAX>(a, t, valid, v, thr, need_eq, rank, cnt_s);
  }
  __syncthreads();
  if (tid < E) a.tile_counts[(size_t)r * E + tid] = cnt_s[tid];
  if (last_block_done(fin.ctr)) finalize_counts_loss<EMAX>(fin, reinterpret_cast<uint8_t*>(h));
}

int race_plan(int T, int sms, int* tpc) {
  int g = sms < kRaceMaxCtas ? sms : kRaceMaxCtas;
  const int by4 = (T + 3) / 4;
  if (g > by4) g = by4;
  if (g < 1) g = 1;
  int per = (T + g - 1) / g;
  per = (per + 3) / 4 * 4;         // a multiple of 4 tokens keeps every range's start 16-byte aligned
  *tpc = per;
  return (T + per - 1) / per;
}

cudaError_t launch_race_select(const RaceArgs& a, const FinalizeArgs& fin, cudaStream_t s) {
  RaceArgs ra = a;
  FinalizeArgs fa = fin;
  void* args[] = {(void*)&ra, (void*)&fa};
  const dim3 grid((unsigned)a.grid), block(kRaceThreads);
  if (a.E <= 8) return cudaLaunchCooperativeKernel((const void*)race_select_kernel<8>, grid, block, args, 0, s);
  if (a.E <= 16) return cudaLaunchCooperativeKernel((const void*)race_select_kernel<16>, grid, block, args, 0, s);
  return cudaLaunchCooperativeKernel((const void*)race_select_kernel<32>, grid, block, args, 0, s);
}

}  // namespace moe
