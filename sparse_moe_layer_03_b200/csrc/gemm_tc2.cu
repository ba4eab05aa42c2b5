// Grouped expert GEMM on CTA pairs: tcgen05.mma.cta_group::2 (sm_100a).
//
// The same problems and epilogues as the single-CTA kernel (expert MLP =
// W2 gelu(W1 x), "Scaling Diffusion Transformers to 16 Billion Parameters",
// "MOE-DIT" eq. MLP), but every output tile is 256 x BN (BN = 256, and one
// narrower tile per row block when BN does not divide N) and belongs to a pair
// of CTAs on the two SMs of a TPC (a cluster of 2).  Each CTA loads its own
// 128 rows of A and its own half of the tile's B rows, so per FLOP each SM
// pulls 2/3 of the operand bytes of a 128 x 256 single-CTA tile; the pair's
// tensor cores read the peer's half through the CTA pair, and each CTA's TMEM
// receives its 128 rows of the accumulator.  Every TMA load fills one CTA's own
// shared memory (nothing is broadcast to several CTAs).
//
// Roles per CTA (6 warps): warp 0 = TMA producer (both CTAs; loads complete on
// the leader's barrier); warp 1 = TMEM allocation (both) and the MMA issuer
// (leader only); warps 2-5 = epilogue (both CTAs, one per TMEM lane quadrant),
// storing through TMA.  The gathering instantiation adds warps 6-7: the row
// gather of a routed problem whose A rows are rows of x picked by row_token
// (16-byte cp.async into the swizzled stage, reported on the leader's stage
// barrier two stages later, after a proxy fence).
// Synchronisation: the leader's MMA thread commits MMA completion to the
// "stage empty" and "accumulator full" barriers of both CTAs (one commit per
// CTA, by shared::cluster address); every epilogue warp of both CTAs arrives
// on the leader's "accumulator empty" barrier; both CTAs' TMA loads complete
// on the leader's "stage full" barrier.  All waits are bounded.
// Pipeline: a stage holds two 64-wide k-blocks (per k-block an A box and a B box, 64 KB per CTA,
// 3 stages), one in the row-gathering instantiation (32 KB, 5 stages).  The launches' time went
// with the number of stages they turned over rather than with their bytes: two k-blocks per
// stage made GEMM1 8% and the layer backward 5% faster than one, three were slower than two.
//
// Scheduling: persistent pairs.  Without the folded combine, pair c runs tiles
// c, c + pairs, c + 2 pairs, ... (consecutive tiles share their A row block and
// run side by side).  With it, pairs claim tiles in increasing order from a
// counter in global memory (the leader's producer claims one tile ahead and
// hands each id to the other roles of both CTAs through a small ring in shared
// memory).  Routed tiles are numbered before shared ones, so a shared tile can
// only wait for routed tiles that resident pairs have already claimed: no wait
// depends on a pair that is not running, however many pairs the device holds
// at once.  (Bringing the operand boxes of later stages into L2 with TMA
// prefetches made both GEMMs 1.5x slower: the TMA unit's throughput, not the
// latency of L2, bounds the loads.)
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kPairBM = 256;            // rows of a pair tile (128 per CTA)
constexpr int kPairBK = 64;             // 16-bit elements per 128-byte swizzle row
constexpr int kPairEpiWarps = 4 * kPairEpiSplit;   // kPairEpiSplit per TMEM lane quadrant, each on its own column boxes
constexpr int kPairGatherWarps = 2;
// What one instantiation can do, fixed at compile time so that a launch carries only the code
// its problems use (the forward GEMMs measured 4-10% slower when compiled together with the
// backward's and the gather's paths):
constexpr int kFeatClaim = 1;             // tiles claimed in order (the folded combine)
constexpr int kFeatGather = 2;            // routed A rows copied from x by the gather warps
constexpr int kFeatBwd = 4;               // MN-major operands, weight-gradient problems, fp32 output, GELU backward
template <int F>
constexpr int pair_threads() { return 64 + 32 * kPairEpiWarps + ((F & kFeatGather) ? 32 * kPairGatherWarps : 0); }
// 64-wide k-blocks per pipeline stage: two, or one where the gather warps fill the stages' A rows
template <int F>
constexpr int pair_kps() { return (F & kFeatGather) ? 1 : 2; }
constexpr int kPairSmemLimit = 232448;
constexpr int kSchedSlots = 4;                                  // tile ids handed out ahead
constexpr int kSchedConsumers = 2 + 2 * kPairEpiWarps;          // peer producer, MMA issuer, epilogue warps

template <int BN, int KPS = 1>
struct PairCfg {
  static constexpr int A_BYTES = 128 * kPairBK * 2;     // one k-block of this CTA's A rows
  static constexpr int B_BYTES = (BN / 2) * kPairBK * 2;
  static constexpr int KB_BYTES = A_BYTES + B_BYTES;    // one k-block: its A box, then its B box
  static constexpr int STAGE = KPS * KB_BYTES;
  // epilogue staging: two 32 rows x 128 bytes buffers per epilogue warp for TMA stores
  // (a single buffer, trading 16 KB for one more operand stage, measured 1.8x slower on GEMM1)
  static constexpr int EPI_BYTES = kPairEpiWarps * 2 * 4096;
  // keep 4 KB of the 227 KB for barriers, the 1 KB alignment slack and static shared memory
  // (with 4 epilogue warps and one k-block per stage this gives 5 stages; a 6th, which fits in 3 KB,
  // measured 3% slower on GEMM2 + combine at XL); with two k-blocks per stage, 3 stages fit in 3 KB
  static constexpr int FIT = (kPairSmemLimit - (KPS > 1 ? 3072 : 4096) - EPI_BYTES) / STAGE;
  static constexpr int STAGES = FIT > 8 ? 8 : FIT;
  static constexpr int SMEM = STAGES * STAGE + EPI_BYTES + 2048;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static_assert(STAGES >= 2, "the operand ring needs two stages at least");
  static_assert(SMEM <= kPairSmemLimit, "shared memory above the per-block limit");
  static_assert(STAGE % 1024 == 0, "stages must keep the 1024-byte alignment of the 128-byte swizzle");
};

struct PairPlan {
  int poff[33];
  int cnt[32];
  int eorder[32];     // weight-gradient problems: experts by row count, largest first (ties: lower id)
  int ntiles[2];
  int nm[2];          // kgrouped problems: 256-row tiles of each [M, N] output
  int nn[2];          // column tiles per row block: nfull of width BN, then one of width nrem if nrem > 0
  int nfull[2];
  int nrem[2];
  int total;
};

struct PairTile {
  int p, row0, valid, brow, n0, width, e, nk;
  int k0;             // first K row of the operands held MN-major (rows = K)
  int bk0;            // first K row of an MN-major B (an expert's block of the weights, or k0)
};

template <int BN, bool BWD>
__device__ __forceinline__ PairTile pair_decode(int tile, const PairPlan& pl, const GemmArgs& a) {
  PairTile ti;
  int t = tile;
  ti.p = 0;
  if (t >= pl.ntiles[0]) { t -= pl.ntiles[0]; ti.p = 1; }
  const GemmProblem& pr = a.p[ti.p];
  ti.k0 = 0;
  ti.bk0 = 0;
  if (BWD && pr.kgrouped) {
    // weight gradient: tiles of expert e's [M, N] output; the reduction runs over the expert's
    // rows of the permuted buffers (a dense problem has one segment of K rows)
    const int per = pl.nm[ti.p] * pl.nn[ti.p];
    const int e = pr.routed ? pl.eorder[t / per] : t / per, r = t % per;
    const int mt = r / pl.nn[ti.p], nt = r % pl.nn[ti.p];
    ti.e = e;
    ti.row0 = mt * kPairBM;
    ti.n0 = nt * BN;
    ti.width = nt < pl.nfull[ti.p] ? BN : pl.nrem[ti.p];
    const int v = pr.M - ti.row0;
    ti.valid = v < kPairBM ? v : kPairBM;
    ti.brow = 0;
    if (pr.routed) {
      ti.k0 = pl.poff[e];
      ti.nk = (pl.cnt[e] + kPairBK - 1) / kPairBK;
    } else {
      ti.nk = (pr.K + kPairBK - 1) / kPairBK;
    }
    ti.bk0 = ti.k0;
    return ti;
  }
  const int mt = t / pl.nn[ti.p], nt = t % pl.nn[ti.p];
  ti.row0 = mt * kPairBM;
  ti.n0 = nt * BN;
  ti.width = nt < pl.nfull[ti.p] ? BN : pl.nrem[ti.p];
  ti.nk = pr.K / kPairBK;
  if (pr.routed) {
    int e = 0;
    while (e < a.E - 1 && ti.row0 >= pl.poff[e + 1]) ++e;
    ti.e = e;
    const int v = pl.poff[e] + pl.cnt[e] - ti.row0;
    ti.valid = v < kPairBM ? v : kPairBM;
    ti.brow = e * pr.N + ti.n0;
    ti.bk0 = e * pr.K;                 // MN-major B: expert e's weights are rows [e K, (e + 1) K)
  } else {
    ti.e = 0;
    const int v = pr.M - ti.row0;
    ti.valid = v < kPairBM ? v : kPairBM;
    ti.brow = ti.n0;
  }
  return ti;
}

// Next tile id of a consumer role (lane 0): wait for the ring slot, read it, and release the
// slot on the leader.  -1: no tile left (or a wait ran out, recorded in the status word).
__device__ __forceinline__ int sched_take(uint64_t* sfull, uint64_t* sempty, volatile int* stile, uint32_t& n,
                                          uint32_t rank, volatile int* abort_flag, int* status, int where) {
  const uint32_t slot = n % kSchedSlots, ph = (n / kSchedSlots) & 1u;
  ++n;
  if (!mbar_wait_cluster(smem_u32(&sfull[slot]), ph, abort_flag, status, where)) return -1;
  const int t = stile[slot];
  if (rank == 0) mbar_arrive(smem_u32(&sempty[slot]));       // the leader's own roles: CTA scope
  else mbar_arrive_release_cluster(map_to_cta(smem_u32(&sempty[slot]), 0));
  return t;
}

// Leader producer (lane 0): hand tile id t (-1 = none left) to both CTAs' ring once the slot
// is free.  False when the wait ran out.
__device__ __forceinline__ bool sched_publish(uint64_t* sfull, uint64_t* sempty, volatile int* stile, uint32_t& n,
                                              int t, volatile int* abort_flag, int* status) {
  const uint32_t slot = n % kSchedSlots, ph = (n / kSchedSlots) & 1u;
  ++n;
  if (!mbar_wait_cluster(smem_u32(&sempty[slot]), ph ^ 1u, abort_flag, status, 507)) return false;
  stile[slot] = t;
  st_shared_cluster_s32(map_to_cta(smem_u32((const void*)&stile[slot]), 1), t);
  mbar_arrive(smem_u32(&sfull[slot]));
  mbar_arrive_release_cluster(map_to_cta(smem_u32(&sfull[slot]), 1));
  return true;
}

// Claim the next tile of the launch (-1 when every tile is taken).
__device__ __forceinline__ int sched_claim(unsigned int* ctr, int total) {
  const int t = (int)atomicAdd(ctr, 1u);
  return t < total ? t : -1;
}

template <int BN, typename S, int F>
__global__ void __launch_bounds__(pair_threads<F>(), 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap tb0,
                 const __grid_constant__ CUtensorMap ta1, const __grid_constant__ CUtensorMap tb1,
                 const __grid_constant__ CUtensorMap to0, const __grid_constant__ CUtensorMap to1,
                 const __grid_constant__ CUtensorMap tbn0, const __grid_constant__ CUtensorMap tbn1, GemmArgs a) {
  constexpr int kKps = pair_kps<F>();
  using C = PairCfg<BN, kKps>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + C::STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_base + C::EPI_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* sched_full = drain + 1;
  uint64_t* sched_empty = sched_full + kSchedSlots;
  volatile int* sched_tile = reinterpret_cast<volatile int*>(sched_empty + kSchedSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_empty + kSchedSlots) + kSchedSlots;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ PairPlan pl;

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();          // 0 = leader of the pair
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  // tiles claimed in order (the folded combine's guarantee of progress) or a fixed order
  constexpr bool kClaim = (F & kFeatClaim) != 0, kGather = (F & kFeatGather) != 0, kBwd = (F & kFeatBwd) != 0;
  // claimed in order: the folded combine (its guarantee of progress) and the weight-gradient
  // launches (tiles of very different lengths, longest first)
  const bool dyn = kClaim && a.sched_ctr != nullptr;
  // the routed A rows come from x through the gather warps (GEMM1 only: fixed tile order)
  const bool gather_lsu = kGather && a.p[0].gather_rows != nullptr;
  // launched as a programmatic dependent: wait here for the kernel before (its rows, offsets and
  // outputs), and let the next one get resident as this grid's CTAs finish
  grid_dependency_wait();
  launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      // leader: its producer's expect_tx arrive (+ one arrive per gather warp of both CTAs)
      mbar_init(smem_u32(&full[s]), gather_lsu ? 1 + 2 * kPairGatherWarps : 1);
      mbar_init(smem_u32(&empty[s]), 1);            // one MMA-completion commit per phase
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), 2 * kPairEpiWarps);   // leader: every epilogue warp of both CTAs
    }
    mbar_init(smem_u32(drain), 1);
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(smem_u32(&sched_full[i]), 1);                  // the leader producer's hand-over
      mbar_init(smem_u32(&sched_empty[i]), kSchedConsumers);  // leader: every consumer role of the pair
    }
    *abort_flag = 0;
    fence_barrier_init();
    bool bad = false;
    int p = 0;
    pl.poff[0] = 0;
    for (int e = 0; e < a.E; ++e) {
      int c = a.offsets ? a.offsets[e + 1] - a.offsets[e] : 0;
      if (c < 0) { c = 0; bad = true; }
      pl.cnt[e] = c;
      p += (c + kSegAlign - 1) / kSegAlign * kSegAlign;
      pl.poff[e + 1] = p;
    }
    if ((long long)p > a.r_max) bad = true;
    for (int e = 0; e < a.E; ++e) {                 // insertion sort, stable: largest count first
      int j = e;
      while (j > 0 && pl.cnt[pl.eorder[j - 1]] < pl.cnt[e]) {
        pl.eorder[j] = pl.eorder[j - 1];
        --j;
      }
      pl.eorder[j] = e;
    }
    for (int q = 0; q < 2; ++q) {
      if (q >= a.nprob) { pl.ntiles[q] = 0; pl.nn[q] = 1; pl.nm[q] = 1; pl.nfull[q] = 1; pl.nrem[q] = 0; continue; }
      const GemmProblem& pr = a.p[q];
      pl.nfull[q] = pr.N / BN;
      pl.nrem[q] = pr.N % BN;
      pl.nn[q] = pl.nfull[q] + (pl.nrem[q] ? 1 : 0);
      pl.nm[q] = (pr.M + kPairBM - 1) / kPairBM;
      if (kBwd && pr.kgrouped) {
        pl.ntiles[q] = (pr.routed ? (bad ? 0 : a.E) : 1) * pl.nm[q] * pl.nn[q];
        continue;
      }
      const int mt = pr.routed ? (bad ? 0 : p / kPairBM) : (pr.M + kPairBM - 1) / kPairBM;
      pl.ntiles[q] = mt * pl.nn[q];
    }
    pl.total = pl.ntiles[0] + pl.ntiles[1];
    if (bad && rank == 0 && blockIdx.x == 0) set_status(a.status, DEV_BAD_INDEX, 500);
    prefetch_tmap(&ta0);
    prefetch_tmap(&tb0);
    prefetch_tmap(&ta1);
    prefetch_tmap(&tb1);
    prefetch_tmap(&to0);
    prefetch_tmap(&to1);
    if (a.b_half) {
      prefetch_tmap(&tbn0);
      prefetch_tmap(&tbn1);
    }
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                   // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Lane 0 loads the tiles.  When the routed problem gathers its A rows, it loads only B:
    // the two gather warps copy this CTA's 128 A rows into the stage with cp.async and
    // arrive on the leader's full barrier themselves.
    const uint64_t pol_w = policy_evict_last();
    // A tiles are reused by every column tile of their row block (consecutive tiles, run
    // side by side): keep them in L2 normally; evict-first sent them back to DRAM 3.5x
    const uint64_t pol_a = policy_evict_normal();
    int stage = 0;
    uint32_t phase = 0;
    bool alive = true;
    uint32_t sn = 0;
    int next = (dyn && rank == 0 && lane == 0) ? sched_claim(a.sched_ctr, pl.total) : -1;
    int kstat = 0;                                  // fixed order: this pair's k-th tile is cid + k * ncl
    while (alive) {
      // the leader hands its claimed tile to both CTAs and claims the one after it while the
      // loads go out; the peer takes the tile from its ring
      int tile = -1, ok = 1;
      if (!dyn) {
        tile = cid + kstat * ncl;
        ++kstat;
        if (tile >= pl.total) tile = -1;
      } else if (lane == 0) {
        if (rank == 0) {
          tile = next;
          ok = sched_publish(sched_full, sched_empty, sched_tile, sn, tile, abort_flag, a.status) ? 1 : 0;
          if (ok && tile >= 0) next = sched_claim(a.sched_ctr, pl.total);
        } else {
          tile = sched_take(sched_full, sched_empty, sched_tile, sn, rank, abort_flag, a.status, 508);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (!ok) { alive = false; break; }
      if (tile < 0) break;
      const PairTile ti = pair_decode<BN, kBwd>(tile, pl, a);
      const GemmProblem& pr = a.p[ti.p];
      const CUtensorMap* tA = ti.p ? &ta1 : &ta0;
      const CUtensorMap* tB = ti.p ? &tb1 : &tb0;
      const int ksplit = pr.ksplit;
      const int nrows = pr.N;
      const bool gather = kGather && pr.gather_rows != nullptr;   // the gather warps bring this tile's A rows
      // a tile at most BN/2 wide reads BN/4 B rows per CTA: load only those (a 16 KB box would bring
      // twice the B bytes the MMAs use, and these tiles are bound by their operand loads)
      const bool half_b = a.b_half && 2 * ti.width <= BN && !(kBwd && pr.b_mn);
      const CUtensorMap* tBk = half_b ? (ti.p ? &tbn1 : &tbn0) : tB;
      const uint32_t bbytes = half_b ? C::B_BYTES / 2 : C::B_BYTES;
      for (int kb0 = 0; kb0 < ti.nk; kb0 += kKps) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.status, 501) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { alive = false; break; }
        const uint32_t fb_local = smem_u32(&full[stage]);
        const uint32_t fb_leader = map_to_cta(fb_local, 0);
        // the stage's k-blocks (the last stage of a tile may hold fewer), each an A box then a B box
        const int nkb = ti.nk - kb0 < kKps ? ti.nk - kb0 : kKps;
        if (lane == 0) {
          if (rank == 0)                                  // both CTAs' TMA bytes
            mbar_arrive_expect_tx(fb_local, (uint32_t)nkb * (gather ? 2 * bbytes : 2 * (C::A_BYTES + bbytes)));
          for (int j = 0; j < nkb; ++j) {
            const int kb = kb0 + j;
            uint8_t* sa = stage_base + stage * C::STAGE + j * C::KB_BYTES;
            const int bx = ksplit ? (kb * kPairBK) % ksplit : kb * kPairBK;
            // each CTA holds half of the tile's B rows (for a tile between BN/2 and BN wide, the box also
            // brings rows it does not use)
            const int by = (ksplit ? ((kb * kPairBK) / ksplit) * nrows : 0) + ti.brow + (int)rank * (ti.width / 2);
            if (kBwd && pr.a_mn) {
              // A held [K rows, M columns]: this CTA's 128 M columns as two 64-column boxes of 64 K rows
              const int ax = ti.row0 + (int)rank * 128, ay = ti.k0 + kb * kPairBK;
              tma_load_2d_pair(smem_u32(sa), tA, ax, ay, fb_leader, pol_a);
              tma_load_2d_pair(smem_u32(sa) + 8192, tA, ax + 64, ay, fb_leader, pol_a);
            } else if (!gather) {
              tma_load_2d_pair(smem_u32(sa), tA, kb * kPairBK, ti.row0 + (int)rank * 128, fb_leader, pol_a);
            }
            if (kBwd && pr.b_mn) {
              // B held [K rows, N columns]: this CTA's half of the tile's columns as two 64-column boxes
              // (a narrower tile's second box brings columns it does not use, zeros past the tensor)
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const int n = ti.n0 + (int)rank * (ti.width / 2) + 64 * i;
                int x = n, y = ti.bk0 + kb * kPairBK;
                if (pr.b_split) { x = n % pr.b_split; y += (n / pr.b_split) * pr.K; }
                tma_load_2d_pair(smem_u32(sa + C::A_BYTES) + 8192 * i, tB, x, y, fb_leader, pol_w);
              }
            } else {
              tma_load_2d_pair(smem_u32(sa + C::A_BYTES), tBk, bx, by, fb_leader, pol_w);
            }
          }
        }
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    __syncwarp();
    if (!alive) goto done;
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false;
      uint32_t sn = 0;
      for (int local = 0;; ++local) {
        int tile = cid + local * ncl;
        if (dyn) tile = sched_take(sched_full, sched_empty, sched_tile, sn, rank, abort_flag, a.status, 509);
        else if (tile >= pl.total) tile = -1;
        if (tile < 0) break;
        const PairTile ti = pair_decode<BN, kBwd>(tile, pl, a);
        const int acc = local & 1;
        const uint32_t accph = (local >> 1) & 1;
        if (!mbar_wait(smem_u32(&acc_empty[acc]), accph ^ 1u, abort_flag, a.status, 502)) goto mma_out;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        const GemmProblem& pr = a.p[ti.p];
        const bool amn = kBwd && pr.a_mn, bmn = kBwd && pr.b_mn;
        const uint32_t idesc = idesc_f16kind_f32(kPairBM, ti.width, S::kFmt) | (kBwd ? idesc_major_bits(amn, bmn) : 0u);
        // a k16 step advances 32 bytes inside a K-major row, or 16 rows (2048 bytes) of an MN-major tile
        const uint64_t astep = amn ? 128 : 2, bstep = bmn ? 128 : 2;
        for (int kb0 = 0; kb0 < ti.nk; kb0 += kKps) {
          // gathered rows arrive from both CTAs' gather warps (cluster scope); else TMA only
          if (!(gather_lsu ? mbar_wait_cluster(smem_u32(&full[stage]), phase, abort_flag, a.status, 503)
                           : mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.status, 503)))
            goto mma_out;
          tc_fence_after();
          const int nkb = ti.nk - kb0 < kKps ? ti.nk - kb0 : kKps;
          for (int j = 0; j < nkb; ++j) {
            const uint32_t sa = smem_u32(stage_base + stage * C::STAGE + j * C::KB_BYTES);
            const uint64_t adesc = amn ? smem_desc_mn_sw128(sa) : smem_desc_sw128(sa);
            const uint64_t bdesc = bmn ? smem_desc_mn_sw128(sa + C::A_BYTES) : smem_desc_sw128(sa + C::A_BYTES);
#pragma unroll
            for (int kk = 0; kk < kPairBK / 16; ++kk)
              umma_kindf16_pair(d, adesc + astep * kk, bdesc + bstep * kk, idesc, ((kb0 + j) | kk) ? 1u : 0u);
          }
          issued_any = true;
          // stage free in both CTAs once these MMAs finish
          const uint32_t eb = smem_u32(&empty[stage]);
          umma_commit_pair(eb);
          umma_commit_pair(map_to_cta(eb, 1));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        const uint32_t fb = smem_u32(&acc_full[acc]);   // accumulator ready in both CTAs
        umma_commit_pair(fb);
        umma_commit_pair(map_to_cta(fb, 1));
      }
    mma_out:
      if (issued_any) {
        umma_commit_pair(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0, nullptr, a.status, 504);
      }
    }
    __syncwarp();
  } else if (warp < 2 + kPairEpiWarps) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Each warp owns 32 TMEM lanes = 32 rows of this CTA's half, and every
    // kPairEpiSplit-th column box of the tile (the warps of one lane quadrant
    // share its boxes).  Per 128-byte column box it loads the accumulator,
    // applies the epilogue, writes the 32 x 128-byte box into a swizzled shared
    // buffer and hands it to a TMA store (two buffers per warp, so a store
    // overlaps the next box).
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;               // which of the quadrant's warps
    const int r = q * 32 + lane;                   // row inside this CTA's 128-row half
    const uint32_t acc_empty_leader0 = map_to_cta(smem_u32(&acc_empty[0]), 0);
    const uint32_t acc_empty_leader1 = map_to_cta(smem_u32(&acc_empty[1]), 0);
    const uint32_t sbuf = smem_u32(epi_base + (warp - 2) * 8192);
    // combine folded into the shared tiles: every epilogue warp of both CTAs counts each routed tile
    const bool count_routed = a.nprob > 1 && a.p[1].epi == 2 && a.done_ctr != nullptr;
    const unsigned int done_target = (unsigned int)pl.ntiles[0] * 2u * kPairEpiWarps;
    // test words (host-written, zero in normal use): bit 0 of word 0 makes the routed tiles skip
    // their count, so the shared tiles' wait cannot end; word 1 shortens that wait to microseconds
    const uint32_t tflags = (count_routed && a.test != nullptr) ? __ldcg(a.test) : 0u;
    const uint32_t tlimit_us = (count_routed && a.test != nullptr) ? __ldcg(a.test + 1) : 0u;
    const uint64_t done_limit = tlimit_us ? (uint64_t)tlimit_us * 1000ull : kWaitLimitNs;
    bool routed_done = false;
    int nstore = 0;
    uint32_t sn = 0;
    for (int local = 0;; ++local) {
      int tile = cid + local * ncl;
      if (dyn) {
        if (lane == 0) tile = sched_take(sched_full, sched_empty, sched_tile, sn, rank, abort_flag, a.status, 510);
        tile = __shfl_sync(0xffffffffu, tile, 0);
      } else if (tile >= pl.total) {
        tile = -1;
      }
      if (tile < 0) break;
      const PairTile ti = pair_decode<BN, kBwd>(tile, pl, a);
      const GemmProblem& pr = a.p[ti.p];
      const CUtensorMap* tO = ti.p ? &to1 : &to0;
      if (kBwd && !dyn) {
        // GELU backward: bring this lane's row of u for the pair's next tile (fixed order) into L2
        // now, a tile ahead of its loads; the epilogue's own loads reach only one box ahead
        const int nt_ = tile + ncl;
        if (nt_ < pl.total) {
          const PairTile tn = pair_decode<BN, kBwd>(nt_, pl, a);
          const GemmProblem& pn = a.p[tn.p];
          if (pn.epi == 4 && pn.aux != nullptr && r < tn.valid - (int)rank * 128) {
            const uint16_t* un = reinterpret_cast<const uint16_t*>(pn.aux) +
                                 ((long long)tn.row0 + (int)rank * 128 + r) * pn.N + tn.n0;
            for (int c = 0; c < tn.width; c += 64) prefetch_l2(un + c);
          }
        }
      }
      const int acc = local & 1;
      const uint32_t accph = (local >> 1) & 1;
      if (!mbar_wait(smem_u32(&acc_full[acc]), accph, abort_flag, a.status, 505)) break;
      tc_fence_after();
      const int valid_here = ti.valid - (int)rank * 128;
      const bool rv = r < valid_here;
      const long long grow = (long long)ti.row0 + (int)rank * 128 + r;
      const int box_row = ti.row0 + (int)rank * 128 + q * 32;
      const float gate = (pr.gate != nullptr && rv) ? pr.gate[grow] : 1.0f;
      const uint16_t* bias =
          pr.bias ? reinterpret_cast<const uint16_t*>(pr.bias) + (long long)ti.e * pr.bias_stride : nullptr;
      constexpr int box_cols = 64;                          // 128 bytes of 16-bit h or y
      // tanh GELU, erf GELU, gate, the combine (routed rows + shared output), or the GELU backward
      const int mode = pr.epi == 0 ? (a.act == 1 ? 1 : 0) : (pr.epi == 2 ? 3 : ((kBwd && pr.epi == 4) ? 4 : 2));
      float dgacc = 0.f;
      int ns = 0;
      const int32_t* prow = nullptr;
      if (mode == 3) {
        if (!routed_done) {
          // every routed tile of this launch has its y rows stored (bounded wait)
          if (lane == 0) {
            const uint64_t t0 = global_ns();
            while (ld_acquire_gpu_u32(a.done_ctr) < done_target) {
              if (global_ns() - t0 > done_limit) { set_status(a.status, DEV_TIMEOUT, 506); break; }
              __nanosleep(64);
            }
          }
          __syncwarp();
          routed_done = true;
        }
        if (rv) {
          ns = a.n_sel ? a.n_sel[grow] : a.kdef;
          ns = ns < 0 ? 0 : (ns > a.kmax ? a.kmax : ns);
          prow = a.pos + grow * a.kmax;
        }
      }
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      if (kBwd && pr.out_f32) {
        // weight gradients: 32 fp32 columns per box through the 3-D output map [z, M, N] (rows past
        // M are clipped by the map); a tile with no reduction rows (an expert that took no token)
        // stores zeros
#pragma unroll 1
        for (int c0 = grp * 32; c0 < ti.width; c0 += 32 * kPairEpiSplit) {
          uint32_t v[32];
          if (ti.nk > 0) {
            tmem_ld_32x32b_x32(tbase + c0, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0u;
          }
          const uint32_t buf = sbuf + (nstore & 1) * 4096;
          if (lane == 0) bulk_wait_read_le1();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + lane * 128 + ((j ^ (lane & 7)) << 4)),
                         "r"(v[4 * j]), "r"(v[4 * j + 1]), "r"(v[4 * j + 2]), "r"(v[4 * j + 3])
                         : "memory");
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            const int col = ti.n0 + c0;
            int x = col, z = (pr.kgrouped && pr.routed) ? ti.e : 0;
            if (pr.out_split) { z = col / pr.out_split; x = col % pr.out_split; }
            tma_store_3d(tO, buf, x, box_row, z);
            bulk_commit();
          }
          ++nstore;
        }
      } else {
      // GELU backward: the stored pre-activation u of the row's next box (64 columns), loaded one
      // box ahead so that its latency hides behind the current box's work.  Plain (L1-cached) loads:
      // a lane's eight 16-byte loads of a box share its row's 128-byte line, which each address
      // is read once before dU overwrites it (L1 holds no stale copy a later load could see)
      const uint16_t* urow = (kBwd && mode == 4 && rv)
                                 ? reinterpret_cast<const uint16_t*>(pr.aux) + grow * pr.N + ti.n0 : nullptr;
      uint4 unext[8];
      if (kBwd && mode == 4) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          unext[u] = (urow && grp * box_cols < ti.width)
                         ? *(reinterpret_cast<const uint4*>(urow + grp * box_cols) + u) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll 1
      for (int c0 = grp * box_cols; c0 < ti.width; c0 += box_cols * kPairEpiSplit) {
        uint4 o[8];
        uint4 ucur[8];
        if (kBwd && mode == 4) {
          const int cn = c0 + box_cols * kPairEpiSplit;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            ucur[u] = unext[u];
            unext[u] = (urow && cn < ti.width) ? *(reinterpret_cast<const uint4*>(urow + cn) + u)
                                               : make_uint4(0u, 0u, 0u, 0u);
          }
        }
        uint32_t vv[2][32];
        tmem_ld_32x32b_x32(tbase + c0, vv[0]);
        tmem_ld_32x32b_x32(tbase + c0 + 32, vv[1]);
        tmem_ld_wait();                              // both halves in flight before one wait
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half * 32 >= box_cols) break;
          const int cc = c0 + half * 32;
          uint32_t* v = vv[half];
          const int col0 = ti.n0 + cc;
          if (bias) {
            // acc + (the bias rows' sum, in row order): one fp32 add per element, kept in v
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float bs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
              for (int br = 0; br < pr.bias_rows; ++br) {
                float t8[8];
                S::x8_to_f32(__ldg(reinterpret_cast<const uint4*>(bias + (long long)br * pr.N + col0) + u), t8);
#pragma unroll
                for (int j = 0; j < 8; ++j) bs[j] += t8[j];
              }
#pragma unroll
              for (int j = 0; j < 8; ++j) v[8 * u + j] = __float_as_uint(__uint_as_float(v[8 * u + j]) + bs[j]);
            }
          }
          // GEMM1: gelu(acc + b1); GEMM2: gate * (acc + b2); both rounded once to 16 bits.  The
          // mode is uniform per tile, so each element loop holds one form only.
          uint32_t* ow = reinterpret_cast<uint32_t*>(&o[half * 4]);
          if (mode == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              ow[j / 2] = S::pack2(gelu_act<true>(__uint_as_float(v[j]), 0), gelu_act<true>(__uint_as_float(v[j + 1]), 0));
          } else if (mode == 1) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              ow[j / 2] = S::pack2(gelu_act<true>(__uint_as_float(v[j]), 1), gelu_act<true>(__uint_as_float(v[j + 1]), 1));
          } else if (mode == 2) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              ow[j / 2] = S::pack2(__uint_as_float(v[j]) * gate, __uint_as_float(v[j + 1]) * gate);
          } else if (kBwd && mode == 4) {
            // GELU backward: acc = dY W (ungated), u the stored pre-activation of these columns;
            // dU = gate * acc * gelu'(u) (zero on padding rows), and the row's sum of acc * gelu(u)
            float uf[32];                            // zeros on padding rows (ucur is zero there)
#pragma unroll
            for (int u4 = 0; u4 < 4; ++u4) S::x8_to_f32(ucur[half * 4 + u4], uf + 8 * u4);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float g0, d0, g1, d1;
              gelu_tanh_and_grad<true>(uf[j], g0, d0);
              gelu_tanh_and_grad<true>(uf[j + 1], g1, d1);
              const float a0 = __uint_as_float(v[j]), a1 = __uint_as_float(v[j + 1]);
              dgacc = fmaf(a0, g0, dgacc);
              dgacc = fmaf(a1, g1, dgacc);
              ow[j / 2] = S::pack2(rv ? gate * a0 * d0 : 0.f, rv ? gate * a1 * d1 : 0.f);
            }
          } else {
            // out = sum over the token's slots of its routed rows (slot order), plus the shared output
            float y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = 0.f;
            for (int k = 0; k < ns; ++k) {
              const int pr_row = __ldcg(prow + k);
              if (pr_row < 0 || pr_row >= a.r_max) continue;
              const uint4* yp = reinterpret_cast<const uint4*>(
                  reinterpret_cast<const uint16_t*>(a.y_routed) + (long long)pr_row * pr.N + col0);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                float t8[8];
                S::x8_to_f32(__ldcg(yp + u), t8);
#pragma unroll
                for (int j = 0; j < 8; ++j) y[8 * u + j] += t8[j];
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] += __uint_as_float(v[j]);
            if (a.x_res != nullptr && rv) {
              // adaLN-Zero residual: x_res + alpha[image] * (layer output)
              const uint4* xp = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.x_res) +
                                                               grow * pr.N + col0);
              const uint4* ap = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.alpha) +
                                                               (grow / a.img_len) * pr.N + col0);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                float r8[8], g8[8];
                S::x8_to_f32(__ldg(xp + u), r8);
                S::x8_to_f32(__ldg(ap + u), g8);
#pragma unroll
                for (int j = 0; j < 8; ++j) y[8 * u + j] = r8[j] + g8[j] * y[8 * u + j];
              }
            }
#pragma unroll
            for (int j = 0; j < 32; j += 2) ow[j / 2] = S::pack2(y[j], y[j + 1]);
          }
        }
        // stage the 32 x 128-byte box (128-byte swizzle) and store it with TMA; rows past the
        // segment's tokens are padding rows of the permuted buffers (or clipped past T)
        const uint32_t buf = sbuf + (nstore & 1) * 4096;
        if (lane == 0) bulk_wait_read_le1();   // the store that last used this buffer has read it
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + lane * 128 + ((j ^ (lane & 7)) << 4)),
                       "r"(o[j].x), "r"(o[j].y), "r"(o[j].z), "r"(o[j].w)
                       : "memory");
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tO, buf, ti.n0 + c0, box_row);
          bulk_commit();
        }
        ++nstore;
      }
      if (kBwd && mode == 4 && pr.dg != nullptr && rv) pr.dg[grow * pr.dg_stride + (ti.n0 / BN) * kPairEpiSplit + grp] = dgacc;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? acc_empty_leader1 : acc_empty_leader0);
      if (count_routed && ti.p == 0 && lane == 0 && !(tflags & 1u)) {
        // this warp's rows of a routed tile are in global memory: count them for the combine
        bulk_wait_all();
        fence_proxy_async_all();
        __threadfence();
        atomicAdd(a.done_ctr, 1u);
        __threadfence();                           // the count lands before this CTA reports its exit
      }
    }
    if (lane == 0) bulk_wait_all();            // stores done before the CTA may exit
  } else if (kGather && gather_lsu) {
    // ------------------------------------------------------------ row gather (both CTAs)
    // Thread u of the two warps copies 16-byte chunk u % 8 of this CTA's rows u / 8 + 8 i
    // (i < 16) of every stage of a routed tile: row r of the tile is row row_token[r] of x
    // (padding rows read row 0; their results are never used).  Each stage is one cp.async
    // group; when a stage's group is kLag groups old it has landed: fence it for the tensor
    // cores (async proxy) and arrive on the leader's barrier of that stage.  Stages of the
    // shared problem (A by TMA) are reported too, with empty groups, so every stage's barrier
    // counts the same arrivals.  kLag < STAGES: a stage is reported before its ring slot is
    // needed again.
    constexpr int kLag = 2;
    const int u = (warp - 2 - kPairEpiWarps) * 32 + lane;
    const int cq = u & 7, rq = u >> 3;
    const GemmProblem& pg = a.p[0];
    const uint16_t* xa = reinterpret_cast<const uint16_t*>(pg.A);
    const long long ld = pg.K;
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    auto report = [&](int s) {
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive_release_cluster(map_to_cta(smem_u32(&full[s]), 0));
    };
    for (int k = 0;; ++k) {
      const int tile = cid + k * ncl;
      if (tile >= pl.total) break;
      const PairTile ti = pair_decode<BN, kBwd>(tile, pl, a);
      const bool mine = ti.p == 0;
      int rowid[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        int v = 0;
        if (mine) {
          v = __ldg(pg.gather_rows + (long long)ti.row0 + (int)rank * 128 + rq + 8 * i);
          v = (v >= 0 && v < pg.gather_nrows) ? v : 0;
        }
        rowid[i] = v;
      }
      for (int kb = 0; kb < ti.nk; ++kb) {
        int okw = 1;
        if (lane == 0) okw = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.status, 511) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) {
          cp_async_wait<0>();                       // nothing of this warp's left in flight
          goto gather_out;
        }
        if (mine) {
          const uint32_t sa = smem_u32(stage_base + stage * C::STAGE);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = rq + 8 * i;
            cp_async_16(sa + r * 128 + ((cq ^ (r & 7)) << 4), xa + (long long)rowid[i] * ld + kb * kPairBK + cq * 8);
          }
        }
        cp_async_commit();
        if (issued >= kLag) {
          cp_async_wait<kLag>();
          report((stage - kLag + C::STAGES) % C::STAGES);
        }
        ++issued;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait<0>();
    for (int n = issued > kLag ? issued - kLag : 0; n < issued; ++n) report(n % C::STAGES);
  gather_out:;
  }
done:
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                   // no CTA leaves while its peer may still use it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  if (threadIdx.x == 0) {
    // the last CTA out resets the tile counter and the combine count for the next launch (every
    // claim of every CTA has returned before its exit is counted; the fixed order claims nothing)
    __threadfence();
    if (atomicAdd(a.exit_ctr, 1u) == gridDim.x - 1) {
      *a.sched_ctr = 0u;
      if (a.done_ctr != nullptr) *a.done_ctr = 0u;
      *a.exit_ctr = 0u;
      __threadfence();
    }
  }
}

template <int BN, typename S, int F>
static cudaError_t launch_pair_bn(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb,
                                  const CUtensorMap* to, const CUtensorMap* tbn, int num_sms, int max_pairs,
                                  cudaStream_t s) {
  using C = PairCfg<BN, pair_kps<F>()>;
  cudaError_t err = cudaFuncSetAttribute(gemm_pair_kernel<BN, S, F>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms & ~1, 1, 1);
  cfg.blockDim = dim3(pair_threads<F>(), 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // pairs the device can hold at once (one per TPC normally; fewer on a partitioned device):
  // asked once per device, then at most that many are launched
  static std::mutex mu;
  static int fit[kMaxDevicesCached] = {0};
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  int pairs = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < kMaxDevicesCached && fit[dev] > 0) {
      pairs = fit[dev];
    } else {
      err = cudaOccupancyMaxActiveClusters(&pairs, gemm_pair_kernel<BN, S, F>, &cfg);
      if (err != cudaSuccess) return err;
      if (pairs < 1) return cudaErrorInvalidConfiguration;
      if (dev >= 0 && dev < kMaxDevicesCached) fit[dev] = pairs;
    }
  }
  const int grid = pair_grid(num_sms, pairs, max_pairs);
  if (grid < 2) return cudaErrorInvalidConfiguration;
  cfg.gridDim = dim3(grid, 1, 1);
  GemmArgs ak = a;
  ak.b_half = tbn != nullptr ? 1 : 0;
  const CUtensorMap* tn = tbn != nullptr ? tbn : tb;
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<BN, S, F>, ta[0], tb[0], ta[1], tb[1], to[0], to[1], tn[0], tn[1],
                            ak);
}

// Tiles are 256 columns wide, with one narrower tile (a multiple of 64 columns)
// for the rest of a row block: N = 1152 runs as 4 x 256 + 128, so each A row
// block is read 4.5 times instead of 6 (192-wide tiles).
int gemm_pair_pick_bn(int n0, int n1) {
  if (n0 % 64 == 0 && (n1 == 0 || n1 % 64 == 0)) return 256;
  return 0;
}

cudaError_t launch_gemm_pair(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb, const CUtensorMap* to,
                             const CUtensorMap* tbn, int bn, int num_sms, int max_pairs, cudaStream_t s) {
  if (bn != 256) return cudaErrorInvalidValue;
  int f = 0;
  if (a.nprob > 1 && a.p[1].epi == 2 && a.done_ctr != nullptr) f |= kFeatClaim;
  if (a.p[0].gather_rows != nullptr) f |= kFeatGather;
  for (int q = 0; q < a.nprob && q < 2; ++q) {
    const GemmProblem& p = a.p[q];
    if (p.a_mn || p.b_mn || p.kgrouped || p.out_f32 || p.epi == 4) f |= kFeatBwd;
    if (p.kgrouped) f |= kFeatClaim;
  }
  if ((f & kFeatClaim) && a.sched_ctr == nullptr) return cudaErrorInvalidValue;
#define MOE_PAIR_LAUNCH(FEAT)                                                                    \
  case FEAT:                                                                                     \
    return a.f16 ? launch_pair_bn<256, StoreF16, FEAT>(a, ta, tb, to, tbn, num_sms, max_pairs, s)    \
                 : launch_pair_bn<256, StoreBF16, FEAT>(a, ta, tb, to, tbn, num_sms, max_pairs, s);
  switch (f) {
    MOE_PAIR_LAUNCH(0)
    MOE_PAIR_LAUNCH(kFeatClaim)
    MOE_PAIR_LAUNCH(kFeatGather)
    MOE_PAIR_LAUNCH(kFeatBwd)
    MOE_PAIR_LAUNCH(kFeatBwd | kFeatClaim)
    default:
      return cudaErrorNotSupported;                 // no instantiation gathers rows and claims tiles
  }
#undef MOE_PAIR_LAUNCH
}

}  // namespace moe
