// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One persistent launch computes every 128 x BN output tile of up to two
// problems: the routed experts (rows grouped in 256-aligned expert segments,
// segment bounds read on the device from the dispatch offsets) and the shared
// experts (dense rows, packed weights).  Expert MLP = W2 gelu(W1 x) ("Scaling
// Diffusion Transformers to 16 Billion Parameters", "MOE-DIT" eq. MLP; tanh
// GELU per "Scalable Diffusion Models with Transformers", DiT block details),
// each expert a pair of these GEMMs:
//   GEMM1 epilogue: + b1, GELU, round to 16 bits        -> h
//   GEMM2 epilogue: + b2, times the row's gate (routed)  -> y (16 bits)
//
// CTA = 6 warps: warp 0 issues TMA loads (128-byte swizzled K-major tiles) into
// a ring of shared-memory stages; warp 1 allocates TMEM and one thread issues
// tcgen05.mma (M=128, N=BN, K=16, fp32 accumulate) into one of two TMEM
// accumulators; warps 2-5 drain the other accumulator with tcgen05.ld, apply
// the epilogue and store, so the epilogue of tile i overlaps the MMAs of tile
// i+1.  Every wait is bounded (1 s) and records a timeout instead of hanging.
#include <cuda.h>
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kBM = 128;
constexpr int kBK = 64;                 // 16-bit elements in one 128-byte swizzle row
constexpr int kTcThreads = 192;
constexpr int kSmemLimit = 232448;      // 227 KB opt-in dynamic shared memory per block

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int FIT = (kSmemLimit - 2048) / STAGE;
  static constexpr int STAGES = FIT > 8 ? 8 : FIT;
  static constexpr int SMEM = STAGES * STAGE + 2048;
  static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
};

struct TilePlan {
  int poff[33];      // padded segment starts (routed problem)
  int cnt[32];
  int ntiles[2];
  int nn[2];         // n-tiles per m-tile
  int total;
};

struct TileInfo {
  int p, row0, valid, brow, n0, e, nk;
};

template <int BN>
__device__ __forceinline__ TileInfo decode_tile(int tile, const TilePlan& pl, const GemmArgs& a) {
  TileInfo ti;
  int t = tile;
  ti.p = 0;
  if (t >= pl.ntiles[0]) { t -= pl.ntiles[0]; ti.p = 1; }
  const GemmProblem& pr = a.p[ti.p];
  const int mt = t / pl.nn[ti.p], nt = t % pl.nn[ti.p];
  ti.row0 = mt * kBM;
  ti.n0 = nt * BN;
  ti.nk = pr.K / kBK;
  if (pr.routed) {
    int e = 0;
    while (e < a.E - 1 && ti.row0 >= pl.poff[e + 1]) ++e;
    ti.e = e;
    const int v = pl.poff[e] + pl.cnt[e] - ti.row0;
    ti.valid = v < kBM ? v : kBM;
    ti.brow = e * pr.N + ti.n0;
  } else {
    ti.e = 0;
    const int v = pr.M - ti.row0;
    ti.valid = v < kBM ? v : kBM;
    ti.brow = ti.n0;
  }
  return ti;
}

template <int BN, typename S>
__global__ void __launch_bounds__(kTcThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap tb0,
               const __grid_constant__ CUtensorMap ta1, const __grid_constant__ CUtensorMap tb1,
               GemmArgs a) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stage_base = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ TilePlan pl;

  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), 4 * 32);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
    // tile plan: padded expert segments from the unpadded offsets
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
    if ((long long)p > a.r_max) { bad = true; }
    for (int q = 0; q < 2; ++q) {
      if (q >= a.nprob) { pl.ntiles[q] = 0; pl.nn[q] = 1; continue; }
      const GemmProblem& pr = a.p[q];
      pl.nn[q] = pr.N / BN;
      const int mt = pr.routed ? (bad ? 0 : p / kBM) : (pr.M + kBM - 1) / kBM;
      pl.ntiles[q] = mt * pl.nn[q];
    }
    pl.total = pl.ntiles[0] + pl.ntiles[1];
    if (bad) set_status(a.status, DEV_BAD_INDEX, 300);
    prefetch_tmap(&ta0);
    prefetch_tmap(&tb0);
    prefetch_tmap(&ta1);
    prefetch_tmap(&tb1);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t idesc = idesc_f16kind_f32(kBM, BN, S::kFmt);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_last();
      // A tiles are reused by every column tile of their row block (consecutive tiles, run
      // side by side): keep them in L2 normally; evict-first sent them back to DRAM 3.5x
      const uint64_t pol_a = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < pl.total; tile += gridDim.x) {
        const TileInfo ti = decode_tile<BN>(tile, pl, a);
        const CUtensorMap* tA = ti.p ? &ta1 : &ta0;
        const CUtensorMap* tB = ti.p ? &tb1 : &tb0;
        const int ksplit = a.p[ti.p].ksplit;
        const int nrows = a.p[ti.p].N;
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.status, 301)) goto done;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, C::STAGE);
          uint8_t* sa = stage_base + stage * C::STAGE;
          // B of a K-split problem is a stack [K/ksplit][N][ksplit]: block kb lies in one slice
          const int bx = ksplit ? (kb * kBK) % ksplit : kb * kBK;
          const int by = ksplit ? ((kb * kBK) / ksplit) * nrows + ti.brow : ti.brow;
          tma_load_2d_hint(smem_u32(sa), tA, kb * kBK, ti.row0, fb, pol_a);
          tma_load_2d_hint(smem_u32(sa + C::A_BYTES), tB, bx, by, fb, pol_w);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < pl.total; tile += gridDim.x, ++local) {
        const TileInfo ti = decode_tile<BN>(tile, pl, a);
        const int acc = local & 1;
        const uint32_t accph = (local >> 1) & 1;
        if (!mbar_wait(smem_u32(&acc_empty[acc]), accph ^ 1u, abort_flag, a.status, 302)) goto mma_out;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.status, 303)) goto mma_out;
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * C::STAGE);
          const uint64_t adesc = smem_desc_sw128(sa);
          const uint64_t bdesc = smem_desc_sw128(sa + C::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_kindf16(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) ? 1u : 0u);
          issued_any = true;
          umma_commit(smem_u32(&empty[stage]));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        umma_commit(smem_u32(&acc_full[acc]));
      }
    mma_out:
      if (issued_any) {
        // let every issued MMA finish before TMEM is released
        umma_commit(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0, nullptr, a.status, 304);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;            // row inside the tile
    int local = 0;
    for (int tile = blockIdx.x; tile < pl.total; tile += gridDim.x, ++local) {
      const TileInfo ti = decode_tile<BN>(tile, pl, a);
      const GemmProblem& pr = a.p[ti.p];
      const int acc = local & 1;
      const uint32_t accph = (local >> 1) & 1;
      if (!mbar_wait(smem_u32(&acc_full[acc]), accph, abort_flag, a.status, 305)) break;
      tc_fence_after();
      const bool rv = r < ti.valid;
      const long long grow = (long long)ti.row0 + r;
      const float gate = (pr.gate != nullptr && rv) ? pr.gate[grow] : 1.0f;
      const uint16_t* bias =
          pr.bias ? reinterpret_cast<const uint16_t*>(pr.bias) + (long long)ti.e * pr.bias_stride : nullptr;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c * 32, v);
        tmem_ld_wait();
        const int col0 = ti.n0 + c * 32;
        float b[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) b[j] = 0.f;
        if (bias) {
          for (int br = 0; br < pr.bias_rows; ++br) {
            const uint4* bp = reinterpret_cast<const uint4*>(bias + (long long)br * pr.N + col0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float t8[8];
              S::x8_to_f32(__ldg(bp + u), t8);
#pragma unroll
              for (int j = 0; j < 8; ++j) b[8 * u + j] += t8[j];
            }
          }
        }
        if (rv) {
          // GEMM1: gelu(acc + b1); GEMM2: gate * (acc + b2); both rounded once to 16 bits
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(pr.out) + grow * pr.ld_out + col0);
          uint4 o[4];
          uint32_t* ow = reinterpret_cast<uint32_t*>(o);
          const int mode = pr.epi == 0 ? (a.act == 1 ? 1 : 0) : 2;
          if (mode == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              ow[j / 2] = S::pack2(gelu_act<true>(__uint_as_float(v[j]) + b[j], 0),
                                      gelu_act<true>(__uint_as_float(v[j + 1]) + b[j + 1], 0));
          } else if (mode == 1) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              ow[j / 2] = S::pack2(gelu_act<true>(__uint_as_float(v[j]) + b[j], 1),
                                      gelu_act<true>(__uint_as_float(v[j + 1]) + b[j + 1], 1));
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              ow[j / 2] = S::pack2((__uint_as_float(v[j]) + b[j]) * gate, (__uint_as_float(v[j + 1]) + b[j + 1]) * gate);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = o[u];
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[acc]));
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

int gemm_tc_pick_bn(int n0, int n1) {
  const int cands[4] = {256, 192, 128, 64};
  for (int i = 0; i < 4; ++i) {
    const int bn = cands[i];
    if (n0 % bn == 0 && (n1 == 0 || n1 % bn == 0)) return bn;
  }
  return 0;
}

template <int BN, typename S>
static cudaError_t launch_bn_t(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb, int grid,
                               cudaStream_t s) {
  using C = TcCfg<BN>;
  cudaError_t err = cudaFuncSetAttribute(gemm_tc_kernel<BN, S>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (err != cudaSuccess) return err;
  gemm_tc_kernel<BN, S><<<grid, kTcThreads, C::SMEM, s>>>(ta[0], tb[0], ta[1], tb[1], a);
  return cudaGetLastError();
}
template <int BN>
static cudaError_t launch_bn(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb, int grid,
                             cudaStream_t s) {
  return a.f16 ? launch_bn_t<BN, StoreF16>(a, ta, tb, grid, s) : launch_bn_t<BN, StoreBF16>(a, ta, tb, grid, s);
}

cudaError_t launch_gemm_tc(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb, int bn,
                           int num_sms, cudaStream_t s) {
  switch (bn) {
    case 256: return launch_bn<256>(a, ta, tb, num_sms, s);
    case 192: return launch_bn<192>(a, ta, tb, num_sms, s);
    case 128: return launch_bn<128>(a, ta, tb, num_sms, s);
    case 64: return launch_bn<64>(a, ta, tb, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
