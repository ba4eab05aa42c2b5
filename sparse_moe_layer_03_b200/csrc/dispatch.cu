// Dispatch: permute tokens into expert-contiguous blocks so that only the
// selected experts are computed ("Scaling Diffusion Transformers to 16 Billion
// Parameters", "MOE 回顾": with a sparse g, unused experts need not be run).
//
// Layout: expert i owns rows [P_i, P_i + counts_i), P_i = sum_{j<i}
// round_up(counts_j, 256), tokens ascending inside a segment.  Positions come
// from integer counts and prefix sums only (no order-dependent atomics), so
// the permutation is deterministic and equals the canonical one bit for bit.
//
//   count kernel  (one block per group of 256 tokens): the group's count per
//                 expert, and each slot's rank among the group's slots of the
//                 same expert (warp ballots), parked in `pos`.  No scan, no
//                 grid-wide step: it ends as soon as its counts are written.
//   gather kernel (launched as a programmatic dependent of the count kernel):
//                 every block first reads all group counts (4 KB at XL, one
//                 round of loads) and works out the segment starts and its
//                 own group's first row in every segment, redundantly.
//                 Blocks 0..E: block e < E marks the padding rows of segment
//                 e (row_token -1, gate 0, zero rows in x_perm: every row of a
//                 segment's 256-row tiles then holds finite values, which the
//                 weight gradients reduce over); block E marks the rows after
//                 the last segment; block 0 writes the offsets.  The other
//                 blocks take 64 tokens each: one thread per slot turns ranks
//                 into rows (group base + rank) and writes pos, row_token and
//                 row_gate; then each warp's lane 0 moves its tokens' rows by
//                 bulk copies through two shared-memory row buffers, storing
//                 each row once per selected expert (each warp's first row is
//                 requested before the wait, while the count kernel runs).
//   A last-block scan inside the count kernel (fence, counter, two rounds of
//   loads) took half of its 8.6 us, measured with a timer probe.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDispatchThreads = 256;
constexpr int kGroup = kDispatchThreads;      // tokens per group: one count block, one token per thread

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// The segment plan from the group counts cnt[e * ngroups + g], computed by every gather block:
// total_s[e] = expert e's rows, before_s[e] = its rows in groups before g0, poff_s[e] = the first
// row of segment e (poff_s[E] = rows of all segments).  Warp w takes experts w, w + 8, ...; its
// lanes read 32 consecutive groups per load (coalesced), eight loads in flight.  Every thread
// of the block calls it.
__device__ void segment_plan(const DispatchArgs& a, int g0, int* total_s, int* before_s, long long* poff_s) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, NW = kDispatchThreads / 32;
  const int E = a.E, ng = a.ngroups;
  for (int e = w; e < E; e += NW) {
    const int32_t* row = a.group_base + (size_t)e * ng;
    int tot = 0, bef = 0;
    for (int c0 = 0; c0 < ng; c0 += 8 * 32) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int g = c0 + u * 32 + lane;
        v[u] = g < ng ? __ldcg(row + g) : 0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int g = c0 + u * 32 + lane;
        tot += v[u];
        bef += g < g0 ? v[u] : 0;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
      bef += __shfl_xor_sync(0xffffffffu, bef, o);
    }
    if (lane == 0) { total_s[e] = tot; before_s[e] = bef; }
  }
  __syncthreads();
  if (tid == 0) {
    long long p = 0;
    for (int e = 0; e < E; ++e) {
      poff_s[e] = p;
      p += (total_s[e] + kSegAlign - 1) / kSegAlign * kSegAlign;
    }
    poff_s[E] = p;
  }
  __syncthreads();
}

// One group of kGroup tokens per block, one token per thread: the group's count
// per expert, and each slot's rank among the group's slots of the same expert
// (rank inside the warp from a ballot, plus the counts of the earlier warps).
template <int EMAX>
__global__ void __launch_bounds__(kDispatchThreads) dispatch_count_kernel(DispatchArgs a) {
  constexpr int NW = kDispatchThreads / 32;
  __shared__ uint32_t bal[NW][EMAX];
  __shared__ int wbase[NW][EMAX];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = blockIdx.x;
  const int Kmax = a.Kmax, E = a.E;
  grid_dependency_wait();                               // the router's selection
  launch_dependents();                                  // the gather kernel may start loading x rows
  const int t = g * kGroup + tid;
  const bool valid = t < a.T;
  const int ns = valid ? (a.n_sel ? a.n_sel[t] : a.K) : 0;
  int ek[EMAX];
  uint32_t m = 0;
#pragma unroll
  for (int k = 0; k < EMAX; ++k) {
    int e = -1;
    if (k < Kmax && k < ns) {
      e = a.topk_idx[(size_t)t * Kmax + k];
      if (e >= E) { set_status(a.status, DEV_BAD_INDEX, 200); e = -1; }
      else if (e >= 0 && ((m >> e) & 1u)) { set_status(a.status, DEV_BAD_INDEX, 202); e = -1; }   // repeated expert
      if (e >= 0) m |= 1u << e;
    }
    ek[k] = e < 0 ? -1 : e;
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
      const uint32_t b = __ballot_sync(0xffffffffu, (m >> e) & 1u);
      if (lane == 0) bal[w][e] = b;
    }
  }
  __syncthreads();
  if (tid < E) {
    int run = 0;
#pragma unroll
    for (int v = 0; v < NW; ++v) {
      wbase[v][tid] = run;
      run += __popc(bal[v][tid]);
    }
    a.group_base[(size_t)tid * a.ngroups + g] = run;     // the group's count of expert tid
  }
  __syncthreads();
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int k = 0; k < EMAX; ++k)
    if (k < Kmax && valid)
      a.pos[(size_t)t * Kmax + k] = ek[k] >= 0 ? wbase[w][ek[k]] + __popc(bal[w][ek[k]] & lt) : -1;
}

// untiled bulk copy from this CTA's shared memory to global memory, completing in a bulk group
// (both addresses 16-byte aligned, the size a multiple of 16)
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}

// One row copy: P x 32 lanes x 16 bytes covers up to P*32 vectors of the row.
template <int P>
__device__ __forceinline__ void load_row(const uint4* src, int nvec, int lane, uint4* buf) {
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int v = u * 32 + lane;
    if (v < nvec) buf[u] = src[v];
  }
}
template <int P>
__device__ __forceinline__ void store_row(uint4* dst, int nvec, int lane, const uint4* buf) {
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int v = u * 32 + lane;
    if (v < nvec) dst[v] = buf[u];
  }
}

// Gather block: tokens [t0, t0 + tpb), all in group g0 = t0 / 256.  Phase 1, one thread per slot,
// all slots of the block at once: row = segment start + the expert's rows in earlier groups +
// rank inside the group; writes pos, row_token, row_gate and keeps the row in shared memory.
// Phase 2 copies the rows, token l of the block by warp l mod 8, once per selected slot:
//   P = -1 (when the row buffers fit): bulk copies (TMA); lane 0 of each warp loads a row into one
//          of the warp's two shared-memory row buffers and stores it from there, the warp's next
//          row loading while the current one is stored;
//   P > 0: 16-byte vectors through registers (P per lane; P = 0: wide rows in pieces).
// Each warp's first row is requested before the kernel waits for the count kernel (programmatic
// dependent launch), so it loads while the counts are worked out.
template <typename T, int P>
__device__ __forceinline__ void gather_block(const DispatchArgs& a, int* spos, int blk) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  __shared__ uint64_t rbar[kDispatchThreads / 32][2];
  const uint32_t row_bytes = (uint32_t)a.D * (uint32_t)sizeof(T);
  uint8_t* rbuf = reinterpret_cast<uint8_t*>(spos) + ((a.tpb * a.Kmax * 4 + 127) & ~127) + (size_t)w * 2 * row_bytes;
  const int Kmax = a.Kmax;
  const int nvec = a.D * (int)sizeof(T) / 16;
  const int t0 = blk * a.tpb;
  const int nt = min(a.tpb, a.T - t0);
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  uint4* xp = reinterpret_cast<uint4*>(a.x_perm);
  constexpr int NW = kDispatchThreads / 32;
  uint4 buf[P > 0 ? P : 1];
  const bool copy = a.x_perm != nullptr;               // else positions only
  // each warp's first row loads before the wait (x only: it overlaps the count kernel)
  if (P > 0 && copy && w < nt) load_row<P>(xv + (size_t)(t0 + w) * nvec, nvec, lane, buf);
  if (P < 0 && copy && lane == 0) {
    mbar_init(smem_u32(&rbar[w][0]), 1);
    mbar_init(smem_u32(&rbar[w][1]), 1);
    fence_barrier_init();
    if (w < nt) {
      mbar_arrive_expect_tx(smem_u32(&rbar[w][0]), row_bytes);
      bulk_load(smem_u32(rbuf), xv + (size_t)(t0 + w) * nvec, row_bytes, smem_u32(&rbar[w][0]));
    }
  }
  grid_dependency_wait();                              // the count kernel's counts and ranks from here on
  __shared__ int total_s[32], before_s[32];
  __shared__ long long poff_s[33];
  segment_plan(a, t0 / kGroup, total_s, before_s, poff_s);

  for (int i = tid; i < nt * Kmax; i += kDispatchThreads) {
    const int t = t0 + i / Kmax, k = i % Kmax;
    const size_t slot = (size_t)t0 * Kmax + i;
    const int ns = a.n_sel ? a.n_sel[t] : a.K;
    int p = -1;
    if (k < ns) {
      const int e = a.topk_idx[slot];
      const int r = a.pos[slot];
      if (e >= 0 && e < a.E && r >= 0) {
        const long long q = poff_s[e] + before_s[e] + r;
        p = (int)q;
        if (q < 0 || q >= a.r_max) { set_status(a.status, DEV_BAD_INDEX, 201); p = -1; }
        else {
          a.row_token[p] = t;
          a.row_gate[p] = a.topk_w[slot];
        }
      }
    }
    a.pos[slot] = p;
    spos[i] = p;
  }
  if (!copy) return;
  __syncthreads();

  if (P < 0) {
    if (lane == 0) {
      int it = 0;
      for (int l = w; l < nt; l += NW, ++it) {
        const int b = it & 1;
        if (l + NW < nt) {
          bulk_wait_read_all();                      // the stores out of the other buffer have read it
          mbar_arrive_expect_tx(smem_u32(&rbar[w][b ^ 1]), row_bytes);
          bulk_load(smem_u32(rbuf + (b ^ 1) * row_bytes), xv + (size_t)(t0 + l + NW) * nvec, row_bytes,
                    smem_u32(&rbar[w][b ^ 1]));
        }
        if (!mbar_wait(smem_u32(&rbar[w][b]), (uint32_t)(it >> 1) & 1u, nullptr, a.status, 204)) break;
        for (int k = 0; k < Kmax; ++k) {
          const int p = spos[l * Kmax + k];
          if (p >= 0) bulk_store(xp + (size_t)p * nvec, smem_u32(rbuf + b * row_bytes), row_bytes);
        }
        bulk_commit();
      }
      bulk_wait_all();                               // every row stored before the block ends
    }
    return;
  }

  for (int l = w; l < nt; l += NW) {
    const uint4* src = xv + (size_t)(t0 + l) * nvec;
    if (P > 0) {
      if (l != w) load_row<P>(src, nvec, lane, buf);
      for (int k = 0; k < Kmax; ++k) {
        const int p = spos[l * Kmax + k];
        if (p >= 0) store_row<P>(xp + (size_t)p * nvec, nvec, lane, buf);
      }
    } else {
      for (int v0 = 0; v0 < nvec; v0 += 8 * 32) {      // wide rows: pieces of 8 vectors per lane
        uint4 piece[8];
        load_row<8>(src + v0, nvec - v0, lane, piece);
        for (int k = 0; k < Kmax; ++k) {
          const int p = spos[l * Kmax + k];
          if (p >= 0) store_row<8>(xp + (size_t)p * nvec + v0, nvec - v0, lane, piece);
        }
      }
    }
  }
}

// Segment block e <= E: the rows of no token.  e < E: segment e's padding rows [P_e + count_e,
// P_{e+1}) get row_token -1, gate 0 and (with x_perm) zero rows; e = E: the rows after the last
// segment, [P_E, r_max), get row_token -1 and gate 0.  Block 0 also writes the offsets.
template <typename T>
__device__ void segment_block(const DispatchArgs& a, int e) {
  __shared__ int total_s[32], before_s[32];
  __shared__ long long poff_s[33];
  segment_plan(a, 0, total_s, before_s, poff_s);
  const int tid = threadIdx.x;
  const int E = a.E;
  if (e == 0 && tid == 0) {
    int u = 0;
    for (int j = 0; j < E; ++j) {
      a.offsets[j] = u;
      u += total_s[j];
    }
    a.offsets[E] = u;
  }
  const long long lo = e < E ? poff_s[e] + total_s[e] : poff_s[E];
  const long long hi = e < E ? poff_s[e + 1] : a.r_max;
  if (lo < 0 || hi > a.r_max) {
    if (tid == 0) set_status(a.status, DEV_BAD_INDEX, 203);
    return;
  }
  for (long long r = lo + tid; r < hi; r += kDispatchThreads) {
    a.row_token[r] = -1;
    a.row_gate[r] = 0.f;
  }
  if (e < E && a.x_perm != nullptr) {
    const int nvec = a.D * (int)sizeof(T) / 16;
    uint4* xp = reinterpret_cast<uint4*>(a.x_perm);
    const long long n = (hi - lo) * nvec;
    for (long long i = tid; i < n; i += kDispatchThreads) xp[lo * nvec + i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

template <typename T>
__global__ void __launch_bounds__(kDispatchThreads) dispatch_gather_kernel(DispatchArgs a, int seg_blocks, int bulk) {
  extern __shared__ int spos[];                       // [tpb * Kmax] rows of the block's slots
  if ((int)blockIdx.x < seg_blocks) {
    grid_dependency_wait();
    segment_block<T>(a, blockIdx.x);
    return;
  }
  const int blk = blockIdx.x - seg_blocks;
  const int nvec = a.D * (int)sizeof(T) / 16;
  if (bulk) gather_block<T, -1>(a, spos, blk);
  else if (nvec <= 4 * 32) gather_block<T, 4>(a, spos, blk);
  else if (nvec <= 8 * 32) gather_block<T, 8>(a, spos, blk);
  else gather_block<T, 0>(a, spos, blk);
}

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s) {
  // both kernels launch as programmatic dependents of the kernel before them (they wait for it
  // inside, before reading what it wrote), so their launches overlap its tail
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cc = {};
  cc.gridDim = dim3(a.ngroups, 1, 1);
  cc.blockDim = dim3(kDispatchThreads, 1, 1);
  cc.stream = s;
  cc.attrs = attr;
  cc.numAttrs = 1;
  cudaError_t err = a.E <= 8 ? cudaLaunchKernelEx(&cc, dispatch_count_kernel<8>, a)
                    : a.E <= 16 ? cudaLaunchKernelEx(&cc, dispatch_count_kernel<16>, a)
                                : cudaLaunchKernelEx(&cc, dispatch_count_kernel<32>, a);
  if (err != cudaSuccess) return err;
  if (a.tpb <= 0 || kGroup % a.tpb) return cudaErrorInvalidValue;   // a gather block stays inside one group
  const int seg_blocks = a.E + 1;
  const int ggrid = seg_blocks + (a.T + a.tpb - 1) / a.tpb;
  // bulk row copies when the warps' row buffers fit (two rows per warp after the slots' rows)
  const size_t row_bytes = (size_t)a.D * (a.b16 ? 2 : 4);
  const size_t smem_bulk = (((size_t)a.tpb * a.Kmax * sizeof(int) + 127) & ~(size_t)127) +
                           (size_t)(kDispatchThreads / 32) * 2 * row_bytes;
  const int bulk = a.x_perm != nullptr && smem_bulk <= 160 * 1024 ? 1 : 0;
  const size_t smem = bulk ? smem_bulk : (size_t)a.tpb * a.Kmax * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e2 = a.b16 ? cudaFuncSetAttribute(dispatch_gather_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                           : cudaFuncSetAttribute(dispatch_gather_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
  }
  // the gather's first row loads (x only) overlap the count kernel; everything the count kernel
  // writes is read after the wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ggrid, 1, 1);
  cfg.blockDim = dim3(kDispatchThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.b16) return cudaLaunchKernelEx(&cfg, dispatch_gather_kernel<uint16_t>, a, seg_blocks, bulk);
  return cudaLaunchKernelEx(&cfg, dispatch_gather_kernel<float>, a, seg_blocks, bulk);
}

}  // namespace moe
