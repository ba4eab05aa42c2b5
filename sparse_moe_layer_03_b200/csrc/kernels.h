// Internal launchers shared between the kernel files and the C-ABI layer.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// message returned by moe_last_error() on this thread
void set_last_error_message(const char* msg);

// every expert segment of the permuted buffers starts on a multiple of this many rows
constexpr int kSegAlign = 256;

// CTA-pair GEMM: epilogue warps per TMEM lane quadrant (each takes every kPairEpiSplit-th column
// box of a tile); the GELU-backward row dots come per column tile and warp: kPairEpiSplit slots.
// Two per quadrant measured no faster on GEMM1 and 5% slower on GEMM2 + combine at XL.
constexpr int kPairEpiSplit = 1;

// per-device values cached by the launchers (devices 0 .. kMaxDevicesCached-1)
constexpr int kMaxDevicesCached = 64;

// CTAs of a CTA-pair GEMM launch: one pair per two SMs, at most `fit` pairs (what the device
// holds at once) and at most `max_pairs` (0 = no limit of the caller's)
inline int pair_grid(int num_sms, int fit, int max_pairs) {
  int pairs = num_sms / 2;
  if (fit < pairs) pairs = fit;
  if (max_pairs > 0 && max_pairs < pairs) pairs = max_pairs;
  return pairs > 0 ? 2 * pairs : 0;
}

// ---- route.cu
struct RouteArgs {
  const void* x;            // [T,D] act
  const void* wg;           // [E,D] act
  const float* bias;        // [E] or null
  int T, D, E, K;
  int b16, f16;             // 16-bit storage (bf16 or fp16); fp16
  int tile_rows, ntiles, grid;
  int tmap3d;               // 16-bit router: 1 = one 3-D box {64, 16 rows, blocks} per part, 0 = 2-D boxes
  int32_t* topk_idx;        // top-K mode: [T,K]
  float* topk_w;
  int32_t* n_sel;           // may be null (top-K)
  float* P;                 // [T,E] scores (scratch) for Expert-Race or per-image losses, else null
  int race;                 // 1: P only, the selection happens later
  int32_t* tile_counts;     // [ntiles,E] (top-K)
  float* tile_psum;         // [ntiles,E]
  uint32_t* zero;           // block 0 clears zero[0, nzero) first (the Expert-Race scratch), or null
  int nzero;
  // adaLN modulation (16-bit router only): the router routes on
  // m = gamma[t / img_len] * LayerNorm(x_t) + beta[t / img_len] and stores m through tmap_m
  const void* gamma;        // [T/img_len, D] act, or null (route on x itself)
  const void* beta;
  int img_len;
  float eps;
  int* status;
};
size_t route_smem_bytes(int D, int E, int tile_rows, int b16);
size_t route_smem_total(int D, int E, int tile_rows, int b16, int modulate);
int route_mma_stages(int D, int E, int modulate);
int route_box_blocks(int D, int E, int modulate);   // 16-bit router: 64-column blocks per TMA box
void route_plan(int T, int D, int E, int b16, int modulate, int sms, int* tile_rows, int* threads);

// partial counts / score sums -> counts[E] and the balance loss
struct FinalizeArgs {
  const int32_t* tile_counts; int ntiles_counts;
  const float* tile_psum; int ntiles_psum;
  int T, E, K; float alpha;
  int32_t* counts; float* aux_loss;   // counts == null: the router leaves finalizing to a later kernel
  double* score_sum;                  // [E] sum_t P[t,i] of the call (fp64) out, or null
  unsigned int* ctr;                  // blocks-done counter in ws (zero between calls)
};
cudaError_t launch_route(const RouteArgs& a, const FinalizeArgs& fin, const CUtensorMap* tmap_x,
                         const CUtensorMap* tmap_m, cudaStream_t s);

// balance-loss statistics of a call ([counts, score sums], fp64) and the loss from
// statistics summed over several calls or ranks
cudaError_t launch_balance_stats(const int32_t* counts, const double* score_sum, int E, double* stats, cudaStream_t s);
cudaError_t launch_balance_loss_from_stats(const double* stats, int E, int K, long long T_total, float alpha,
                                           float* aux_loss, cudaStream_t s);

// per-image balance loss (seq_len > 0): overwrites aux_loss with the mean over images
struct SeqLossArgs {
  const float* P;               // [T,E] scores
  const int32_t* topk_idx;      // [T,Kmax]
  const int32_t* n_sel;         // [T] or null
  int T, E, K, Kmax, L;
  float alpha;
  double* seq_loss;             // [T/L] scratch
  unsigned int* ctr;            // blocks-done counter in ws (zero between calls)
  float* aux_loss;
};
cudaError_t launch_seq_loss(const SeqLossArgs& a, cudaStream_t s);

// ---- backward.cu: the balance loss's gradient through the router
struct BalanceGradArgs {
  const void* x; const void* wg; const float* bias;   // x [T,D], wg [E,D] act; bias [E] or null
  const int32_t* counts;                              // [E] from the forward selection
  int T, D, E, K;
  int dtype;                                          // moe_dtype_t of x and wg (and dx)
  float alpha, scale;                                 // scale = dObjective / dL_balance
  void* dx;                                           // [T,D] act or null
  float* dwg;                                         // [E,D]
  float* dbias;                                       // [E] or null
  // the gates' gradient (router backward of the whole layer), or null for the balance loss alone:
  // dJ/dP[t, topk_idx[t,k]] += dgate[t,k] for the token's selected slots
  const float* dgate; const int32_t* topk_idx; const int32_t* n_sel; int Kmax;
  int dx_accumulate;                                  // 1: dx += dl Wg (dx holds the experts' part)
  int pass_grid, pass_tpc;                             // > 0: the one-pass kernel, CTAs and tokens per CTA
  int mma_grid;                                       // > 0: the bf16 mma.sync kernel on this many CTAs
  const CUtensorMap* tmap_x;                          // its x map (3-D half-row boxes of 16 rows)
  float* dl;                                          // [T,E] scratch: dL/dlogits
  float* db_part;                                     // [blocks,E] scratch
  float* partials;                                    // [chunks,E,D] scratch
};
constexpr int kBwdMaxBlocks = 1024;
int balance_grad_chunks(int T);
// the one-pass router backward: whether a row and the CTA's scratch fit, and its grid
bool router_bwd_pass_fits(int D, int E, int dtype, int T, int sms);
// the bf16 router backward on mma.sync: whether it applies, and its shared memory
bool router_bwd_mma_fits(int D, int E, int dtype);
size_t router_bwd_mma_smem(int D);
int router_bwd_pass_grid(int T, int sms, int* tpc);
cudaError_t launch_balance_grad(const BalanceGradArgs& a, int blocks, cudaStream_t s);

// ---- stats.cu: expert-selection frequency per label
struct FreqArgs {
  const int32_t* topk_idx; const int32_t* n_sel;
  int T, E, K, Kmax, L;
  const int32_t* labels;        // [T/L] or null (label = t mod L)
  int n_labels;
  int32_t* hist;                // [n_labels,E]
  int* status;
};
cudaError_t launch_frequency(const FreqArgs& a, cudaStream_t s);

// Expert-Race selection: one cooperative launch of `grid` CTAs (at most one per
// SM), CTA r owning tokens [r*tpc, (r+1)*tpc)
constexpr int kRaceMaxCtas = 256;
constexpr int kRaceSyncWords = 4096 + 4096 + 256 + 16;   // digit histograms 1..3, grid-barrier counter
struct RaceArgs {
  const float* P;           // [T,E] scores
  int T, E, K;
  uint32_t* sync;           // [kRaceSyncWords], zero on entry (the router clears it)
  uint32_t* loc;            // [grid,256] per-CTA histograms of the last digit
  int grid, tpc;            // CTAs; tokens per CTA (a multiple of 4)
  int32_t* topk_idx;        // [T,E]
  float* topk_w;            // [T,E]
  int32_t* n_sel;           // [T]
  int32_t* tile_counts;     // [grid,E]
  int* status;
  const uint32_t* test;     // two host-written test words (flags, wait limit in us) or null
};
// CTAs for T tokens on `sms` SMs; *tpc = tokens per CTA
int race_plan(int T, int sms, int* tpc);
// selection, per-CTA counts, then the last CTA turns counts and score sums into counts[E] and the loss
cudaError_t launch_race_select(const RaceArgs& a, const FinalizeArgs& fin, cudaStream_t s);

// ---- dispatch.cu
struct DispatchArgs {
  const void* x; int b16;   // 16-bit storage (rows are copied as bytes)
  const int32_t* topk_idx; const float* topk_w; const int32_t* n_sel;
  int T, D, E, K, Kmax;
  int ngroups;              // ceil(T/256): groups of 256 tokens
  int tpb;                  // tokens per gather block
  long long r_max;
  int32_t* group_base;      // [E,ngroups] scratch: counts, then each group's first row in every segment
  int32_t* offsets;         // [E+1]
  int32_t* pos; int32_t* row_token; float* row_gate;
  void* x_perm;             // null: positions only (GEMM1 gathers the rows itself)
  int* status;
};
cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s);

// ---- gemm (tcgen05 and FFMA)
struct GemmProblem {
  int routed;               // 1: rows grouped by expert segments (offsets), 0: dense rows
  int M;                    // dense: rows; routed: unused (from offsets); kgrouped: rows of each output
  int N, K;                 // per-expert output width and reduction length (kgrouped: K from offsets)
  int epi;                  // 0: bias + GELU -> act store; 1: (bias) * gate -> act store;
                            // 2 (dense rows, CTA-pair kernel only): out = sum_k y_routed[pos[t,k]] + (acc + bias);
                            // 4 (CTA-pair kernel only): out = gate * acc * gelu'(u) with u read from `aux`
                            //   (same layout as out, may alias it), and dg[row, column tile] = sum acc * gelu(u)
  // CTA-pair kernel only: operands held MN-major in memory ([K rows, M or N columns] row-major, as
  // the weights of a backward GEMM or the activations of a weight gradient are), and the weight
  // gradient's grouping: one [M, N] output per expert whose reduction runs over that expert's rows
  // of the permuted buffers (segments from offsets, padded to 256; padding rows must be zero)
  int a_mn, b_mn;
  int kgrouped;
  int b_split;              // MN-major B whose N runs over b_split-wide blocks stacked along K (the n_s
                            // shared W2 [n_s, D, H] seen as [n_s*D, H]): block n / b_split sits K rows lower
  int out_f32;              // fp32 output through a 3-D map [z, M, N]: z = expert (kgrouped), n / out_split, or 0
  int out_split;
  const void* aux;          // epi 4: u [rows, N] act
  float* dg;                // epi 4: [rows, dg_stride] row dots per column tile and epilogue warp, or null
  int dg_stride;
  const void* A;            // [rows,K] act (FFMA path; the TMA path uses tensor maps)
  const void* B;            // [E*N or N, K] act
  void* out; long long ld_out;
  const void* bias; long long bias_stride;   // per-expert stride in elements, null = none
  int bias_rows;            // bias rows summed per column (n_s for the shared GEMM2, else 1)
  int ksplit;               // 0, or: B is [K/ksplit blocks][N][ksplit] (shared W2 stack)
  const float* gate;        // per-row gate or null
  // routed problem on the CTA-pair kernel: A row r is row gather_rows[r] of the A tensor (rows
  // < 0 read row 0), copied into the swizzled A stage by the kernel's cp.async gather warps
  const int32_t* gather_rows;
  int gather_nrows;         // rows of the A tensor
};
struct GemmArgs {
  GemmProblem p[2]; int nprob;
  const int32_t* offsets; int E;
  long long r_max;
  int act;
  int* status;
  int b16, f16;             // 16-bit storage (bf16 or fp16); fp16
  // combine folded into the shared-expert epilogue (epi 2 on problem 1): the routed
  // tiles of the same launch write y_routed; each epilogue warp counts its finished
  // routed tiles in done_ctr, and the shared tiles wait for all of them
  unsigned int* sched_ctr;  // CTA-pair kernel: tile claim counter, zero on entry; the last CTA resets it
  unsigned int* exit_ctr;   // CTAs that finished (the last one resets the counters)
  const uint32_t* test;     // two host-written test words (flags, wait limit in us) or null
  const int32_t* pos;       // [T,kmax] rows of y_routed per token slot (-1 unused)
  const int32_t* n_sel;     // [T] or null (then kdef slots per token)
  int kmax, kdef;
  const void* y_routed;     // [r_max, N] act
  unsigned int* done_ctr;   // zero on entry; the launch's last CTA resets it
  const void* x_res;        // adaLN-Zero residual in the epi-2 output: x_res + alpha[t / img_len] * sum, or null
  const void* alpha;
  int img_len;
  int b_half;               // CTA-pair kernel (set by its launcher): tiles at most BN/2 wide load their B rows
                            // through the half-height boxes of the tbn maps
};
cudaError_t launch_gemm_tc(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb, int bn,
                           int num_sms, cudaStream_t s);
int gemm_tc_pick_bn(int n0, int n1);
// tbn: the two problems' B maps with boxes of bn/4 rows (half of a CTA's usual B box), used by the
// tiles at most bn/2 wide so that they do not load rows they never read; null: every tile uses tb
cudaError_t launch_gemm_pair(const GemmArgs& a, const CUtensorMap* ta, const CUtensorMap* tb, const CUtensorMap* to,
                             const CUtensorMap* tbn, int bn, int num_sms, int max_pairs, cudaStream_t s);
int gemm_pair_pick_bn(int n0, int n1);
cudaError_t launch_gemm_simt(const GemmArgs& a, cudaStream_t s);

// ---- expert_backward.cu: memory-bound parts of the expert MLPs' backward
struct ExpertBwdArgs {
  const void* dout;          // [T,D] act: dJ/dMoE(x)
  const int32_t* row_token;  // [rows] from moe_dispatch (-1 on padding rows)
  const float* row_gate;     // [rows]
  long long rows;            // R_max
  int T, D, E, K, Kmax, f16;
  void* dout_perm;           // [rows,D] act out: dY in permuted order
  void* dz_perm;             // [rows,D] act out: g * dY in permuted order
  // dgate
  const int32_t* pos; const int32_t* topk_idx; const int32_t* n_sel;
  const float* dg; int dg_stride;   // [rows, dg_stride] row dots per column tile of the GELU-backward GEMM
  const void* b2;            // [E,D] act or null
  float* dgate;              // [T,Kmax] out
};
cudaError_t launch_bwd_gather(const ExpertBwdArgs& a, cudaStream_t s);
cudaError_t launch_dgate(const ExpertBwdArgs& a, cudaStream_t s);
// column sums of X [nrows, C] (16-bit) per expert segment (offsets) or over all rows (offsets null),
// each written nrep times: out [nseg * nrep, C] fp32; partial: [colsum_chunks(nrows), C] fp32 scratch
int colsum_chunks(long long nrows);
cudaError_t launch_colsum(const void* X, long long nrows, int C, const int32_t* offsets, int E, int nrep,
                          float* partial, float* out, int f16, cudaStream_t s);

// ---- combine.cu
struct CombineArgs {
  const void* y_perm; const void* y_sh; const int32_t* pos; const int32_t* n_sel;   // act dtype
  void* out; int b16, f16;
  int T, D, K, Kmax;
  long long r_max;
  const void* x_res;        // adaLN-Zero residual: out = x_res + alpha[t / img_len] * MoE, or null
  const void* alpha;
  int img_len;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

}  // namespace moe
