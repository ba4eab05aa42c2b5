/*
 * moe.h -- C ABI of the B200 (sm_100a) DiT-MoE sparse expert layer: the
 * forward, the balance loss's statistics over ranks and its gradient.
 *
 * The layer (for every image-patch token x_t, width D):
 *   logits  l[t,i] = x_t . Wg[i] (+ b_i)                 i = 0..E-1
 *   scores  P[t,i] = softmax_i(l[t,:])
 *   select  top-K experts per token (or Expert-Race: the S = K*T largest P
 *           over the whole T x E matrix), gate g[t,i] = P[t,i] on the selection
 *   output  MoE(x_t) = sum_{i in sel_t} g[t,i] e_i(x_t) + sum_{j<n_s} s_j(x_t)
 *           e_i(x) = W2_i gelu_tanh(W1_i x + b1_i) + b2_i   (same form for s_j)
 *   loss    L = alpha * sum_i (E/(K T)) counts_i * (1/T) sum_t P[t,i]
 *
 * Sources (page title, section):
 *   "Scaling Diffusion Transformers to 16 Billion Parameters" (reading note):
 *     "MOE 回顾" eq. MoE(x); "MOE-DIT" eq. MLP, shared-expert routing,
 *     expert-level balance loss eq. L_balance.
 *   "DiT-MoE" hub page, section 1 "MoE Gate 路由机制": MoEGate (weight
 *     (n_routed_experts, gating_dim), softmax scoring, top_k, aux_loss_alpha).
 *   "Scalable Diffusion Models with Transformers (DiT)", "DiT block 实现细节":
 *     tanh-approximate GELU in the core transformer.
 *   "Expert Race: A Flexible Routing Strategy for Scaling Diffusion
 *     Transformer with Mixture of Experts", abstract: tokens and experts
 *     compete together and the top candidates win.
 *
 * Conventions for every entry point:
 *   - Every pointer argument named as a tensor is DEVICE memory owned by the
 *     caller; the library never allocates, frees or keeps it.  Tensors are
 *     row-major and contiguous; every tensor pointer must be 16-byte aligned.
 *   - "act" tensors (x, x_perm, h_perm, h_sh, y_perm, y_sh, out) and
 *     weights/biases have the storage type cfg->dtype (fp32, bf16 or fp16);
 *     scores, gates and gradients are fp32; indices are int32.  Every sum runs
 *     in fp32 (fp64 where the balance loss is finalised).
 *   - Weights follow nn.Linear (out x in): W1 [E,H,D], b1 [E,H], W2 [E,D,H],
 *     b2 [E,D].  The n_s shared experts come stacked the same way: W1s
 *     [n_s,H,D], b1s [n_s,H], W2s [n_s,D,H], b2s [n_s,D].  The kernels treat
 *     W1s as one [n_s*H, D] layer and sum_j W2_j h_j + sum_j b2_j as one
 *     K = n_s*H contraction, which is sum_j s_j(x) exactly.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream), never synchronise and never read device data on the
 *     host.  Group sizes stay on the device.
 *   - `ws` is caller-owned device scratch of at least moe_workspace_size(cfg)
 *     bytes, 256-byte aligned.  Its first 256 bytes hold a status word that
 *     kernels set on a device-detected error (bad index, a bounded wait that
 *     ran out) and the blocks-done counters kernels use between launches;
 *     moe_workspace_init() clears them and moe_check_status() reads the status.
 *     A workspace must not be shared by calls that may overlap on the GPU.
 *   - Return value: MOE_OK, or a negative moe_status_t with a message
 *     available from moe_last_error() (thread-local).  Argument errors are
 *     detected on the host before anything is launched.
 *   - T = 0 is valid: outputs are empty, counts are zeroed and aux_loss = 0.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,  /* null / misaligned pointer, bad size, K > E ... */
  MOE_ERR_UNSUPPORTED = -2,  /* valid but not built: D or H not a multiple of 64, E > 32 ... */
  MOE_ERR_WORKSPACE = -3,    /* ws_bytes < moe_workspace_size(cfg) */
  MOE_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_CHECK = -5, /* a kernel found a bad index (status word) */
  MOE_ERR_TIMEOUT = -6       /* a kernel's bounded wait ran out (status word) */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_F16 = 2 } moe_dtype_t;
typedef enum { MOE_ROUTE_TOPK = 0, MOE_ROUTE_RACE = 1 } moe_routing_t;
typedef enum {
  MOE_GEMM_AUTO = 0, /* bf16 / fp16: tcgen05 on CTA pairs (256-row tiles); fp32: FFMA */
  MOE_GEMM_SIMT = 1, /* FFMA for every dtype (a second implementation, for checks) */
  MOE_GEMM_TC1 = 2   /* bf16 / fp16: tcgen05 on single CTAs (128-row tiles) */
} moe_gemm_impl_t;

typedef struct {
  int32_t T;         /* tokens in this call (batch x patch tokens), >= 0 */
  int32_t D;         /* model width (MoEGate gating_dim), multiple of 64 */
  int32_t H;         /* expert hidden width, multiple of 64 */
  int32_t E;         /* routed experts (n_routed_experts), 1..32 */
  int32_t K;         /* experts per token (top_k); race: S = K*T winners, 1..E */
  int32_t n_shared;  /* shared experts n_s, 0..8 */
  int32_t dtype;     /* moe_dtype_t: storage type of activations and weights */
  int32_t routing;   /* moe_routing_t */
  float alpha;       /* balance-loss factor (aux_loss_alpha) */
  int32_t act;       /* 0 = gelu tanh form (DiT core), 1 = exact erf form */
  int32_t gemm_impl; /* moe_gemm_impl_t */
  int32_t seq_len;   /* tokens per image for the balance loss: 0 = the whole call is one
                        sequence; L > 0 (L divides T) = mean over the T/L images of the loss
                        taken over each image's tokens ("MOE-DIT": T in L_balance is the
                        length of the image-patch sequence) */
  int32_t gemm_pairs; /* CTA pairs (two SMs each) the tensor-core expert GEMMs may occupy at
                         once: 0 = as many as the device holds; a smaller value leaves SMs free
                         for work on other streams.  The result does not depend on it. */
} moe_config_t;

/* The adaLN-Zero residual connection around the layer, applied where the
 * combine writes `out` ("Scalable Diffusion Models with Transformers (DiT)",
 * DiT block details: a per-sample, per-dimension gate alpha scales each branch
 * before its residual connection):
 *     out[t] = x_res[t] + alpha[t / img_len] * MoE(x)[t]   (fp32, rounded once) */
typedef struct {
  const void* x_res;   /* [T,D] act: the residual stream entering the block */
  const void* alpha;   /* [T/img_len, D] act: the gate of each image */
  int32_t img_len;     /* tokens per image, >= 1, dividing T */
} moe_residual_t;

/* adaLN modulation of the layer input, applied inside moe_route
 * ("Diffusion Transformer (DiT) 技术全景解析" 2.2.3, AdaLN: a plain layer_norm
 * over the features, then a per-sample scale gamma and shift beta):
 *     m[t] = gamma[t / img_len] * (x[t] - mean) / sqrt(var + eps) + beta[t / img_len]
 * The router routes on m and writes it to x_mod, rounded to the act type;
 * moe_dispatch and the shared experts' GEMM1 then take x_mod as their x.
 * 16-bit types only. */
typedef struct {
  const void* gamma;   /* [T/img_len, D] act */
  const void* beta;    /* [T/img_len, D] act */
  int32_t img_len;     /* tokens per image, >= 1, dividing T */
  float eps;           /* > 0; the pages' layer_norm uses the library default 1e-5 */
  void* x_mod;         /* [T, D] act out: m */
} moe_adaln_t;

/* Library version (major*10000 + minor*100 + patch). */
int32_t moe_version(void);

/* Message of the last failing call on this thread ("" if none). */
const char* moe_last_error(void);

/* Bytes of scratch `ws` that every call of this configuration needs (host only). */
size_t moe_workspace_size(const moe_config_t* cfg);

/* Row capacity R_max of the expert-contiguous buffers x_perm, h_perm, y_perm,
 * row_token, row_gate: each expert segment starts on a 256-row boundary, so
 * R_max = round_up(K*T + 255*E, 256).  Host only. */
int64_t moe_max_rows(const moe_config_t* cfg);

/* Zero the first 256 bytes of `ws`: the status word and the counters the kernels keep
 * between launches (asynchronous on `stream`).  Once before first use.
 * Layout of those bytes: status word and error site (0, 4); blocks-done counters of the
 * router (64) and the per-image loss (192); bytes 128..191 reserved; the fused GEMM2's count of
 * finished routed tiles (224); the CTA-pair GEMM's exit and tile-claim counters (228, 232).
 * Every kernel leaves its counters at zero when it ends.
 * Bytes 240..247 are two test words that only the host writes (zero in normal use); they let a
 * test make a bounded wait run out without faulting anything:
 *   word at 240, bit 0: the routed tiles of moe_expert_gemm2_combine do not report themselves
 *                       done, so the shared tiles' wait for them cannot end;
 *                bit 1: each grid barrier of the Expert-Race selection waits for one arrival
 *                       more than the launch makes;
 *   word at 244: limit of those two waits in microseconds (0 = the default of 1 s).
 * A wait that runs out records MOE_ERR_TIMEOUT for moe_check_status; the kernel then finishes
 * with invalid outputs, and the next call (with the words cleared) is unaffected. */
int moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read the status word of `ws`, clear it, and return
 * MOE_OK, MOE_ERR_DEVICE_CHECK or MOE_ERR_TIMEOUT.  The only call that blocks. */
int moe_check_status(void* ws, void* stream);

/*
 * moe_route -- router of the layer (MoEGate): gate logits, softmax, selection,
 * per-expert counts and the expert-level balance loss.
 *   x           [T,D] act      input tokens
 *   wg          [E,D] act      gate weight
 *   router_bias [E] fp32 or NULL   added to the logits
 *   topk_idx    [T,Kmax] int32 out  Kmax = K (top-K) or E (race).  Each token's
 *               experts in descending score, ties to the lower id; race pads
 *               a token's unused slots with -1
 *   topk_w      [T,Kmax] fp32 out   g = the selected softmax scores (not
 *               renormalised); 0 on padded slots
 *   n_sel       [T] int32 out or NULL  experts chosen per token (race:
 *               required, 0..E; top-K: K for every token)
 *   counts      [E] int32 out   sum_t I(t,i)
 *   aux_loss    [1] fp32 out    L_balance with T = this call's tokens (seq_len = 0), or the
 *               mean over images of L_balance with T = seq_len tokens per image
 *   mod         adaLN modulation of x before routing (see moe_adaln_t), or NULL
 * Race selection: the S = K*T largest scores of the flattened T x E matrix,
 * ties to the lower flat index t*E+i, found by an exact radix select on the
 * fp32 score bits.
 */
int moe_route(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
              int32_t* topk_idx, float* topk_w, int32_t* n_sel, int32_t* counts, float* aux_loss,
              const moe_adaln_t* mod, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_dispatch -- permute tokens into expert-contiguous order (only the
 * selected experts are computed, "MOE 回顾").  Expert i's rows occupy
 * [P_i, P_i + counts_i) with P_i = sum_{j<i} round_up(counts_j, 256); tokens
 * ascend inside a segment.  Deterministic (no order-dependent atomics).
 *   x          [T,D] act          tokens
 *   topk_idx   [T,Kmax] int32     from moe_route (-1 = unused slot)
 *   topk_w     [T,Kmax] fp32      gates
 *   n_sel      [T] int32 or NULL  NULL means K for every token (top-K)
 *   offsets    [E+1] int32 out    unpadded exclusive scan of the counts
 *   pos        [T,Kmax] int32 out row of (t, slot k) in the permuted buffers, -1 if unused
 *   row_token  [R_max] int32 out  token of each row, -1 on padding rows
 *   row_gate   [R_max] fp32 out   gate of each row, 0 on padding rows
 *   x_perm     [R_max,D] act out  x_perm[pos[t,k]] = x[t]; the padding rows of each expert
 *              segment are written with zeros (rows after the last segment are untouched).  NULL:
 *              write the positions only (x may then be NULL too), for
 *              moe_expert_gemm1_gather, which reads the rows of x itself
 * An index outside [0,E) is skipped and sets MOE_ERR_DEVICE_CHECK in ws.
 */
int moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const float* topk_w,
                 const int32_t* n_sel, int32_t* offsets, int32_t* pos, int32_t* row_token,
                 float* row_gate, void* x_perm, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_gemm1 -- first expert layer with bias and GELU fused:
 *   h_perm[r] = gelu(W1_{e(r)} x_perm[r] + b1_{e(r)})  for the rows of every
 *               expert segment (e(r) read from `offsets` on the device)
 *   h_sh[t]   = gelu(W1s x[t] + b1s)  (all n_s shared experts side by side)
 *   offsets [E+1] int32 (moe_dispatch output); b1 [E,H] / b1s [n_s,H] may be NULL;
 *   h_perm [R_max,H] act out; h_sh [T,n_s*H] act out (NULL when n_s = 0).
 * bf16 / fp16: one persistent tcgen05 kernel (TMA-fed, TMEM accumulators,
 * 256 x 256 tiles on CTA pairs, one narrower column tile per row block where
 * 256 does not divide the width) runs the routed segments and the shared block
 * together.  fp32: FFMA kernel.
 */
int moe_expert_gemm1(const moe_config_t* cfg, const int32_t* offsets, const void* x_perm,
                     const void* x, const void* w1, const void* b1, const void* w1s, const void* b1s,
                     void* h_perm, void* h_sh, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_gemm1_gather -- moe_expert_gemm1 without x_perm: each routed row
 * r of the expert-contiguous layout is row row_token[r] of x, copied into
 * shared memory by two gather warps of the GEMM (16-byte cp.async into the
 * swizzled stage), so the dispatch writes positions only and the permuted copy
 * of x never exists.  Padding rows (row_token -1) read row 0; their h rows are
 * never used.
 *   row_token [R_max] int32 from moe_dispatch; other arguments as moe_expert_gemm1.
 * Only for bf16 or fp16 with gemm_impl AUTO (MOE_ERR_UNSUPPORTED otherwise).
 */
int moe_expert_gemm1_gather(const moe_config_t* cfg, const int32_t* offsets, const int32_t* row_token, const void* x,
                            const void* w1, const void* b1, const void* w1s, const void* b1s, void* h_perm,
                            void* h_sh, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_gemm2 -- second expert layer with bias and gate scaling fused:
 *   y_perm[r] = row_gate[r] * (W2_{e(r)} h_perm[r] + b2_{e(r)})   act [R_max,D]
 *   y_sh[t]   = sum_j (W2s_j h_sh[t, j*H:(j+1)*H] + b2s_j)         act [T,D]
 *   (fp32 accumulation and epilogue; one rounding to the act type on store)
 *   b2 [E,D] / b2s [n_s,D] may be NULL; y_sh NULL when n_s = 0.
 */
int moe_expert_gemm2(const moe_config_t* cfg, const int32_t* offsets, const void* h_perm,
                     const void* h_sh, const void* w2, const void* b2, const void* w2s,
                     const void* b2s, const float* row_gate, void* y_perm, void* y_sh,
                     void* ws, size_t ws_bytes, void* stream);

/* moe_expert_mlp -- moe_expert_gemm1 followed by moe_expert_gemm2. */
int moe_expert_mlp(const moe_config_t* cfg, const int32_t* offsets, const void* x_perm,
                   const void* x, const void* w1, const void* b1, const void* w2, const void* b2,
                   const void* w1s, const void* b1s, const void* w2s, const void* b2s,
                   const float* row_gate, void* h_perm, void* h_sh, void* y_perm, void* y_sh,
                   void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_gemm2_combine -- moe_expert_gemm2 and moe_combine in one launch:
 * the shared experts' GEMM2 tiles add each token's routed rows y_perm[pos[t,k]]
 * (slot order, fp32) to their own output and write `out` directly, so the
 * shared output never goes to memory.  The routed tiles of the same launch
 * write y_perm first; the shared tiles' epilogue waits (bounded) until every
 * routed tile is stored.
 *   Arguments as moe_expert_gemm2 (no y_sh), plus pos [T,Kmax] and n_sel [T]
 *   (or NULL for top-K) from moe_dispatch / moe_route, and out [T,D] act.
 *   out[t] = sum_k y_perm[pos[t,k]] + sum_j (W2s_j h_sh_j + b2s_j), rounded once;
 *   with `res` (or NULL), out[t] = x_res[t] + alpha[t/img_len] * (that sum).
 * Only for bf16 or fp16 with gemm_impl AUTO and n_shared >= 1 (MOE_ERR_UNSUPPORTED
 * otherwise: call moe_expert_gemm2 and moe_combine).  Uses the counters at byte
 * offsets 224..235 of ws, which must be zero on entry (moe_workspace_init; each
 * launch leaves them zero).  Tiles are claimed in increasing order, routed ones
 * first, so the shared tiles only ever wait for routed tiles that running CTA
 * pairs hold: the wait ends however few pairs the device runs at once (other
 * streams' kernels included).  A wait that runs out (1 s) reports
 * MOE_ERR_TIMEOUT through moe_check_status.
 */
int moe_expert_gemm2_combine(const moe_config_t* cfg, const int32_t* offsets, const void* h_perm, const void* h_sh,
                             const void* w2, const void* b2, const void* w2s, const void* b2s, const float* row_gate,
                             const int32_t* pos, const int32_t* n_sel, void* y_perm, const moe_residual_t* res,
                             void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_combine -- MoE(x_t) = sum_{k < n_sel[t]} y_perm[pos[t,k]] + y_sh[t]
 * (the gates are already applied in y_perm), summed in fp32 in slot order
 * then the shared term, rounded once to the act type.
 *   y_perm [R_max,D] act; y_sh [T,D] act or NULL (n_s = 0);
 *   pos [T,Kmax] int32; n_sel [T] or NULL (= K); out [T,D] act;
 *   res: the adaLN-Zero residual (out[t] = x_res[t] + alpha[t/img_len] * MoE(x_t)),
 *   or NULL for MoE(x) alone.
 */
int moe_combine(const moe_config_t* cfg, const void* y_perm, const void* y_sh,
                const int32_t* pos, const int32_t* n_sel, const moe_residual_t* res, void* out, void* stream);

/*
 * moe_route_static -- moe_route for callers that cannot allocate device memory.
 * (No counterpart on the pages: this is a deployment convenience.)
 *
 * Same arguments, results and errors as moe_route, minus the workspace and the
 * adaLN modulation (it routes on x as given): the
 * router's scratch comes from a fixed 4 MiB array built into the library
 * (reserved on every GPU that loads it, until the process exits), so a caller
 * whose framework gives it no allocator, or that must not call cudaMalloc
 * after start-up, needs none.
 *   - Configurations whose scratch (moe_workspace_size) exceeds 4 MiB are
 *     rejected with MOE_ERR_WORKSPACE and a message; nothing is launched.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.  The call allocates nothing itself.
 *   - All calls share the one array: calls that may overlap on the GPU (other
 *     streams, other threads) race and must be serialised by the caller.  Each
 *     call clears the array's counters itself.  Device-detected errors (a
 *     bounded wait that ran out, for instance) stay in the array's status word
 *     until moe_route_static_check_status reads them.
 */
int moe_route_static(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                     int32_t* topk_idx, float* topk_w, int32_t* n_sel, int32_t* counts, float* aux_loss,
                     void* stream);

/* moe_check_status for the built-in array of moe_route_static on the current
 * device: synchronise `stream`, read the first error the router's kernels
 * recorded since the last check (MOE_OK, MOE_ERR_DEVICE_CHECK or
 * MOE_ERR_TIMEOUT) and clear it.  Blocks; allocates nothing. */
int moe_route_static_check_status(void* stream);

/*
 * moe_balance_stats -- the statistics the balance loss is made of, for a loss
 * over a batch split between ranks (or between calls).  "MOE-DIT", eq.
 * L_balance: L = alpha sum_i f_i p_i with f_i = (E/(K T)) counts_i and
 * p_i = (1/T) sum_t P[t,i] depends on the batch only through counts_i and
 * s_i = sum_t P[t,i], and both add over disjoint parts of the batch.
 *   counts      [E] int32   from the last moe_route on this ws
 *   ws          the workspace that moe_route call used (its score sums stay there
 *               until the next moe_route on it)
 *   stats       [2E] fp64 out: counts_0..counts_{E-1}, then s_0..s_{E-1}
 *               (s_i summed in fp64 in the router's fixed order)
 * Sum stats over the ranks (one all-reduce of 2E values, e.g. NCCL over
 * NVLink), then moe_balance_loss_from_stats.  A call that routed zero tokens
 * gives zeros.  Not available after moe_route_static (no workspace).
 */
int moe_balance_stats(const moe_config_t* cfg, const int32_t* counts, const void* ws, size_t ws_bytes, double* stats,
                      void* stream);

/*
 * moe_balance_loss_from_stats -- L_balance of a batch from its summed
 * statistics: alpha sum_i (E/(K T_total)) stats[i] (stats[E+i] / T_total),
 * accumulated in fp64 in a fixed order, written as fp32.
 *   stats       [2E] fp64   moe_balance_stats of every part, summed
 *   T_total     tokens of the whole batch (the parts' T added); 0 gives 0
 *   aux_loss    [1] fp32 out
 * cfg supplies E, K and alpha.  With Expert-Race routing, K T_total is the
 * batch's number of selected pairs, as in the per-call loss.  This is the
 * whole-batch loss (seq_len is ignored): the per-image loss of seq_len > 0 is
 * a mean over images and is not a function of these sums.
 */
int moe_balance_loss_from_stats(const moe_config_t* cfg, const double* stats, long long T_total, float* aux_loss,
                                void* stream);

/*
 * moe_balance_loss_backward -- gradient of the expert-level balance loss with
 * respect to the router ("MOE-DIT", eq. L_balance; the counts come from the
 * discrete selection and carry no gradient): dL/dP[t,i] = alpha f_i / T, back
 * through the softmax to the logits, then through l = x Wg^T + b.
 *   x, wg, router_bias   as given to moe_route (the logits are recomputed in fp32)
 *   counts      [E] int32 from moe_route
 *   grad_scale  dObjective/dL_balance (1 for the loss alone)
 *   dwg         [E,D] fp32 out; dbias [E] fp32 out or NULL; dx [T,D] act out or NULL
 *   bws         scratch of moe_backward_workspace_size(cfg) bytes, 256-byte aligned
 * Whole-call loss only (seq_len = 0; MOE_ERR_UNSUPPORTED otherwise).  The sums
 * run in a fixed order: bit-reproducible.
 */
size_t moe_backward_workspace_size(const moe_config_t* cfg);
int moe_balance_loss_backward(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                              const int32_t* counts, float grad_scale, float* dwg, float* dbias, void* dx,
                              void* bws, size_t bws_bytes, void* stream);

/*
 * The expert MLPs' backward ("Scaling Diffusion Transformers to 16 Billion
 * Parameters": the DiT-MoE models are trained; "MOE 回顾" eq. MoE(x) and
 * "MOE-DIT" eq. MLP give the forward it differentiates).  For an objective J
 * with dout = dJ/dMoE(x):
 *   dZ_r  = g_r dout[t_r]                    (each routed row r of token t_r)
 *   dH_r  = dZ_r W2_e,  dU_r = dH_r * gelu'(u_r),  u_r = W1_e x_r + b1_e
 *   dW2_e = sum_r dZ_r^T gelu(u_r),  db2_e = sum_r dZ_r
 *   dW1_e = sum_r dU_r^T x_r,        db1_e = sum_r dU_r
 *   dgate[t,k] = dJ/dg = <dout_t, e_i(x_t)> for the token's k-th selected expert i
 *   dx_t  = sum_k (dU W1)[pos[t,k]] + the shared experts' part (weight 1, same forms)
 * The selection is discrete (no gradient through it); moe_router_backward takes
 * dgate the rest of the way to Wg, the router bias and x.
 */
typedef struct {
  const void* w1; const void* b1;     /* [E,H,D] act, [E,H] act or NULL */
  const void* w2; const void* b2;     /* [E,D,H], [E,D] or NULL */
  const void* w1s; const void* b1s;   /* [n_s,H,D], [n_s,H] or NULL (n_s = 0: NULL) */
  const void* w2s; const void* b2s;   /* [n_s,D,H], [n_s,D] or NULL */
} moe_expert_weights_t;

typedef struct {                      /* fp32, the weights' shapes; overwritten.  Bias gradients may be NULL */
  float* dw1; float* db1; float* dw2; float* db2;
  float* dws1; float* dbs1; float* dws2; float* dbs2;
} moe_expert_grads_t;

/* Scratch of moe_expert_backward: dout and g*dout in permuted order, the
 * pre-activations (overwritten by dU), dx per routed row, the gates' row dots
 * and column-sum partials.  Host only. */
size_t moe_expert_backward_workspace_size(const moe_config_t* cfg);

/*
 * moe_expert_backward -- gradients of the expert MLPs, of their input and of the gates.
 *   x, x_perm, offsets, pos, topk_idx, n_sel, row_token, row_gate: the forward's
 *               input and its moe_route / moe_dispatch outputs (x_perm's padding
 *               rows are the zeros moe_dispatch writes)
 *   wts         the forward's expert weights
 *   h_perm, h_sh  the forward's moe_expert_gemm1 outputs (gelu(u) per row)
 *   dout        [T,D] act: dJ/dMoE(x)
 *   grads       fp32 weight gradients out (see moe_expert_grads_t)
 *   dgate       [T,Kmax] fp32 out: dJ/dg per selected slot, 0 on unused slots
 *   dx          [T,D] act out: the experts' part of dJ/dx
 *   ws          the forward's workspace (status word and GEMM counters)
 *   bws         scratch of moe_expert_backward_workspace_size(cfg) bytes, 256-byte aligned
 * Every GEMM runs on the CTA-pair tensor cores (the weights and the weight
 * gradients' operands are read MN-major by TMA, no transposed copies): the
 * pre-activations again, dU with the GELU derivative and the gates' row dots in
 * its epilogue, dx with the combine folded in, and dW2, dW1 reducing over each
 * expert's rows.  bf16 or fp16 with gemm_impl AUTO and act = 0 only
 * (MOE_ERR_UNSUPPORTED otherwise).  Sums of the bias gradients run in a fixed order.
 */
int moe_expert_backward(const moe_config_t* cfg, const void* x, const void* x_perm, const int32_t* offsets,
                        const int32_t* pos, const int32_t* topk_idx, const int32_t* n_sel, const int32_t* row_token,
                        const float* row_gate, const moe_expert_weights_t* wts, const void* h_perm, const void* h_sh,
                        const void* dout, const moe_expert_grads_t* grads, float* dgate, void* dx, void* ws,
                        size_t ws_bytes, void* bws, size_t bws_bytes, void* stream);

/*
 * moe_router_backward -- the router's part of the layer's backward: dJ/dP =
 * aux_scale * (the balance loss's alpha f_i / T on every score) + dgate on the
 * selected slots, back through the softmax and l = x Wg^T + b.
 *   x, wg, router_bias, counts, topk_idx, n_sel  as in the forward
 *   dgate       [T,Kmax] fp32 from moe_expert_backward, or NULL (balance loss only)
 *   dwg [E,D] fp32 out; dbias [E] fp32 out or NULL; dx [T,D] act or NULL
 *   dx_accumulate  1: dx += the router's part (dx holds the experts' part), 0: dx = it
 *   bws         scratch of moe_backward_workspace_size(cfg) bytes
 * Whole-call balance loss only (seq_len = 0).  Fixed-order sums: bit-reproducible.
 */
int moe_router_backward(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                        const int32_t* counts, const int32_t* topk_idx, const int32_t* n_sel, const float* dgate,
                        float aux_scale, float* dwg, float* dbias, void* dx, int32_t dx_accumulate, void* bws,
                        size_t bws_bytes, void* stream);

/*
 * moe_expert_frequency -- expert-selection frequency per label, the statistic of
 * the expert specialisation analysis ("Scaling Diffusion Transformers to 16
 * Billion Parameters": selection frequency by image class, spatial position
 * and denoising timestep).
 *   topk_idx    [T,Kmax] int32   selection from moe_route (-1 = unused slot)
 *   n_sel       [T] int32 or NULL  (race: required)
 *   seq_len     tokens per image, >= 1, dividing T
 *   seq_labels  [T/seq_len] int32 or NULL: the label of each image (its class,
 *               or its timestep or timestep bucket).  NULL labels every token
 *               by its patch position t mod seq_len.
 *   n_labels    rows of hist (NULL seq_labels: must equal seq_len)
 *   hist        [n_labels,E] int32 out: hist[b*E+i] = number of selected pairs
 *               (t,i) whose token carries label b.  Overwritten.
 *   ws          status word only (a label outside [0, n_labels) or an expert
 *               id >= E is skipped and reported through moe_check_status)
 * Integer counts: the result does not depend on the order of the atomics.
 */
int moe_expert_frequency(const moe_config_t* cfg, const int32_t* topk_idx, const int32_t* n_sel, int32_t seq_len,
                         const int32_t* seq_labels, int32_t n_labels, int32_t* hist, void* ws, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
