// C ABI of the layer: argument validation, workspace layout, TMA descriptor
// encoding and kernel launches.  Every entry point is asynchronous on the
// caller's stream; nothing is allocated; device data is never read on the host
// (except in moe_check_status, which exists to do exactly that).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "kernels.h"

using namespace moe;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}
int ok() {
  g_last_error.clear();
  return MOE_OK;
}
int cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// bf16 and fp16 share every 16-bit path; only conversions and MMA operand formats differ
bool is16(const moe_config_t* c) { return c->dtype == MOE_BF16 || c->dtype == MOE_F16; }
int elem_bytes(const moe_config_t* c) { return is16(c) ? 2 : 4; }

constexpr int kMaxT = 262144;

int validate(const moe_config_t* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", c->T);
  if (c->T > kMaxT) return fail(MOE_ERR_UNSUPPORTED, "T=%d above the supported %d", c->T, kMaxT);
  if (c->D <= 0 || c->H <= 0) return fail(MOE_ERR_INVALID_ARG, "D=%d H=%d must be positive", c->D, c->H);
  if (c->D % 64 || c->H % 64) return fail(MOE_ERR_UNSUPPORTED, "D=%d and H=%d must be multiples of 64", c->D, c->H);
  if (c->E < 1 || c->E > 32) return fail(MOE_ERR_UNSUPPORTED, "E=%d outside 1..32", c->E);
  if (c->K < 1 || c->K > c->E) return fail(MOE_ERR_INVALID_ARG, "K=%d outside 1..E=%d", c->K, c->E);
  if (c->n_shared < 0 || c->n_shared > 8) return fail(MOE_ERR_UNSUPPORTED, "n_shared=%d outside 0..8", c->n_shared);
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16 && c->dtype != MOE_F16) return fail(MOE_ERR_INVALID_ARG, "dtype=%d", c->dtype);
  if (c->routing != MOE_ROUTE_TOPK && c->routing != MOE_ROUTE_RACE) return fail(MOE_ERR_INVALID_ARG, "routing=%d", c->routing);
  if (c->act != 0 && c->act != 1) return fail(MOE_ERR_INVALID_ARG, "act=%d", c->act);
  if (c->gemm_impl < MOE_GEMM_AUTO || c->gemm_impl > MOE_GEMM_TC1) return fail(MOE_ERR_INVALID_ARG, "gemm_impl=%d", c->gemm_impl);
  if (c->seq_len < 0) return fail(MOE_ERR_INVALID_ARG, "seq_len=%d < 0", c->seq_len);
  if (c->gemm_pairs < 0) return fail(MOE_ERR_INVALID_ARG, "gemm_pairs=%d < 0", c->gemm_pairs);
  if (c->seq_len > 0 && c->T % c->seq_len)
    return fail(MOE_ERR_INVALID_ARG, "seq_len=%d does not divide T=%d", c->seq_len, c->T);
  if (route_smem_total(c->D, c->E, 32, is16(c), 1) > 232448 ||
      (is16(c) && route_mma_stages(c->D, c->E, 1) < 1))
    return fail(MOE_ERR_UNSUPPORTED, "E=%d x D=%d too large for the router's shared memory", c->E, c->D);
  return MOE_OK;
}

int kmax_of(const moe_config_t* c) { return c->routing == MOE_ROUTE_RACE ? c->E : c->K; }

long long max_rows(const moe_config_t* c) {
  const long long S = (long long)c->K * c->T;
  return (long long)round_up((size_t)(S + (long long)(kSegAlign - 1) * c->E), kSegAlign);
}

// dispatch: groups of 256 tokens (counts and ranks), 64 tokens per gather block
constexpr int kDispatchGroup = 256;
constexpr int kGatherTokens = 64;
int ngroups_of(int T) { return (T + kDispatchGroup - 1) / kDispatchGroup; }

struct WsLayout {
  size_t status, tile_counts, tile_psum, score_sum, P, seq_loss, race_sync, race_loc, race_counts, group_base, total;
};

WsLayout ws_layout(const moe_config_t* c) {
  WsLayout L{};
  const size_t T = (size_t)c->T, E = (size_t)c->E;
  // partial rows: one per router CTA (<= one per 16 tokens) or per fp32 token tile (>= 32 rows)
  const size_t max_route_tiles = (T + 15) / 16 + 1;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += round_up(bytes ? bytes : 1, 256); return o; };
  L.status = take(256);
  L.tile_counts = take(max_route_tiles * E * 4);
  L.tile_psum = take(max_route_tiles * E * 4);
  L.score_sum = take(E * 8);
  const bool race = c->routing == MOE_ROUTE_RACE;
  const bool per_image = c->seq_len > 0;
  L.P = take(race || per_image ? T * E * 4 : 0);
  L.seq_loss = take(per_image ? (T / (size_t)c->seq_len) * 8 : 0);
  L.race_sync = take(race ? (size_t)kRaceSyncWords * 4 : 0);
  L.race_loc = take(race ? (size_t)kRaceMaxCtas * 256 * 4 : 0);
  L.race_counts = take(race ? (size_t)kRaceMaxCtas * E * 4 : 0);
  L.group_base = take((size_t)ngroups_of(c->T) * E * 4);
  L.total = off;
  return L;
}

int check_ws(const moe_config_t* c, void* ws, size_t ws_bytes) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "ws is NULL");
  if ((uintptr_t)ws & 255u) return fail(MOE_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  const size_t need = ws_layout(c).total;
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "ws_bytes=%zu < %zu", ws_bytes, need);
  return MOE_OK;
}

#define REQUIRE_PTR(p)                                                              \
  do {                                                                              \
    if (!(p)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #p);                   \
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)
#define OPTIONAL_PTR(p)                                                             \
  do {                                                                              \
    if ((p) && !aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)

// words of the workspace's first 256 bytes (besides the status word at 0): blocks-done counters
// of the router (64), the dispatch count (128) and the per-image loss (192); the fused GEMM2's
// routed-tile count (224); the CTA-pair GEMM's exit counter (228) and tile claim counter (232);
// two test words written only by the host (240: flags, 244: wait limit in microseconds)
constexpr size_t kWsDoneCtr = 224, kWsExitCtr = 228, kWsSchedCtr = 232, kWsTestWords = 240;

int* status_ptr(void* ws) { return reinterpret_cast<int*>(ws); }
template <typename T> T* ws_at(void* ws, size_t off) { return reinterpret_cast<T*>((uint8_t*)ws + off); }

// ---------------------------------------------------------------- device info
int num_sms_current() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// ---------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major [rows, cols] tensor, 128-byte swizzled boxes of box_rows x (128 B)
int make_tmap(CUtensorMap* m, const void* base, int dtype, long long rows, long long cols, int box_rows,
              const char* what) {
  auto fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const int eb = dtype == MOE_F32 ? 4 : 2;
  const CUtensorMapDataType ty = dtype == MOE_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == MOE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * eb};
  cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, ty, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (CUresult %d)", what, (int)r);
  return MOE_OK;
}

// x [rows, cols] 16-bit seen as 3-D {64 columns, rows, cols/64 blocks}: one box brings
// `box_rows` rows x ceil(cols/128) swizzled 128-byte blocks (half of each row),
// block-major.  Returns false when the driver does not accept the layout (the
// caller then uses 2-D boxes).
bool make_tmap_rows3d(CUtensorMap* m, const void* base, int dtype, long long rows, long long cols, int box_rows,
                      int box_blocks = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)(rows > 0 ? rows : 1), (cuuint64_t)(cols / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, 128};
  // one box = box_blocks 64-column blocks (default: half of a row block)
  const cuuint32_t blocks = (cuuint32_t)(box_blocks > 0 ? box_blocks : (cols / 64 + 1) / 2);
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  if (blocks > 256) return false;
  CUresult r = fn(m, dtype == MOE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

void moe::set_last_error_message(const char* msg) { g_last_error = msg ? msg : ""; }

// ====================================================================== ABI
extern "C" {

int32_t moe_version(void) { return 100; }

const char* moe_last_error(void) { return g_last_error.c_str(); }

size_t moe_workspace_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return ws_layout(cfg).total;
}

int64_t moe_max_rows(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return -1;
  return max_rows(cfg);
}

int moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) return fail(MOE_ERR_INVALID_ARG, "ws is NULL or smaller than 256 bytes");
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "moe_workspace_init");
  return ok();
}

int moe_check_status(void* ws, void* stream) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "ws is NULL");
  int h[2] = {0, 0};
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_check_status");
  if (h[0] != 0) {
    e = cudaMemsetAsync(ws, 0, 256, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (h[0] == 2 /* timeout */) return fail(MOE_ERR_TIMEOUT, "a kernel's bounded wait ran out (site %d)", h[1]);
    return fail(MOE_ERR_DEVICE_CHECK, "a kernel found a bad index (site %d)", h[1]);
  }
  return ok();
}

int moe_route(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
              int32_t* topk_idx, float* topk_w, int32_t* n_sel, int32_t* counts, float* aux_loss,
              const moe_adaln_t* mod, void* ws, size_t ws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  const bool race = cfg->routing == MOE_ROUTE_RACE;
  REQUIRE_PTR(counts);
  if (!aux_loss) return fail(MOE_ERR_INVALID_ARG, "aux_loss is NULL");
  if ((rc = check_ws(cfg, ws, ws_bytes))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if (cfg->T == 0) {
    if ((e = cudaMemsetAsync(counts, 0, cfg->E * sizeof(int32_t), s)) != cudaSuccess) return cuda_fail(e, "moe_route");
    if ((e = cudaMemsetAsync(aux_loss, 0, sizeof(float), s)) != cudaSuccess) return cuda_fail(e, "moe_route");
    if ((e = cudaMemsetAsync(ws_at<double>(ws, ws_layout(cfg).score_sum), 0, cfg->E * sizeof(double), s)) !=
        cudaSuccess)
      return cuda_fail(e, "moe_route");
    return ok();
  }
  REQUIRE_PTR(x);
  REQUIRE_PTR(wg);
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(topk_w);
  OPTIONAL_PTR(router_bias);
  OPTIONAL_PTR(n_sel);
  if (race && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  if (mod) {
    if (!is16(cfg)) return fail(MOE_ERR_UNSUPPORTED, "adaLN modulation in the router needs a 16-bit act type");
    REQUIRE_PTR(mod->gamma);
    REQUIRE_PTR(mod->beta);
    REQUIRE_PTR(mod->x_mod);
    if (mod->img_len < 1 || cfg->T % mod->img_len)
      return fail(MOE_ERR_INVALID_ARG, "mod->img_len=%d does not divide T=%d", mod->img_len, cfg->T);
    if (!(mod->eps > 0.f) || mod->eps > 1.f) return fail(MOE_ERR_INVALID_ARG, "mod->eps=%g outside (0, 1]", mod->eps);
  }
  const WsLayout L = ws_layout(cfg);
  const int sms = num_sms_current();
  int tile = 0, threads = 0;
  const bool b16 = is16(cfg);
  route_plan(cfg->T, cfg->D, cfg->E, b16, mod != nullptr, sms, &tile, &threads);
  const int ntiles = (cfg->T + tile - 1) / tile;
  const int grid = ntiles < sms ? ntiles : sms;
  // partial sums: one row per CTA (16-bit kernel) or per token tile (fp32 kernel)
  const int nparts = b16 ? grid : ntiles;
  CUtensorMap tm, tmm;
  int tmap3d = 0;
  const int box_blocks = b16 ? route_box_blocks(cfg->D, cfg->E, mod != nullptr) : 0;
  if (b16 && make_tmap_rows3d(&tm, x, cfg->dtype, cfg->T, cfg->D, tile, box_blocks)) tmap3d = 1;
  else if ((rc = make_tmap(&tm, x, cfg->dtype, cfg->T, cfg->D, tile, "x"))) return rc;
  // the modulated rows go out with the same box geometry as x comes in
  tmm = tm;
  if (mod) {
    if (tmap3d) {
      if (!make_tmap_rows3d(&tmm, mod->x_mod, cfg->dtype, cfg->T, cfg->D, tile, box_blocks))
        return fail(MOE_ERR_CUDA, "tensor map for mod->x_mod failed");
    } else if ((rc = make_tmap(&tmm, mod->x_mod, cfg->dtype, cfg->T, cfg->D, tile, "x_mod"))) {
      return rc;
    }
  }
  RouteArgs ra{};
  ra.tmap3d = tmap3d;
  ra.x = x; ra.wg = wg; ra.bias = router_bias;
  ra.T = cfg->T; ra.D = cfg->D; ra.E = cfg->E; ra.K = cfg->K; ra.b16 = b16; ra.f16 = cfg->dtype == MOE_F16;
  ra.tile_rows = tile; ra.ntiles = ntiles; ra.grid = grid;
  ra.topk_idx = topk_idx; ra.topk_w = topk_w; ra.n_sel = race ? nullptr : n_sel;
  const bool per_image = cfg->seq_len > 0;
  ra.P = race || per_image ? ws_at<float>(ws, L.P) : nullptr;
  ra.race = race;
  SeqLossArgs sl{};
  sl.P = ra.P; sl.topk_idx = topk_idx; sl.n_sel = n_sel;
  sl.T = cfg->T; sl.E = cfg->E; sl.K = cfg->K; sl.Kmax = kmax_of(cfg); sl.L = cfg->seq_len;
  sl.alpha = cfg->alpha;
  sl.seq_loss = per_image ? ws_at<double>(ws, L.seq_loss) : nullptr;
  sl.ctr = ws_at<unsigned int>(ws, 192);
  sl.aux_loss = aux_loss;
  ra.tile_counts = ws_at<int32_t>(ws, L.tile_counts);
  ra.tile_psum = ws_at<float>(ws, L.tile_psum);
  ra.status = status_ptr(ws);
  if (mod) { ra.gamma = mod->gamma; ra.beta = mod->beta; ra.img_len = mod->img_len; ra.eps = mod->eps; }
  FinalizeArgs fa{};
  fa.T = cfg->T; fa.E = cfg->E; fa.K = cfg->K; fa.alpha = cfg->alpha;
  fa.counts = counts; fa.aux_loss = aux_loss;
  fa.score_sum = ws_at<double>(ws, L.score_sum);
  fa.tile_psum = ra.tile_psum; fa.ntiles_psum = nparts;
  fa.tile_counts = ra.tile_counts; fa.ntiles_counts = nparts;
  fa.ctr = ws_at<unsigned int>(ws, 64);
  if (!race) {
    // the router's last block finalizes counts and loss
    if ((e = launch_route(ra, fa, &tm, &tmm, s)) != cudaSuccess) return cuda_fail(e, "route kernel");
    if (per_image && (e = launch_seq_loss(sl, s)) != cudaSuccess) return cuda_fail(e, "per-image loss kernel");
    return ok();
  }
  // Expert-Race: the router writes the score matrix (and clears the selection's
  // scratch); one cooperative launch selects and finalizes.
  ra.zero = ws_at<uint32_t>(ws, L.race_sync);
  ra.nzero = kRaceSyncWords;
  FinalizeArgs none{};
  if ((e = launch_route(ra, none, &tm, &tmm, s)) != cudaSuccess) return cuda_fail(e, "route kernel");
  RaceArgs rr{};
  rr.P = ra.P; rr.T = cfg->T; rr.E = cfg->E; rr.K = cfg->K;
  rr.sync = ra.zero;
  rr.loc = ws_at<uint32_t>(ws, L.race_loc);
  rr.grid = race_plan(cfg->T, sms, &rr.tpc);
  rr.topk_idx = topk_idx; rr.topk_w = topk_w; rr.n_sel = n_sel;
  rr.tile_counts = ws_at<int32_t>(ws, L.race_counts);
  rr.status = status_ptr(ws);
  rr.test = ws_at<const uint32_t>(ws, kWsTestWords);
  fa.tile_counts = rr.tile_counts; fa.ntiles_counts = rr.grid;
  if ((e = launch_race_select(rr, fa, s)) != cudaSuccess) return cuda_fail(e, "Expert-Race select kernel");
  if (per_image && (e = launch_seq_loss(sl, s)) != cudaSuccess) return cuda_fail(e, "per-image loss kernel");
  return ok();
}

int moe_balance_stats(const moe_config_t* cfg, const int32_t* counts, const void* ws, size_t ws_bytes, double* stats,
                      void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  REQUIRE_PTR(counts);
  REQUIRE_PTR(stats);
  if ((rc = check_ws(cfg, const_cast<void*>(ws), ws_bytes))) return rc;
  const double* ssum = ws_at<double>(const_cast<void*>(ws), ws_layout(cfg).score_sum);
  cudaError_t e = launch_balance_stats(counts, ssum, cfg->E, stats, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "balance statistics kernel");
  return ok();
}

int moe_balance_loss_from_stats(const moe_config_t* cfg, const double* stats, long long T_total, float* aux_loss,
                                void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  REQUIRE_PTR(stats);
  if (!aux_loss) return fail(MOE_ERR_INVALID_ARG, "aux_loss is NULL");
  if (T_total < 0) return fail(MOE_ERR_INVALID_ARG, "T_total=%lld < 0", T_total);
  cudaError_t e = launch_balance_loss_from_stats(stats, cfg->E, cfg->K, T_total, cfg->alpha, aux_loss,
                                                 (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "balance loss kernel");
  return ok();
}

namespace {
struct BwdLayout { size_t dl, db_part, partials, total; };
BwdLayout bwd_layout(const moe_config_t* c) {
  BwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += round_up(bytes ? bytes : 1, 256); return o; };
  L.dl = take((size_t)c->T * c->E * sizeof(float));
  L.db_part = take((size_t)kBwdMaxBlocks * c->E * sizeof(float));
  // partial rows: one per chunk of tokens (three-kernel path) or per CTA of the one-pass kernel
  int pass_tpc = 0;
  const size_t pass_rows = (size_t)router_bwd_pass_grid(c->T, num_sms_current(), &pass_tpc);
  const size_t chunks = (size_t)balance_grad_chunks(c->T);
  const size_t nparts = chunks > pass_rows ? chunks : pass_rows;
  L.partials = take(nparts * c->E * c->D * sizeof(float));
  L.total = off;
  return L;
}
}  // namespace

size_t moe_backward_workspace_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return bwd_layout(cfg).total;
}

namespace {
// The router's backward: dJ/dP = the balance loss's term (times aux_scale) on every score plus
// dgate on the selected slots (or none), through the softmax and l = x Wg^T + b.
int router_backward(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                    const int32_t* counts, const int32_t* topk_idx, const int32_t* n_sel, const float* dgate,
                    float aux_scale, float* dwg, float* dbias, void* dx, int dx_accumulate, void* bws,
                    size_t bws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (cfg->seq_len > 0)
    return fail(MOE_ERR_UNSUPPORTED, "the balance-loss backward covers the whole-call loss (seq_len = 0)");
  if ((size_t)cfg->E * cfg->D * elem_bytes(cfg) > 232448)
    return fail(MOE_ERR_UNSUPPORTED, "E=%d x D=%d: the gate weight does not fit the backward's shared memory", cfg->E,
                cfg->D);
  REQUIRE_PTR(dwg);
  OPTIONAL_PTR(dbias);
  if (!bws) return fail(MOE_ERR_INVALID_ARG, "bws is NULL");
  if ((uintptr_t)bws & 255u) return fail(MOE_ERR_INVALID_ARG, "bws must be 256-byte aligned");
  if (bws_bytes < moe_backward_workspace_size(cfg))
    return fail(MOE_ERR_WORKSPACE, "bws_bytes=%zu < %zu", bws_bytes, moe_backward_workspace_size(cfg));
  if (dx_accumulate && !dx) return fail(MOE_ERR_INVALID_ARG, "dx_accumulate needs dx");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if (cfg->T == 0) {
    if ((e = cudaMemsetAsync(dwg, 0, (size_t)cfg->E * cfg->D * sizeof(float), s)) != cudaSuccess) return cuda_fail(e, "backward");
    if (dbias && (e = cudaMemsetAsync(dbias, 0, cfg->E * sizeof(float), s)) != cudaSuccess) return cuda_fail(e, "backward");
    return ok();
  }
  REQUIRE_PTR(x);
  REQUIRE_PTR(wg);
  REQUIRE_PTR(counts);
  OPTIONAL_PTR(router_bias);
  OPTIONAL_PTR(dx);
  if (dgate) {
    REQUIRE_PTR(topk_idx);
    OPTIONAL_PTR(n_sel);
    if (cfg->routing == MOE_ROUTE_RACE && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  }
  BalanceGradArgs a{};
  a.x = x; a.wg = wg; a.bias = router_bias; a.counts = counts;
  a.T = cfg->T; a.D = cfg->D; a.E = cfg->E; a.K = cfg->K; a.dtype = cfg->dtype;
  a.alpha = cfg->alpha; a.scale = aux_scale;
  a.dgate = dgate; a.topk_idx = topk_idx; a.n_sel = n_sel; a.Kmax = kmax_of(cfg); a.dx_accumulate = dx_accumulate;
  const BwdLayout BL = bwd_layout(cfg);
  a.dx = dx; a.dwg = dwg; a.dbias = dbias;
  a.dl = ws_at<float>(bws, BL.dl);
  a.db_part = ws_at<float>(bws, BL.db_part);
  a.partials = ws_at<float>(bws, BL.partials);
  CUtensorMap tmx;
  if (router_bwd_mma_fits(cfg->D, cfg->E, cfg->dtype) && make_tmap_rows3d(&tmx, x, cfg->dtype, cfg->T, cfg->D, 16)) {
    const int nrb = (cfg->T + 15) / 16;
    a.mma_grid = nrb < num_sms_current() ? nrb : num_sms_current();
    a.tmap_x = &tmx;
  } else if (router_bwd_pass_fits(cfg->D, cfg->E, cfg->dtype, cfg->T, num_sms_current())) {
    a.pass_grid = router_bwd_pass_grid(cfg->T, num_sms_current(), &a.pass_tpc);
  }
  // 8 tokens per block (one per warp) at a time: enough blocks to keep every SM's memory pipe busy
  int blocks = num_sms_current() * 4;
  if (blocks > kBwdMaxBlocks) blocks = kBwdMaxBlocks;
  const int need = (cfg->T + 7) / 8;
  if (blocks > need) blocks = need;
  if ((e = launch_balance_grad(a, blocks, s)) != cudaSuccess) return cuda_fail(e, "router backward kernels");
  return ok();
}
}  // namespace

int moe_balance_loss_backward(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                              const int32_t* counts, float grad_scale, float* dwg, float* dbias, void* dx,
                              void* bws, size_t bws_bytes, void* stream) {
  return router_backward(cfg, x, wg, router_bias, counts, nullptr, nullptr, nullptr, grad_scale, dwg, dbias, dx, 0,
                         bws, bws_bytes, stream);
}

int moe_expert_frequency(const moe_config_t* cfg, const int32_t* topk_idx, const int32_t* n_sel, int32_t seq_len,
                         const int32_t* seq_labels, int32_t n_labels, int32_t* hist, void* ws, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (seq_len < 1) return fail(MOE_ERR_INVALID_ARG, "seq_len=%d < 1", seq_len);
  if (cfg->T % seq_len) return fail(MOE_ERR_INVALID_ARG, "seq_len=%d does not divide T=%d", seq_len, cfg->T);
  if (n_labels < 1 || (long long)n_labels * cfg->E > (1ll << 30))
    return fail(MOE_ERR_INVALID_ARG, "n_labels=%d outside 1..2^30/E", n_labels);
  if (!seq_labels && n_labels != seq_len)
    return fail(MOE_ERR_INVALID_ARG, "position labels need n_labels == seq_len (%d != %d)", n_labels, seq_len);
  REQUIRE_PTR(hist);
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "ws is NULL");
  if ((uintptr_t)ws & 255u) return fail(MOE_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  if (cfg->T > 0) {
    REQUIRE_PTR(topk_idx);
    OPTIONAL_PTR(n_sel);
    OPTIONAL_PTR(seq_labels);
    if (cfg->routing == MOE_ROUTE_RACE && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  }
  FreqArgs fa{};
  fa.topk_idx = topk_idx; fa.n_sel = n_sel;
  fa.T = cfg->T; fa.E = cfg->E; fa.K = cfg->K; fa.Kmax = kmax_of(cfg); fa.L = seq_len;
  fa.labels = seq_labels; fa.n_labels = n_labels; fa.hist = hist;
  fa.status = status_ptr(ws);
  cudaError_t e = launch_frequency(fa, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "frequency kernel");
  return ok();
}

int moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const float* topk_w,
                 const int32_t* n_sel, int32_t* offsets, int32_t* pos, int32_t* row_token,
                 float* row_gate, void* x_perm, void* ws, size_t ws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  const bool race = cfg->routing == MOE_ROUTE_RACE;
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(row_token);
  REQUIRE_PTR(row_gate);
  if ((rc = check_ws(cfg, ws, ws_bytes))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  const long long R = max_rows(cfg);
  if (cfg->T == 0) {
    if ((e = cudaMemsetAsync(offsets, 0, (cfg->E + 1) * sizeof(int32_t), s)) != cudaSuccess) return cuda_fail(e, "moe_dispatch");
    if ((e = cudaMemsetAsync(row_token, 0xFF, R * sizeof(int32_t), s)) != cudaSuccess) return cuda_fail(e, "moe_dispatch");
    if ((e = cudaMemsetAsync(row_gate, 0, R * sizeof(float), s)) != cudaSuccess) return cuda_fail(e, "moe_dispatch");
    return ok();
  }
  if (x_perm) REQUIRE_PTR(x);           // without x_perm only positions are written (GEMM1 gathers the rows)
  REQUIRE_PTR(topk_idx);
  REQUIRE_PTR(topk_w);
  REQUIRE_PTR(pos);
  OPTIONAL_PTR(x_perm);
  OPTIONAL_PTR(n_sel);
  if (race && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  const WsLayout L = ws_layout(cfg);
  DispatchArgs da{};
  da.x = x; da.b16 = is16(cfg);
  da.topk_idx = topk_idx; da.topk_w = topk_w; da.n_sel = n_sel;
  da.T = cfg->T; da.D = cfg->D; da.E = cfg->E; da.K = cfg->K; da.Kmax = kmax_of(cfg);
  da.ngroups = ngroups_of(cfg->T);
  da.tpb = kGatherTokens;
  da.r_max = R;
  da.group_base = ws_at<int32_t>(ws, L.group_base);
  da.offsets = offsets; da.pos = pos; da.row_token = row_token; da.row_gate = row_gate;
  da.x_perm = x_perm;
  da.status = status_ptr(ws);
  if ((e = launch_dispatch(da, s)) != cudaSuccess) return cuda_fail(e, "dispatch kernels");
  return ok();
}

namespace {

// adaLN-Zero residual argument: both pointers 16-byte aligned, img_len dividing T
int check_residual(const moe_config_t* cfg, const moe_residual_t* res) {
  if (!res) return MOE_OK;
  if (!res->x_res || !res->alpha) return fail(MOE_ERR_INVALID_ARG, "res->x_res and res->alpha must be set");
  if (!aligned16(res->x_res) || !aligned16(res->alpha))
    return fail(MOE_ERR_INVALID_ARG, "res->x_res and res->alpha must be 16-byte aligned");
  if (res->img_len < 1 || cfg->T % res->img_len)
    return fail(MOE_ERR_INVALID_ARG, "res->img_len=%d does not divide T=%d", res->img_len, cfg->T);
  return MOE_OK;
}

}  // namespace

namespace {

// A0/B0: routed problem (A [rows0, K0], B [brows0, K0]); A1/B1: shared problem
// (A [rows1, K1], B [brows1, bcols1]; bcols1 < K1 when B is a K-split stack)
int run_gemm(const moe_config_t* cfg, GemmArgs& g, const void* A0, long long rows0, const void* B0,
             long long brows0, const void* A1, long long rows1, const void* B1, long long brows1, int K0,
             int K1, int bcols1, void* ws, cudaStream_t s) {
  cudaError_t e;
  const bool tc = is16(cfg) && cfg->gemm_impl != MOE_GEMM_SIMT;
  if (!tc) {
    if ((e = launch_gemm_simt(g, s)) != cudaSuccess) return cuda_fail(e, "FFMA expert GEMM");
    return ok();
  }
  const bool pair = cfg->gemm_impl == MOE_GEMM_AUTO;     // 2-SM tiles unless the 1-SM kernel is asked for
  const int n1 = g.nprob > 1 ? g.p[1].N : 0;
  const int bn = pair ? gemm_pair_pick_bn(g.p[0].N, n1) : gemm_tc_pick_bn(g.p[0].N, n1);
  if (!bn) return fail(MOE_ERR_UNSUPPORTED, "no tile width divides N=%d", g.p[0].N);
  // boxes: A rows per CTA = 128; B rows per CTA = bn (1 SM) or bn/2 (2 SMs)
  const int brows_box = pair ? bn / 2 : bn;
  CUtensorMap ta[2], tb[2];
  int rc;
  if (g.p[0].gather_rows) {
    // gathered A rows: the GEMM's gather warps copy them; the map is not read
    if (!pair) return fail(MOE_ERR_UNSUPPORTED, "row gathering needs the CTA-pair GEMM");
    if ((rc = make_tmap(&ta[0], A0, cfg->dtype, rows0, K0, 128, "A0 (gathered rows)"))) return rc;
  } else if ((rc = make_tmap(&ta[0], A0, cfg->dtype, rows0, K0, 128, "A0"))) {
    return rc;
  }
  if ((rc = make_tmap(&tb[0], B0, cfg->dtype, brows0, K0, brows_box, "B0"))) return rc;
  if (g.nprob > 1) {
    if ((rc = make_tmap(&ta[1], A1, cfg->dtype, rows1, K1, 128, "A1"))) return rc;
    if ((rc = make_tmap(&tb[1], B1, cfg->dtype, brows1, bcols1, brows_box, "B1"))) return rc;
  } else {
    ta[1] = ta[0];
    tb[1] = tb[0];
  }
  if (pair) {
    // output boxes for the TMA-store epilogue: 32 rows x 128 bytes of h or y (act dtype)
    CUtensorMap to[2];
    // the routed output has the permuted layout's R_max rows, whatever the A tensor's row count
    const long long orows0 = g.p[0].routed ? g.r_max : rows0;
    if ((rc = make_tmap(&to[0], g.p[0].out, cfg->dtype, orows0, g.p[0].N, 32, "out0"))) return rc;
    if (g.nprob > 1) {
      if ((rc = make_tmap(&to[1], g.p[1].out, cfg->dtype, rows1, g.p[1].N, 32, "out1"))) return rc;
    } else {
      to[1] = to[0];
    }
    // tile claim counter, exit counter and test words of the workspace header
    g.sched_ctr = ws_at<unsigned int>(ws, kWsSchedCtr);
    g.exit_ctr = ws_at<unsigned int>(ws, kWsExitCtr);
    g.test = ws_at<const uint32_t>(ws, kWsTestWords);
    // B maps with half-height boxes for the narrower column tile (N = 1152: the last 128 columns)
    CUtensorMap tbn[2];
    if ((rc = make_tmap(&tbn[0], B0, cfg->dtype, brows0, K0, brows_box / 2, "B0 (narrow tiles)"))) return rc;
    if (g.nprob > 1) {
      if ((rc = make_tmap(&tbn[1], B1, cfg->dtype, brows1, bcols1, brows_box / 2, "B1 (narrow tiles)"))) return rc;
    } else {
      tbn[1] = tbn[0];
    }
    if ((e = launch_gemm_pair(g, ta, tb, to, tbn, bn, num_sms_current(), cfg->gemm_pairs, s)) != cudaSuccess)
      return cuda_fail(e, "tcgen05 CTA-pair expert GEMM");
    return ok();
  }
  if ((e = launch_gemm_tc(g, ta, tb, bn, num_sms_current(), s)) != cudaSuccess) return cuda_fail(e, "tcgen05 expert GEMM");
  return ok();
}

}  // namespace

namespace {

// 3-D fp32 tensor [z, rows, cols] (row-major), boxes of 32 rows x 32 columns (128 bytes, swizzled)
int make_tmap_f32_3d(CUtensorMap* m, void* base, long long z, long long rows, long long cols, const char* what) {
  auto fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1), (cuuint64_t)(z > 0 ? z : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)(rows * cols * 4)};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (CUresult %d)", what, (int)r);
  return MOE_OK;
}

// One operand of a CTA-pair problem as a 2-D [rows, cols] 16-bit tensor: K-major operands are
// read in boxes of 64 columns (K) x box_rows rows, MN-major ones in boxes of 64 x 64.
struct OperandMap { const void* base; long long rows, cols; int box_rows; };
// The output: 16-bit [rows, cols] in 32-row boxes of 64 columns, or fp32 [z, rows, cols].
struct OutputMap { void* base; int f32; long long z, rows, cols; };

int launch_pair_problems(const moe_config_t* cfg, GemmArgs& g, const OperandMap* A, const OperandMap* B,
                         const OutputMap* O, void* ws, cudaStream_t s) {
  CUtensorMap ta[2], tb[2], to[2];
  int rc;
  for (int q = 0; q < 2; ++q) {
    const int k = q < g.nprob ? q : 0;
    if ((rc = make_tmap(&ta[q], A[k].base, cfg->dtype, A[k].rows, A[k].cols, A[k].box_rows, "A"))) return rc;
    if ((rc = make_tmap(&tb[q], B[k].base, cfg->dtype, B[k].rows, B[k].cols, B[k].box_rows, "B"))) return rc;
    if (O[k].f32) {
      if ((rc = make_tmap_f32_3d(&to[q], O[k].base, O[k].z, O[k].rows, O[k].cols, "out"))) return rc;
    } else if ((rc = make_tmap(&to[q], O[k].base, cfg->dtype, O[k].rows, O[k].cols, 32, "out"))) {
      return rc;
    }
  }
  g.sched_ctr = ws_at<unsigned int>(ws, kWsSchedCtr);
  g.exit_ctr = ws_at<unsigned int>(ws, kWsExitCtr);
  g.test = ws_at<const uint32_t>(ws, kWsTestWords);
  const cudaError_t e = launch_gemm_pair(g, ta, tb, to, nullptr, 256, num_sms_current(), cfg->gemm_pairs, s);
  if (e != cudaSuccess) return cuda_fail(e, "tcgen05 CTA-pair GEMM (backward)");
  return MOE_OK;
}

// Scratch of the expert backward (bytes from the start of bws).
struct EbLayout { size_t dout_perm, dz_perm, du_perm, du_sh, dx_perm, dg, partial, total; int dg_stride; };
EbLayout eb_layout(const moe_config_t* c) {
  EbLayout L{};
  const size_t R = (size_t)max_rows(c), T = (size_t)c->T, D = (size_t)c->D, H = (size_t)c->H;
  const size_t ns = (size_t)c->n_shared, eb = 2;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += round_up(bytes ? bytes : 1, 256); return o; };
  L.dout_perm = take(R * D * eb);
  L.dz_perm = take(R * D * eb);
  L.du_perm = take(R * H * eb);
  L.du_sh = take(T * ns * H * eb);
  L.dx_perm = take(R * D * eb);
  L.dg_stride = (int)((H + 255) / 256) * kPairEpiSplit;   // per 256-column tile and epilogue warp
  L.dg = take(R * (size_t)L.dg_stride * 4);
  size_t cmax = D > H ? D : H;
  if (ns * H > cmax) cmax = ns * H;
  const size_t rmax = R > T ? R : T;
  L.partial = take((size_t)colsum_chunks((long long)rmax) * cmax * 4);
  L.total = off;
  return L;
}

}  // namespace

static int expert_gemm1(const moe_config_t* cfg, const int32_t* offsets, const void* x_perm, const int32_t* row_token,
                        const void* x, const void* w1, const void* b1, const void* w1s, const void* b1s,
                        void* h_perm, void* h_sh, void* ws, size_t ws_bytes, void* stream);

int moe_expert_gemm1(const moe_config_t* cfg, const int32_t* offsets, const void* x_perm,
                     const void* x, const void* w1, const void* b1, const void* w1s, const void* b1s,
                     void* h_perm, void* h_sh, void* ws, size_t ws_bytes, void* stream) {
  return expert_gemm1(cfg, offsets, x_perm, nullptr, x, w1, b1, w1s, b1s, h_perm, h_sh, ws, ws_bytes, stream);
}

int moe_expert_gemm1_gather(const moe_config_t* cfg, const int32_t* offsets, const int32_t* row_token,
                            const void* x, const void* w1, const void* b1, const void* w1s, const void* b1s,
                            void* h_perm, void* h_sh, void* ws, size_t ws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (!is16(cfg) || cfg->gemm_impl != MOE_GEMM_AUTO)
    return fail(MOE_ERR_UNSUPPORTED, "GEMM1 gathers its rows only for bf16 or fp16 with gemm_impl AUTO; "
                                     "use moe_dispatch with x_perm and moe_expert_gemm1");
  if (cfg->T > 0) {
    REQUIRE_PTR(row_token);
    REQUIRE_PTR(x);
  }
  return expert_gemm1(cfg, offsets, nullptr, row_token, x, w1, b1, w1s, b1s, h_perm, h_sh, ws, ws_bytes, stream);
}

static int expert_gemm1(const moe_config_t* cfg, const int32_t* offsets, const void* x_perm, const int32_t* row_token,
                        const void* x, const void* w1, const void* b1, const void* w1s, const void* b1s,
                        void* h_perm, void* h_sh, void* ws, size_t ws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if ((rc = check_ws(cfg, ws, ws_bytes))) return rc;
  if (cfg->T == 0) return ok();
  REQUIRE_PTR(offsets);
  if (!row_token) REQUIRE_PTR(x_perm);
  REQUIRE_PTR(w1);
  REQUIRE_PTR(h_perm);
  OPTIONAL_PTR(b1);
  const int ns = cfg->n_shared;
  if (ns > 0) {
    REQUIRE_PTR(x);
    REQUIRE_PTR(w1s);
    REQUIRE_PTR(h_sh);
    OPTIONAL_PTR(b1s);
  }
  const long long R = max_rows(cfg);
  GemmArgs g{};
  g.offsets = offsets; g.E = cfg->E; g.r_max = R; g.act = cfg->act; g.status = status_ptr(ws);
  g.b16 = is16(cfg); g.f16 = cfg->dtype == MOE_F16;
  g.nprob = ns > 0 ? 2 : 1;
  GemmProblem& p0 = g.p[0];
  p0.routed = 1; p0.N = cfg->H; p0.K = cfg->D; p0.epi = 0;
  p0.A = row_token ? x : x_perm; p0.B = w1; p0.out = h_perm; p0.ld_out = cfg->H; p0.bias = b1;
  p0.bias_stride = cfg->H;
  p0.bias_rows = 1;
  p0.gather_rows = row_token;
  p0.gather_nrows = cfg->T;
  if (ns > 0) {
    // the n_s stacked W1 [n_s,H,D] are one [n_s*H, D] matrix; b1s [n_s,H] one [n_s*H] row
    GemmProblem& p1 = g.p[1];
    p1.routed = 0; p1.M = cfg->T; p1.N = ns * cfg->H; p1.K = cfg->D; p1.epi = 0;
    p1.A = x; p1.B = w1s; p1.out = h_sh; p1.ld_out = (long long)ns * cfg->H; p1.bias = b1s; p1.bias_stride = 0;
    p1.bias_rows = 1;
  }
  return run_gemm(cfg, g, row_token ? x : x_perm, row_token ? (long long)cfg->T : R, w1, (long long)cfg->E * cfg->H,
                  x, cfg->T, w1s, (long long)ns * cfg->H, cfg->D, cfg->D, cfg->D, ws, (cudaStream_t)stream);
}

int moe_expert_gemm2(const moe_config_t* cfg, const int32_t* offsets, const void* h_perm,
                     const void* h_sh, const void* w2, const void* b2, const void* w2s,
                     const void* b2s, const float* row_gate, void* y_perm, void* y_sh,
                     void* ws, size_t ws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if ((rc = check_ws(cfg, ws, ws_bytes))) return rc;
  if (cfg->T == 0) return ok();
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(h_perm);
  REQUIRE_PTR(w2);
  REQUIRE_PTR(row_gate);
  REQUIRE_PTR(y_perm);
  OPTIONAL_PTR(b2);
  const int ns = cfg->n_shared;
  if (ns > 0) {
    REQUIRE_PTR(h_sh);
    REQUIRE_PTR(w2s);
    REQUIRE_PTR(y_sh);
    OPTIONAL_PTR(b2s);
  }
  const long long R = max_rows(cfg);
  GemmArgs g{};
  g.offsets = offsets; g.E = cfg->E; g.r_max = R; g.act = cfg->act; g.status = status_ptr(ws);
  g.b16 = is16(cfg); g.f16 = cfg->dtype == MOE_F16;
  g.nprob = ns > 0 ? 2 : 1;
  GemmProblem& p0 = g.p[0];
  p0.routed = 1; p0.N = cfg->D; p0.K = cfg->H; p0.epi = 1;
  p0.A = h_perm; p0.B = w2; p0.out = y_perm; p0.ld_out = cfg->D; p0.bias = b2; p0.bias_stride = cfg->D;
  p0.bias_rows = 1;
  p0.gate = row_gate;
  if (ns > 0) {
    // sum_j W2_j h_j over the n_s stacked W2 [n_s,D,H]: K = n_s*H walks the stack
    // (ksplit = H); the n_s rows of b2s [n_s,D] are summed in the epilogue
    GemmProblem& p1 = g.p[1];
    p1.routed = 0; p1.M = cfg->T; p1.N = cfg->D; p1.K = ns * cfg->H; p1.epi = 1;
    p1.A = h_sh; p1.B = w2s; p1.out = y_sh; p1.ld_out = cfg->D; p1.bias = b2s; p1.bias_stride = 0;
    p1.bias_rows = ns; p1.ksplit = cfg->H;
    p1.gate = nullptr;
  }
  return run_gemm(cfg, g, h_perm, R, w2, (long long)cfg->E * cfg->D, h_sh, cfg->T, w2s,
                  (long long)ns * cfg->D, cfg->H, ns * cfg->H, cfg->H, ws, (cudaStream_t)stream);
}

int moe_expert_gemm2_combine(const moe_config_t* cfg, const int32_t* offsets, const void* h_perm,
                             const void* h_sh, const void* w2, const void* b2, const void* w2s,
                             const void* b2s, const float* row_gate, const int32_t* pos, const int32_t* n_sel,
                             void* y_perm, const moe_residual_t* res, void* out, void* ws, size_t ws_bytes,
                             void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (!is16(cfg) || cfg->gemm_impl != MOE_GEMM_AUTO || cfg->n_shared < 1)
    return fail(MOE_ERR_UNSUPPORTED,
                "the combine folds into the shared experts' GEMM2 only for bf16 or fp16, gemm_impl AUTO and n_shared >= 1; "
                "use moe_expert_gemm2 + moe_combine");
  if ((rc = check_ws(cfg, ws, ws_bytes))) return rc;
  if (cfg->T == 0) return ok();
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(h_perm);
  REQUIRE_PTR(w2);
  REQUIRE_PTR(row_gate);
  REQUIRE_PTR(y_perm);
  REQUIRE_PTR(h_sh);
  REQUIRE_PTR(w2s);
  REQUIRE_PTR(pos);
  REQUIRE_PTR(out);
  OPTIONAL_PTR(b2);
  OPTIONAL_PTR(b2s);
  OPTIONAL_PTR(n_sel);
  if (cfg->routing == MOE_ROUTE_RACE && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  if ((rc = check_residual(cfg, res))) return rc;
  const int ns = cfg->n_shared;
  const long long R = max_rows(cfg);
  GemmArgs g{};
  g.offsets = offsets; g.E = cfg->E; g.r_max = R; g.act = cfg->act; g.status = status_ptr(ws);
  g.b16 = 1; g.f16 = cfg->dtype == MOE_F16;
  g.nprob = 2;
  GemmProblem& p0 = g.p[0];
  p0.routed = 1; p0.N = cfg->D; p0.K = cfg->H; p0.epi = 1;
  p0.A = h_perm; p0.B = w2; p0.out = y_perm; p0.ld_out = cfg->D; p0.bias = b2; p0.bias_stride = cfg->D;
  p0.bias_rows = 1;
  p0.gate = row_gate;
  GemmProblem& p1 = g.p[1];
  p1.routed = 0; p1.M = cfg->T; p1.N = cfg->D; p1.K = ns * cfg->H; p1.epi = 2;
  p1.A = h_sh; p1.B = w2s; p1.out = out; p1.ld_out = cfg->D; p1.bias = b2s; p1.bias_stride = 0;
  p1.bias_rows = ns; p1.ksplit = cfg->H;
  p1.gate = nullptr;
  g.pos = pos; g.n_sel = n_sel; g.kmax = kmax_of(cfg); g.kdef = cfg->K;
  g.y_routed = y_perm;
  g.done_ctr = ws_at<unsigned int>(ws, kWsDoneCtr);
  if (res) { g.x_res = res->x_res; g.alpha = res->alpha; g.img_len = res->img_len; }
  return run_gemm(cfg, g, h_perm, R, w2, (long long)cfg->E * cfg->D, h_sh, cfg->T, w2s,
                  (long long)ns * cfg->D, cfg->H, ns * cfg->H, cfg->H, ws, (cudaStream_t)stream);
}

int moe_expert_mlp(const moe_config_t* cfg, const int32_t* offsets, const void* x_perm,
                   const void* x, const void* w1, const void* b1, const void* w2, const void* b2,
                   const void* w1s, const void* b1s, const void* w2s, const void* b2s,
                   const float* row_gate, void* h_perm, void* h_sh, void* y_perm, void* y_sh,
                   void* ws, size_t ws_bytes, void* stream) {
  int rc = moe_expert_gemm1(cfg, offsets, x_perm, x, w1, b1, w1s, b1s, h_perm, h_sh, ws, ws_bytes, stream);
  if (rc) return rc;
  return moe_expert_gemm2(cfg, offsets, h_perm, h_sh, w2, b2, w2s, b2s, row_gate, y_perm, y_sh, ws, ws_bytes,
                          stream);
}

size_t moe_expert_backward_workspace_size(const moe_config_t* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return eb_layout(cfg).total;
}

int moe_expert_backward(const moe_config_t* cfg, const void* x, const void* x_perm, const int32_t* offsets,
                        const int32_t* pos, const int32_t* topk_idx, const int32_t* n_sel, const int32_t* row_token,
                        const float* row_gate, const moe_expert_weights_t* wts, const void* h_perm, const void* h_sh,
                        const void* dout, const moe_expert_grads_t* grads, float* dgate, void* dx, void* ws,
                        size_t ws_bytes, void* bws, size_t bws_bytes, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (!is16(cfg) || cfg->gemm_impl != MOE_GEMM_AUTO)
    return fail(MOE_ERR_UNSUPPORTED, "the expert backward runs on the CTA-pair tensor-core GEMM: bf16 or fp16 with "
                                     "gemm_impl AUTO");
  if (cfg->act != 0) return fail(MOE_ERR_UNSUPPORTED, "the expert backward covers the tanh-form GELU (act = 0)");
  if (!wts || !grads) return fail(MOE_ERR_INVALID_ARG, "wts and grads must be given");
  if ((rc = check_ws(cfg, ws, ws_bytes))) return rc;
  if (!bws) return fail(MOE_ERR_INVALID_ARG, "bws is NULL");
  if ((uintptr_t)bws & 255u) return fail(MOE_ERR_INVALID_ARG, "bws must be 256-byte aligned");
  const EbLayout L = eb_layout(cfg);
  if (bws_bytes < L.total) return fail(MOE_ERR_WORKSPACE, "bws_bytes=%zu < %zu", bws_bytes, L.total);
  const int ns = cfg->n_shared;
  REQUIRE_PTR(grads->dw1);
  REQUIRE_PTR(grads->dw2);
  OPTIONAL_PTR(grads->db1);
  OPTIONAL_PTR(grads->db2);
  if (ns > 0) {
    REQUIRE_PTR(grads->dws1);
    REQUIRE_PTR(grads->dws2);
    OPTIONAL_PTR(grads->dbs1);
    OPTIONAL_PTR(grads->dbs2);
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  const long long T = cfg->T, D = cfg->D, H = cfg->H, E = cfg->E, R = max_rows(cfg);
  if (T == 0) {   // no token: zero gradients
    struct { float* p; size_t n; } z[] = {{grads->dw1, (size_t)(E * H * D)}, {grads->db1, (size_t)(E * H)},
                                          {grads->dw2, (size_t)(E * D * H)}, {grads->db2, (size_t)(E * D)},
                                          {grads->dws1, (size_t)(ns * H * D)}, {grads->dbs1, (size_t)(ns * H)},
                                          {grads->dws2, (size_t)(ns * D * H)}, {grads->dbs2, (size_t)(ns * D)}};
    for (auto& q : z)
      if (q.p && q.n && (e = cudaMemsetAsync(q.p, 0, q.n * 4, s)) != cudaSuccess) return cuda_fail(e, "moe_expert_backward");
    return ok();
  }
  REQUIRE_PTR(x);
  REQUIRE_PTR(x_perm);
  REQUIRE_PTR(offsets);
  REQUIRE_PTR(pos);
  REQUIRE_PTR(topk_idx);
  OPTIONAL_PTR(n_sel);
  REQUIRE_PTR(row_token);
  REQUIRE_PTR(row_gate);
  REQUIRE_PTR(wts->w1);
  REQUIRE_PTR(wts->w2);
  OPTIONAL_PTR(wts->b1);
  OPTIONAL_PTR(wts->b2);
  REQUIRE_PTR(h_perm);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(dgate);
  REQUIRE_PTR(dx);
  if (ns > 0) {
    REQUIRE_PTR(wts->w1s);
    REQUIRE_PTR(wts->w2s);
    OPTIONAL_PTR(wts->b1s);
    REQUIRE_PTR(h_sh);
  }
  if (cfg->routing == MOE_ROUTE_RACE && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  const int f16 = cfg->dtype == MOE_F16;
  const int kmax = kmax_of(cfg);
  uint8_t* b = static_cast<uint8_t*>(bws);
  void* dout_perm = b + L.dout_perm;
  void* dz_perm = b + L.dz_perm;
  void* du_perm = b + L.du_perm;
  void* du_sh = b + L.du_sh;
  void* dx_perm = b + L.dx_perm;
  float* dg = reinterpret_cast<float*>(b + L.dg);
  float* partial = reinterpret_cast<float*>(b + L.partial);
  int* status = status_ptr(ws);

  // 1. dY in permuted order, as given and times the row's gate
  ExpertBwdArgs ea{};
  ea.dout = dout; ea.row_token = row_token; ea.row_gate = row_gate; ea.rows = R;
  ea.T = (int)T; ea.D = (int)D; ea.E = (int)E; ea.K = cfg->K; ea.Kmax = kmax; ea.f16 = f16;
  ea.dout_perm = dout_perm; ea.dz_perm = dz_perm;
  ea.pos = pos; ea.topk_idx = topk_idx; ea.n_sel = n_sel; ea.dg = dg; ea.dg_stride = L.dg_stride;
  ea.b2 = wts->b2; ea.dgate = dgate;
  if ((e = launch_bwd_gather(ea, s)) != cudaSuccess) return cuda_fail(e, "backward gather");

  auto base_args = [&](int nprob) {
    GemmArgs g{};
    g.offsets = offsets; g.E = (int)E; g.r_max = R; g.act = 0; g.status = status;
    g.b16 = 1; g.f16 = f16; g.nprob = nprob;
    return g;
  };
  const int np = ns > 0 ? 2 : 1;
  // 2. the pre-activations again: u = x W1^T + b1 (routed rows and shared block), into the dU buffers
  {
    GemmArgs g = base_args(np);
    GemmProblem& p0 = g.p[0];
    p0.routed = 1; p0.N = (int)H; p0.K = (int)D; p0.epi = 1; p0.out = du_perm; p0.ld_out = H;
    p0.bias = wts->b1; p0.bias_stride = H; p0.bias_rows = 1;
    GemmProblem& p1 = g.p[1];
    if (ns > 0) {
      p1.routed = 0; p1.M = (int)T; p1.N = ns * (int)H; p1.K = (int)D; p1.epi = 1; p1.out = du_sh;
      p1.ld_out = ns * H; p1.bias = wts->b1s; p1.bias_stride = 0; p1.bias_rows = 1;
    }
    const OperandMap A[2] = {{x_perm, R, D, 128}, {x, T, D, 128}};
    const OperandMap B[2] = {{wts->w1, E * H, D, 128}, {wts->w1s, (long long)ns * H, D, 128}};
    const OutputMap O[2] = {{du_perm, 0, 1, R, H}, {du_sh, 0, 1, T, (long long)ns * H}};
    if ((rc = launch_pair_problems(cfg, g, A, B, O, ws, s))) return rc;
  }
  // 3. dU = gate * (dY W2) * gelu'(u), written over u; the row dots sum (dY W2) gelu(u) per column
  //    tile give the gates' gradient
  {
    GemmArgs g = base_args(np);
    GemmProblem& p0 = g.p[0];
    p0.routed = 1; p0.N = (int)H; p0.K = (int)D; p0.epi = 4; p0.out = du_perm; p0.ld_out = H;
    p0.b_mn = 1; p0.aux = du_perm; p0.gate = row_gate; p0.dg = dg; p0.dg_stride = L.dg_stride;
    GemmProblem& p1 = g.p[1];
    if (ns > 0) {
      p1.routed = 0; p1.M = (int)T; p1.N = ns * (int)H; p1.K = (int)D; p1.epi = 4; p1.out = du_sh;
      p1.ld_out = ns * H; p1.b_mn = 1; p1.b_split = (int)H; p1.aux = du_sh;
    }
    const OperandMap A[2] = {{dout_perm, R, D, 128}, {dout, T, D, 128}};
    const OperandMap B[2] = {{wts->w2, E * D, H, 64}, {wts->w2s, (long long)ns * D, H, 64}};
    const OutputMap O[2] = {{du_perm, 0, 1, R, H}, {du_sh, 0, 1, T, (long long)ns * H}};
    if ((rc = launch_pair_problems(cfg, g, A, B, O, ws, s))) return rc;
  }
  // 4. dx = sum over the token's slots of (dU W1)[pos] + dU_sh W1s (combine folded into the shared tiles)
  {
    GemmArgs g = base_args(np);
    GemmProblem& p0 = g.p[0];
    p0.routed = 1; p0.N = (int)D; p0.K = (int)H; p0.epi = 1; p0.out = dx_perm; p0.ld_out = D; p0.b_mn = 1;
    p0.bias_rows = 1;
    GemmProblem& p1 = g.p[1];
    if (ns > 0) {
      p1.routed = 0; p1.M = (int)T; p1.N = (int)D; p1.K = ns * (int)H; p1.epi = 2; p1.out = dx; p1.ld_out = D;
      p1.b_mn = 1; p1.bias_rows = 1;
      g.pos = pos; g.n_sel = n_sel; g.kmax = kmax; g.kdef = cfg->K;
      g.y_routed = dx_perm;
      g.done_ctr = ws_at<unsigned int>(ws, kWsDoneCtr);
    }
    const OperandMap A[2] = {{du_perm, R, H, 128}, {du_sh, T, (long long)ns * H, 128}};
    const OperandMap B[2] = {{wts->w1, E * H, D, 64}, {wts->w1s, (long long)ns * H, D, 64}};
    const OutputMap O[2] = {{dx_perm, 0, 1, R, D}, {dx, 0, 1, T, D}};
    if ((rc = launch_pair_problems(cfg, g, A, B, O, ws, s))) return rc;
    if (ns == 0) {
      CombineArgs ca{};
      ca.y_perm = dx_perm; ca.y_sh = nullptr; ca.pos = pos; ca.n_sel = n_sel; ca.out = dx; ca.b16 = 1; ca.f16 = f16;
      ca.T = (int)T; ca.D = (int)D; ca.K = cfg->K; ca.Kmax = kmax; ca.r_max = R;
      if ((e = launch_combine(ca, s)) != cudaSuccess) return cuda_fail(e, "backward combine");
    }
  }
  // 5. dW2 = sum over the expert's rows of (g dY)^T h; dW2s_j = dY^T h_sh_j
  // 6. dW1 = sum over the expert's rows of dU^T x_perm; dW1s = dU_sh^T x
  // The shared problem (K = T reduction rows per tile, the longest tiles) goes first: the tiles
  // are claimed in order, so the last ones to start are the short routed tiles.
  for (int step = 0; step < 2; ++step) {
    GemmArgs g = base_args(np);
    GemmProblem routed{}, shared{};
    OperandMap Ar, Br, As, Bs;
    OutputMap Or, Os;
    routed.routed = 1; routed.kgrouped = 1; routed.K = 0; routed.a_mn = 1; routed.b_mn = 1; routed.out_f32 = 1;
    shared.routed = 0; shared.kgrouped = 1; shared.K = (int)T; shared.a_mn = 1; shared.b_mn = 1; shared.out_f32 = 1;
    if (step == 0) {
      routed.M = (int)D; routed.N = (int)H; routed.out = grads->dw2;
      shared.M = (int)D; shared.N = ns * (int)H; shared.out_split = (int)H; shared.out = grads->dws2;
      Ar = {dz_perm, R, D, 64}; Br = {h_perm, R, H, 64}; Or = {grads->dw2, 1, E, D, H};
      As = {dout, T, D, 64}; Bs = {h_sh, T, (long long)ns * H, 64}; Os = {grads->dws2, 1, ns, D, H};
    } else {
      routed.M = (int)H; routed.N = (int)D; routed.out = grads->dw1;
      shared.M = ns * (int)H; shared.N = (int)D; shared.out = grads->dws1;
      Ar = {du_perm, R, H, 64}; Br = {x_perm, R, D, 64}; Or = {grads->dw1, 1, E, H, D};
      As = {du_sh, T, (long long)ns * H, 64}; Bs = {x, T, D, 64}; Os = {grads->dws1, 1, 1, (long long)ns * H, D};
    }
    if (ns > 0) {
      g.p[0] = shared; g.p[1] = routed;
      const OperandMap A[2] = {As, Ar}, B[2] = {Bs, Br};
      const OutputMap O[2] = {Os, Or};
      if ((rc = launch_pair_problems(cfg, g, A, B, O, ws, s))) return rc;
    } else {
      g.p[0] = routed;
      const OperandMap A[2] = {Ar, Ar}, B[2] = {Br, Br};
      const OutputMap O[2] = {Or, Or};
      if ((rc = launch_pair_problems(cfg, g, A, B, O, ws, s))) return rc;
    }
  }
  // 7. bias gradients: column sums of g dY and dU over each expert's rows, of dY and dU_sh over all tokens
  if (grads->db2 && (e = launch_colsum(dz_perm, R, (int)D, offsets, (int)E, 1, partial, grads->db2, f16, s)) != cudaSuccess)
    return cuda_fail(e, "db2 column sums");
  if (grads->db1 && (e = launch_colsum(du_perm, R, (int)H, offsets, (int)E, 1, partial, grads->db1, f16, s)) != cudaSuccess)
    return cuda_fail(e, "db1 column sums");
  if (ns > 0 && grads->dbs2 &&
      (e = launch_colsum(dout, T, (int)D, nullptr, 1, ns, partial, grads->dbs2, f16, s)) != cudaSuccess)
    return cuda_fail(e, "dbs2 column sums");
  if (ns > 0 && grads->dbs1 &&
      (e = launch_colsum(du_sh, T, ns * (int)H, nullptr, 1, 1, partial, grads->dbs1, f16, s)) != cudaSuccess)
    return cuda_fail(e, "dbs1 column sums");
  // 8. the gates' gradient per selected slot
  if ((e = launch_dgate(ea, s)) != cudaSuccess) return cuda_fail(e, "gate gradient");
  return ok();
}

int moe_router_backward(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                        const int32_t* counts, const int32_t* topk_idx, const int32_t* n_sel, const float* dgate,
                        float aux_scale, float* dwg, float* dbias, void* dx, int32_t dx_accumulate, void* bws,
                        size_t bws_bytes, void* stream) {
  return router_backward(cfg, x, wg, router_bias, counts, topk_idx, n_sel, dgate, aux_scale, dwg, dbias, dx,
                         dx_accumulate, bws, bws_bytes, stream);
}

int moe_combine(const moe_config_t* cfg, const void* y_perm, const void* y_sh,
                const int32_t* pos, const int32_t* n_sel, const moe_residual_t* res, void* out, void* stream) {
  int rc = validate(cfg);
  if (rc) return rc;
  if (cfg->T == 0) return ok();
  REQUIRE_PTR(y_perm);
  REQUIRE_PTR(pos);
  REQUIRE_PTR(out);
  OPTIONAL_PTR(n_sel);
  if (cfg->n_shared > 0) REQUIRE_PTR(y_sh);
  if (cfg->routing == MOE_ROUTE_RACE && !n_sel) return fail(MOE_ERR_INVALID_ARG, "n_sel is required for Expert-Race routing");
  if ((rc = check_residual(cfg, res))) return rc;
  CombineArgs ca{};
  ca.y_perm = y_perm; ca.y_sh = cfg->n_shared > 0 ? y_sh : nullptr; ca.pos = pos; ca.n_sel = n_sel;
  ca.out = out; ca.b16 = is16(cfg); ca.f16 = cfg->dtype == MOE_F16;
  ca.T = cfg->T; ca.D = cfg->D; ca.K = cfg->K; ca.Kmax = kmax_of(cfg); ca.r_max = max_rows(cfg);
  if (res) { ca.x_res = res->x_res; ca.alpha = res->alpha; ca.img_len = res->img_len; }
  cudaError_t e = launch_combine(ca, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "combine kernel");
  return ok();
}

}  // extern "C"
