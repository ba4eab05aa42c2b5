/* A plain C consumer of include/moe.h: builds with gcc, links libmoe.so, and exercises
 * the host-side parts of the ABI (version, sizes, argument validation) without a GPU. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int failures = 0;
#define CHECK(cond, what)                                   \
  do {                                                      \
    if (!(cond)) {                                          \
      printf("FAIL: %s (%s)\n", what, moe_last_error());   \
      ++failures;                                           \
    }                                                       \
  } while (0)

int main(void) {
  moe_config_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.T = 32768; cfg.D = 1152; cfg.H = 4608; cfg.E = 8; cfg.K = 2; cfg.n_shared = 2;
  cfg.dtype = MOE_BF16; cfg.routing = MOE_ROUTE_TOPK; cfg.alpha = 0.01f; cfg.act = 0;
  cfg.gemm_impl = MOE_GEMM_AUTO; cfg.seq_len = 0;

  CHECK(moe_version() > 0, "version");
  CHECK(moe_max_rows(&cfg) == 67584, "R_max = round_up(K*T + 255*E, 256)");
  const size_t ws = moe_workspace_size(&cfg);
  CHECK(ws > 256 && ws % 256 == 0, "workspace size");
  CHECK(moe_backward_workspace_size(&cfg) > 0, "backward workspace size");

  /* invalid configurations: size functions return 0 / -1, calls fail before any launch */
  moe_config_t bad = cfg;
  bad.K = 9;
  CHECK(moe_workspace_size(&bad) == 0 && moe_max_rows(&bad) < 0, "K > E rejected");
  CHECK(moe_route(&bad, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == MOE_ERR_INVALID_ARG, "route: K > E");
  bad = cfg;
  bad.D = 1000;
  CHECK(moe_route(&bad, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == MOE_ERR_UNSUPPORTED, "route: D % 64");

  /* null and misaligned pointers */
  void* fake = (void*)(uintptr_t)(1ull << 40);
  int32_t* fi = (int32_t*)fake;
  float* ff = (float*)fake;
  CHECK(moe_route(&cfg, fake, fake, 0, fi, ff, 0, fi, 0, 0, fake, ws, 0) == MOE_ERR_INVALID_ARG, "route: aux NULL");
  CHECK(moe_route(&cfg, (char*)fake + 8, fake, 0, fi, ff, 0, fi, ff, 0, fake, ws, 0) == MOE_ERR_INVALID_ARG,
        "route: x misaligned");
  CHECK(moe_route(&cfg, fake, fake, 0, fi, ff, 0, fi, ff, 0, fake, ws - 256, 0) == MOE_ERR_WORKSPACE,
        "route: workspace too small");
  CHECK(moe_combine(&cfg, 0, fake, fi, 0, 0, fake, 0) == MOE_ERR_INVALID_ARG, "combine: y_perm NULL");

  /* the fused forms refuse what they do not cover */
  moe_config_t f32 = cfg;
  f32.dtype = MOE_F32;
  CHECK(moe_expert_gemm2_combine(&f32, fi, fake, fake, fake, 0, fake, 0, ff, fi, 0, fake, 0, fake, fake,
                                 moe_workspace_size(&f32), 0) == MOE_ERR_UNSUPPORTED, "fused combine: fp32");
  CHECK(moe_expert_gemm1_gather(&f32, fi, fi, fake, fake, 0, fake, 0, fake, fake, fake,
                                moe_workspace_size(&f32), 0) == MOE_ERR_UNSUPPORTED, "gather: fp32");
  CHECK(strlen(moe_last_error()) > 0, "message on failure");

  /* the balance-loss statistics and the loss from summed statistics */
  double* fd = (double*)fake;
  CHECK(moe_balance_stats(&cfg, fi, fake, ws, 0, 0) == MOE_ERR_INVALID_ARG, "stats: stats NULL");
  CHECK(moe_balance_stats(&cfg, fi, fake, ws - 256, fd, 0) == MOE_ERR_WORKSPACE, "stats: workspace too small");
  CHECK(moe_balance_loss_from_stats(&cfg, fd, -1, ff, 0) == MOE_ERR_INVALID_ARG, "loss from stats: T_total < 0");
  CHECK(moe_balance_loss_from_stats(&cfg, fd, 65536, 0, 0) == MOE_ERR_INVALID_ARG, "loss from stats: aux NULL");

  if (failures == 0) printf("c abi ok\n");
  return failures == 0 ? 0 : 1;
}
