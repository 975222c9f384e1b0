/* A plain C99 host program against include/mla_api.h: it links the library and calls
 * the entry points that need no GPU (version, status strings, cache accounting, the fixed
 * pair sets and argument validation), printing one line per check.  Built and run by
 * tests/test_abi_cpu.py. */
#include <stdio.h>
#include <string.h>

#include "mla_api.h"

static int fails = 0;
#define CHECK(cond, what)                          \
  do {                                             \
    if (cond) {                                    \
      printf("ok   %s\n", what);                   \
    } else {                                       \
      printf("FAIL %s\n", what);                   \
      ++fails;                                     \
    }                                              \
  } while (0)

int main(void) {
  mla_config_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.hidden = 4096; cfg.n_heads = 32; cfg.n_kv_heads = 32; cfg.head_dim = 128; cfg.r_pairs = 4;
  cfg.d_c = 256; cfg.rope_base = 10000.0; cfg.dtype = MLA_BF16; cfg.cache_kind = MLA_CACHE_SAME;

  CHECK(strstr(mla_version(), "sm_100a") != NULL, "version names sm_100a");
  CHECK(strcmp(mla_status_string(MLA_OK), "ok") == 0, "status string of MLA_OK");
  CHECK(mla_cache_bytes_per_token(&cfg) == 256 * 2 + 32 * 8 * 2, "bf16 cache bytes per token");
  cfg.cache_kind = MLA_CACHE_INT4_G32; cfg.d_c = 128;
  CHECK(mla_cache_bytes_per_token(&cfg) == 64 + 8 + 512, "int4 cache bytes per token");
  cfg.cache_kind = MLA_CACHE_INT2_G32;
  CHECK(mla_cache_bytes_per_token(&cfg) == 32 + 8 + 512, "int2 cache bytes per token");
  cfg.cache_kind = MLA_CACHE_SAME; cfg.d_c = 256;

  cfg.softmax_scale = -1.0f;
  CHECK(mla_cache_bytes_per_token(&cfg) == 0, "a negative softmax scale is an invalid config");
  cfg.softmax_scale = 0.0f;

  int32_t pairs[32 * 4];
  CHECK(mla_fixed_pairs(&cfg, MLA_PAIRS_HIGH, pairs) == MLA_OK && pairs[0] == 0 && pairs[3] == 3,
        "high-frequency pair set");
  CHECK(mla_fixed_pairs(&cfg, MLA_PAIRS_UNIFORM, pairs) == MLA_OK && pairs[1] == 16 && pairs[3] == 48,
        "uniform pair set (P = 64, r = 4)");
  CHECK(mla_fixed_pairs(&cfg, 42, pairs) == MLA_ERR_INVALID_ARG, "unknown strategy refused");

  mla_plan_t* plan = NULL;
  CHECK(mla_plan_create(&cfg, NULL, NULL, NULL, NULL, NULL, &plan) == MLA_ERR_INVALID_ARG && plan == NULL,
        "plan without weights refused");
  mla_cache_t cache;
  memset(&cache, 0, sizeof cache);
  CHECK(mla_append(NULL, NULL, NULL, NULL, 1, &cache, NULL) == MLA_ERR_INVALID_ARG, "append without a plan");
  CHECK(mla_decode(NULL, &cache, NULL, NULL, 1, NULL, NULL, 0, NULL) == MLA_ERR_INVALID_ARG,
        "decode without a plan");
  CHECK(mla_decode_noalloc(NULL, &cache, NULL, NULL, 1, NULL, NULL) == MLA_ERR_INVALID_ARG,
        "no-alloc decode without a plan");
  CHECK(mla_decode_workspace_bytes(NULL, 4) == 0, "workspace of no plan");
  printf("%d failed\n", fails);
  return fails ? 1 : 0;
}
