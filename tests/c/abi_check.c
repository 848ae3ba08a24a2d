/* A plain C99 consumer of the library's C ABI: it includes the public header,
 * links libflint_attn.so and calls the entry points that need no GPU (sizes,
 * argument errors, strings). Built and run by tests/test_abi_cpu.py. */
#include <stdio.h>
#include <string.h>

#include "flint_attn.h"

static int fails = 0;
#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++fails;                                                       \
    }                                                                \
  } while (0)

int main(void) {
  flint_attn_params_t p;
  memset(&p, 0, sizeof p);
  p.total_tokens = 4096;
  p.num_docs = 2;
  p.num_q_heads = 32;
  p.num_kv_heads = 4;
  p.head_dim = 128;
  p.window = 512;
  p.use_rope = 1;
  p.rope_theta = 1e6f;
  p.rms_eps = 1e-6f;
  p.dtype = FLINT_BF16;
  CHECK(flint_attn_workspace_bytes(&p, 0) > 0);
  CHECK(flint_attn_workspace_bytes(&p, 1) > flint_attn_workspace_bytes(&p, 0));
  /* errors come back before any launch */
  CHECK(flint_attn_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
        FLINT_ERR_INVALID_ARG);
  CHECK(flint_attn_fwd_padded(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                              NULL, 0, NULL) == FLINT_ERR_INVALID_ARG);
  p.head_dim = 64;
  CHECK(flint_attn_workspace_bytes(&p, 0) == 0);

  flint_decode_params_t d;
  memset(&d, 0, sizeof d);
  d.batch = 8;
  d.cache_capacity = 1024;
  d.num_q_heads = 32;
  d.num_kv_heads = 4;
  d.head_dim = 128;
  d.window = 0;
  d.rms_eps = 1e-6f;
  d.dtype = FLINT_BF16;
  CHECK(flint_attn_decode_workspace_bytes(&d) > 0);
  d.dtype = FLINT_FP32;
  CHECK(flint_attn_decode(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                          NULL, 0, NULL) == FLINT_ERR_UNSUPPORTED);

  CHECK(flint_attn_selftest_wait(1000, 0, NULL, NULL) == FLINT_ERR_INVALID_ARG);
  CHECK(strstr(flint_attn_version(), "sm_100a") != NULL);
  CHECK(strlen(flint_status_string(FLINT_ERR_TIMEOUT)) > 0);
  if (fails == 0) printf("c abi ok\n");
  return fails == 0 ? 0 : 1;
}
