/* Plain-C client of pi_attn.h: compiles as C11 against the header alone and
 * links libpiattn.so; exercises only host-side paths (no device memory is
 * touched), so it runs without a GPU.  Exit status 0 = every check held. */
#include <stdio.h>
#include <string.h>

#include "pi_attn.h"

static int failures = 0;
#define CHECK(cond)                                                    \
  do {                                                                 \
    if (!(cond)) {                                                     \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                      \
    }                                                                  \
  } while (0)

int main(void) {
  pi_attn_desc d;
  memset(&d, 0, sizeof(d));
  d.B = 2; d.Sq = 16; d.P = 0; d.Hq = 8; d.Hkv = 1; d.d = 256;
  d.dtype = PI_BF16; d.softmax_scale = 1.0f; d.mask_batch_stride = 0;

  /* argument errors are reported before anything is launched */
  CHECK(pi_attn_prefill(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == PI_ERR_ARG);
  CHECK(pi_attn_prefill(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == PI_ERR_ARG);
  d.d = 128;
  CHECK(pi_attn_prefill(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == PI_ERR_UNSUPPORTED);
  d.d = 256;

  /* empty problems are no-ops */
  d.B = 0;
  CHECK(pi_attn_prefill(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == PI_OK);
  d.B = 2;

  /* workspace queries are host-only */
  /* bf16, one KV head, d = 256: D (fp32 per row) and the bf16 P / dS tiles */
  CHECK(pi_attn_prefill_backward_workspace_bytes(&d) == 2 * 128 * 4 + 2 * (2 * 128 * 64 * 2));
  /* the split prefill: scratch for bf16 with a batch-shared mask only */
  CHECK(pi_attn_prefill_tail_splits(&d) >= 1);
  d.dtype = PI_F32;
  CHECK(pi_attn_prefill_workspace_bytes(&d) == 0);
  d.dtype = PI_BF16;
  CHECK(pi_attn_prefill_ws(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
        PI_ERR_ARG);
  d.P = 816; d.Sq = 51; d.B = 1;
  (void)pi_attn_suffix_workspace_bytes(&d);
  CHECK(pi_attn_suffix_noalloc_capacity() > 0);

  /* the status strings and the wait bound */
  CHECK(strlen(pi_attn_status_string(PI_OK)) > 0);
  CHECK(strlen(pi_attn_status_string(PI_ERR_TIMEOUT)) > 0);
  {
    const uint64_t prev = pi_attn_set_wait_limit(1000);
    CHECK(pi_attn_set_wait_limit(prev) == 1000);
  }

  /* the steps around the attention */
  {
    pi_rope_desc r;
    memset(&r, 0, sizeof(r));
    r.B = 1; r.S = 4; r.Hq = 8; r.Hkv = 1; r.d = 250; r.dtype = PI_BF16; r.base = 10000.f;
    CHECK(pi_rope_inplace(&r, NULL, NULL, NULL, NULL, NULL, NULL) == PI_ERR_UNSUPPORTED);
    CHECK(pi_euler_update(NULL, NULL, PI_F32, 0.1f, 0, NULL) == PI_OK);
    CHECK(pi_euler_update(NULL, NULL, 7, 0.1f, 16, NULL) == PI_ERR_UNSUPPORTED);
  }

  if (failures) return 1;
  printf("c abi ok\n");
  return 0;
}
