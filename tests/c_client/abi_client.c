/* A plain C99 client of include/attn.h: the header must compile as C and the
 * library must link and answer through the C ABI alone (no Python, no C++).
 * It makes no call that needs a GPU: argument checks happen on the host. */
#include <stdio.h>
#include <stddef.h>

#include "attn.h"

static int expect(const char* what, int got, int want) {
  if (got != want) {
    printf("FAIL %s: got %d (%s), want %d\n", what, got, attn_status_string(got), want);
    return 1;
  }
  printf("ok   %s: %s\n", what, attn_status_string(got));
  return 0;
}

int main(void) {
  int bad = 0;
  char* p = (char*)(uintptr_t)(1u << 20); /* a 16-byte aligned dummy address, never dereferenced */
  /* null query pointer */
  bad += expect("attn_fwd null q",
                attn_fwd(NULL, p, p, p, NULL, 1, 8, 2, 64, 64, 128, 1, 0.088f, NULL), ATTN_ERR_INVALID_ARG);
  /* head dim without a kernel */
  bad += expect("attn_fwd d=96", attn_fwd(p, p, p, p, NULL, 1, 8, 2, 64, 64, 96, 1, 0.088f, NULL),
                ATTN_ERR_UNSUPPORTED);
  /* empty batch: a no-op */
  bad += expect("attn_fwd B=0", attn_fwd(p, p, p, p, NULL, 0, 8, 2, 64, 64, 128, 1, 0.088f, NULL), ATTN_OK);
  /* only 16-token blocks */
  bad += expect("paged_attn_decode block_size=32",
                paged_attn_decode(p, p, p, (const int32_t*)p, (const int32_t*)p, 2, 32, 8, 128, 32, 8, 0, p, NULL),
                ATTN_ERR_UNSUPPORTED);
  bad += expect("paged_attn_decode_fp8 k_scale=0",
                paged_attn_decode_fp8(p, p, p, (const int32_t*)p, (const int32_t*)p, 2, 32, 8, 128, 16, 8, 0,
                                      0.0f, 1.0f, p, NULL),
                ATTN_ERR_INVALID_ARG);
  /* context-parallel halves: a missing lse output, a merge of zero partials */
  bad += expect("paged_attn_decode_partial null lse_part",
                paged_attn_decode_partial(p, p, p, (const int32_t*)p, (const int32_t*)p, 2, 32, 8, 128, 16, 8, 64, 0,
                                          (float*)p, NULL, NULL),
                ATTN_ERR_INVALID_ARG);
  bad += expect("attn_lse_merge R=0", attn_lse_merge((const float*)p, (const float*)p, 0, 2, 32, 128, p, NULL),
                ATTN_ERR_INVALID_ARG);
  printf("attn_check_support(0) = %d (%s)\n", attn_check_support(0), attn_status_string(attn_check_support(0)));
  return bad;
}
