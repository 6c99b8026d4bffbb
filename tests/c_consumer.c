/*
 * A plain C99 user of the library: includes only include/tiled_attention.h, links
 * libtiled_attention.so, and exercises the calls that finish on the host (error texts, workspace
 * sizes, argument validation).  Every attn_* call below returns during argument checking, before
 * any device work, so it runs on a machine without a GPU.  Prints "OK" and exits 0 when every
 * check holds.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "tiled_attention.h"

static int fails = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      printf("FAIL line %d: %s\n", __LINE__, #cond);             \
      ++fails;                                                   \
    }                                                            \
  } while (0)

int main(void) {
  /* a 16-byte aligned, non-null address that validation rejects or never reaches */
  void* fake = (void*)(uintptr_t)(1u << 20);
  void* odd = (void*)(uintptr_t)((1u << 20) + 8u);
  int code;
  size_t ws;

  for (code = ATTN_OK; code >= ATTN_ERR_TIMEOUT; --code) {
    const char* s = attn_error_string(code);
    CHECK(s != NULL && strlen(s) > 0);
  }
  CHECK(strstr(attn_error_string(-99), "unknown") != NULL);
  CHECK(attn_last_cuda_error() != NULL);

  /* workspace: none for the exact mode; the 8-bit modes hold codes, scales, mean, bias, partials */
  CHECK(attn_workspace_bytes(4, 32, 32, 4096, 128, ATTN_MODE_BF16_EXACT) == 0);
  ws = attn_workspace_bytes(2, 32, 8, 8192, 128, ATTN_MODE_INT8_QK);
  CHECK(ws >= (size_t)2 * 32 * 8192 * 128 + (size_t)2 * 8 * 8192 * 128);
  CHECK(attn_workspace_bytes(2, 32, 8, 8192, 128, ATTN_MODE_FP8_QK) > 0);
  CHECK(attn_workspace_bytes(1, 3, 2, 128, 128, ATTN_MODE_INT8_QK) == 0); /* Hq % Hkv != 0 */
  CHECK(attn_decode_workspace_bytes(8, 32, 8, 1, 32768, 128, 148) > 0);
  CHECK(attn_decode_workspace_bytes(8, 32, 8, 1, 32768, 64, 148) == 0); /* decode needs d = 128 */

  /* attn_fwd argument errors */
  CHECK(attn_fwd(NULL, fake, fake, fake, NULL, 1, 2, 2, 128, 64, 0, 0.125f, ATTN_MODE_BF16_EXACT, ATTN_BF16,
                 NULL, 0, NULL) == ATTN_ERR_ARG);
  CHECK(attn_fwd(fake, fake, fake, fake, NULL, 1, 3, 2, 128, 64, 0, 0.125f, ATTN_MODE_BF16_EXACT, ATTN_BF16,
                 NULL, 0, NULL) == ATTN_ERR_ARG);
  CHECK(attn_fwd(fake, fake, fake, fake, NULL, 1, 2, 2, 128, 64, 0, (float)NAN, ATTN_MODE_BF16_EXACT,
                 ATTN_BF16, NULL, 0, NULL) == ATTN_ERR_ARG);
  CHECK(attn_fwd(fake, fake, fake, fake, NULL, 1, 2, 2, 128, 96, 0, 0.125f, ATTN_MODE_BF16_EXACT, ATTN_BF16,
                 NULL, 0, NULL) == ATTN_ERR_UNSUPPORTED);
  CHECK(attn_fwd(odd, fake, fake, fake, NULL, 1, 2, 2, 128, 64, 0, 0.125f, ATTN_MODE_BF16_EXACT, ATTN_BF16,
                 NULL, 0, NULL) == ATTN_ERR_ALIGN);
  CHECK(attn_fwd(fake, fake, fake, fake, NULL, 1, 2, 2, 128, 64, 0, 0.125f, ATTN_MODE_INT8_QK, ATTN_BF16,
                 NULL, 0, NULL) == ATTN_ERR_WORKSPACE);

  /* the other entry points reject bad arguments on the host too */
  CHECK(attn_fwd_host(NULL, fake, fake, fake, NULL, fake, fake, fake, fake, NULL, 1, 2, 2, 128, 64, 0, 0.125f,
                      ATTN_MODE_BF16_EXACT, ATTN_BF16, NULL, 0, NULL) == ATTN_ERR_ARG);
  CHECK(attn_fwd_prefix_masked(fake, fake, fake, fake, NULL, 1, 2, 2, 128, 256, 64, NULL, 0.125f, ATTN_BF16,
                               NULL) == ATTN_ERR_ARG);
  CHECK(attn_decode(fake, fake, fake, NULL, fake, NULL, 1, 2, 2, 1, 256, 128, 2, 0.125f, ATTN_BF16, 8, fake,
                    1u << 20, NULL) == ATTN_ERR_ARG);
  CHECK(attn_decode(fake, fake, fake, NULL, fake, NULL, 1, 2, 2, 1, 256, 64, 0, 0.125f, ATTN_BF16, 8, fake,
                    1u << 20, NULL) == ATTN_ERR_UNSUPPORTED);
  CHECK(attn_test_wait_timeout(0, NULL) == ATTN_ERR_ARG);

  printf(fails ? "FAILED (%d)\n" : "OK\n", fails);
  return fails != 0;
}
