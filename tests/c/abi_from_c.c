/* Uses the library from plain C99 through include/sage.h only: the header
 * must compile as C, and the host-side checks must answer without a GPU.
 * Every compute call made here is one the checks reject (the pointers are
 * fake), so nothing reaches a device.  Exit status 0 = all checks held. */
#include <stdio.h>
#include <string.h>

#include "sage.h"

static int failures = 0;

static void expect(const char* what, int got, int want) {
  if (got != want) {
    printf("FAIL %s: got %d, want %d\n", what, got, want);
    ++failures;
  }
}

int main(void) {
  void* fake = (void*)(uintptr_t)(1u << 20);
  void* odd = (void*)(uintptr_t)((1u << 20) + 8u);
  printf("version %s, v_hat layout %d\n", sage_version(), sage_v_hat_layout());
  expect("status string", strcmp(sage_status_string(SAGE_OK), "ok"), 0);
  expect("d = 96", sage_attn_fwd(fake, fake, fake, fake, 1, 2, 2, 128, 96, 0, 0.125f,
                                 SAGE_VARIANT_B, NULL), SAGE_ERR_UNSUPPORTED);
  expect("misaligned q", sage_attn_fwd(odd, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.125f,
                                       SAGE_VARIANT_8P8, NULL), SAGE_ERR_MISALIGNED);
  expect("unknown variant", sage_attn_fwd(fake, fake, fake, fake, 1, 2, 2, 128, 64, 0, 0.125f,
                                          7, NULL), SAGE_ERR_UNSUPPORTED);
  expect("empty batch", sage_attn_fwd(NULL, NULL, NULL, NULL, 0, 2, 2, 128, 64, 0, 0.125f,
                                      SAGE_VARIANT_8P8_R56, NULL), SAGE_OK);
  expect("v_r out of range", sage_quant_v_fp8(fake, 1, 2, 128, 64, 500.0f, fake, fake, NULL),
         SAGE_ERR_INVALID_ARG);
  expect("rope without tables",
         sage_smooth_quant_qkv_rope(fake, fake, NULL, NULL, fake, 1, 2, 2, 128, 64, 0.125f,
                                    448.0f, fake, fake, NULL, fake, fake, fake, NULL, NULL),
         SAGE_ERR_INVALID_ARG);
  expect("no-alloc past its scratch",
         sage_smooth_quant_qk_noalloc(fake, fake, 1, 32, 32, 32769, 128, 0.125f, fake, fake,
                                      fake, fake, fake, NULL),
         SAGE_ERR_UNSUPPORTED);
  expect("workspace of an empty problem", (int)sage_attn_workspace_bytes(0, 2, 2, 128, 64, 1), 0);
  printf("%s\n", failures ? "FAILED" : "ok");
  return failures ? 1 : 0;
}
