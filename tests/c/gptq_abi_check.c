/* Plain C99 client of the library's C ABI: compiles against include/gptq.h alone, links
 * libgptq_b200.so, and exercises the calls that complete on the host (sizes, status names,
 * argument checks), so it needs no GPU. Prints "ok" and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "gptq.h"

static int failures = 0;

static void check(int cond, const char* what) {
  if (!cond) {
    printf("FAIL: %s\n", what);
    ++failures;
  }
}

int main(void) {
  gptq_params p;
  memset(&p, 0, sizeof p); /* static_groups = 0 by zero-initialisation, as documented */
  p.bits = 4;
  p.group_size = 128;
  p.sym = 0;
  p.order = GPTQ_ORDER_NATURAL;
  p.block_size = 128;
  p.percdamp = 0.01f;

  const size_t ws = gptq_workspace_size(4096, 4096, &p);
  check(ws == (size_t)2 * 4096 * 4096 * 4, "workspace of a natural-order 4096 x 4096 layer");
  p.order = GPTQ_ORDER_DESC_ACT;
  check(gptq_workspace_size(4096, 4096, &p) == ws + (size_t)4096 * 4096 + (size_t)4096 * 4,
        "act-order adds the sweep-order codes and the inverse permutation");
  p.order = GPTQ_ORDER_NATURAL;
  p.bits = 5;
  check(gptq_workspace_size(4096, 4096, &p) == 0, "5-bit codes are rejected");
  p.bits = 4;

  check(gptq_status_string(GPTQ_OK) != NULL && gptq_status_string(GPTQ_ERR_NOT_SPD) != NULL &&
            gptq_status_string(12345) != NULL,
        "status names exist for known and unknown codes");

  /* Never dereferenced: every call below fails a host-side check before anything launches. */
  float* fake_f = (float*)(uintptr_t)0x1000;
  const void* fake_v = (const void*)(uintptr_t)0x1000;
  check(gptq_hessian_accumulate(NULL, 64, 64, fake_v, GPTQ_BF16, 10, 64, 2.0f, 0, NULL, NULL) ==
            GPTQ_ERR_INVALID_ARG,
        "hessian: null H");
  check(gptq_hessian_accumulate(fake_f, 64, 64, fake_v, 7, 10, 64, 2.0f, 0, NULL, NULL) ==
            GPTQ_ERR_UNSUPPORTED,
        "hessian: unknown dtype");
  check(gptq_prepare_hinv(fake_f, 64, &p, fake_f, NULL, (uint8_t*)fake_f, NULL, 0, NULL, NULL) ==
            GPTQ_ERR_INVALID_ARG,
        "prepare: null perm");
  const uint32_t* fake_q = (const uint32_t*)(uintptr_t)0x1000;
  const uint16_t* fake_h = (const uint16_t*)(uintptr_t)0x1000;
  check(gptq_dequant_gemv(fake_q, 64, 100, 4, fake_h, fake_h, 1, -1, NULL, fake_h, 1, 104,
                          fake_f, 64, NULL) == GPTQ_ERR_INVALID_ARG,
        "gemv: d_in not a multiple of 32");
  check(gptq_dequant_gemv(fake_q, 64, 128, 4, fake_h, fake_h, 1, -1, NULL, fake_h, 9, 128,
                          fake_f, 64, NULL) == GPTQ_ERR_INVALID_ARG,
        "gemv: batch above 8");

  check(gptq_dequant_gemm(fake_q, 64, 192, fake_h, fake_h, 1, -1, fake_h, 16, 192, fake_f, 64,
                          NULL, NULL) == GPTQ_ERR_INVALID_ARG,
        "dequant gemm: d_in not a multiple of 128");
  check(gptq_dequant_gemm(fake_q, 64, 256, fake_h, fake_h, 4, 64, fake_h, 16, 256, fake_f, 64,
                          NULL, NULL) == GPTQ_ERR_INVALID_ARG,
        "dequant gemm: groups of 64 columns");

  check(gptq_gemm_f32(8, 8, 8, 1.0f, fake_f, 8, 0, fake_f, 8, 0, 0.0f, NULL, 8, NULL, NULL) ==
            GPTQ_ERR_INVALID_ARG,
        "gemm: null C");
  check(gptq_gemm_f32(8, 8, 8, 1.0f, fake_f, 4, 0, fake_f, 8, 0, 0.0f, fake_f, 8, NULL, NULL) ==
            GPTQ_ERR_INVALID_ARG,
        "gemm: lda shorter than a row of A");

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
