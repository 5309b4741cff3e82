/* A plain C consumer of the library's C ABI (include/qlora_nf4.h and
 * include/qlora_optim.h): compiled with gcc and linked against the shared
 * library, no C++ or CUDA headers.  It runs only the host-side paths that need
 * no GPU: the level table, the workspace queries, the status strings and the
 * argument checks that every entry point performs before touching a device.
 * Exit status 0 when every check holds; otherwise the failing line. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "qlora_nf4.h"
#include "qlora_optim.h"

#define CHECK(cond)                                         \
  do {                                                      \
    if (!(cond)) {                                          \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                             \
    }                                                       \
  } while (0)

int main(void) {
  /* NF4 levels: 16 ascending fp32 values, -1 .. 1, exact zero at code 7. */
  float q[16];
  nf4_levels(q);
  CHECK(q[0] == -1.0f && q[15] == 1.0f && q[7] == 0.0f);
  for (int i = 1; i < 16; ++i) CHECK(q[i] > q[i - 1]);

  /* Workspace sizes: zero tokens need none; sizes grow with M and are 256-aligned. */
  CHECK(qlora_fwd_workspace_size(0, 4096, 4096, 64) == 0);
  const size_t a = qlora_fwd_workspace_size(4096, 4096, 4096, 64);
  const size_t b = qlora_fwd_workspace_size(8192, 4096, 4096, 64);
  CHECK(a > 0 && a <= b && a % 256 == 0);
  CHECK(qlora_bwd_workspace_size(4096, 4096, 4096, 64) >= (size_t)4096 * 2 * 64 * 2 * 2);

  /* Status strings. */
  CHECK(strcmp(qlora_strerror(QLORA_OK), "ok") == 0);
  {
    const int64_t prev = qlora_set_few_token_threshold(0);
    CHECK(prev == ((int64_t)1 << 26));
    CHECK(qlora_set_few_token_threshold(prev) == 0);
  }
  for (int s = 0; s <= QLORA_ERR_INTERNAL; ++s) CHECK(qlora_strerror((qlora_status)s) != NULL);

  /* Argument checks that return before any device work. */
  void* p = (void*)(uintptr_t)256; /* 16-byte aligned, never dereferenced */
  void* odd = (void*)(uintptr_t)264;
  CHECK(nf4_quantize(p, 0, p, p, p, NULL, NULL) == QLORA_OK);             /* numel 0: no-op */
  CHECK(nf4_quantize(NULL, 64, p, p, p, NULL, NULL) == QLORA_ERR_NULL);
  CHECK(nf4_dequantize(p, p, p, -1, p, NULL) == QLORA_ERR_SHAPE);
  nf4_weight w = {(const uint8_t*)p, (const uint8_t*)p, (const float*)p, 4096, 4096};
  CHECK(qlora_linear_fwd(p, 64, w, p, p, 8, 1.0f, p, QLORA_DTYPE_BF16, p, p, 0, NULL, NULL) ==
        QLORA_ERR_SHAPE); /* r = 8 < 16 */
  nf4_weight bad = w;
  bad.k_in = 100; /* not a multiple of 64 */
  CHECK(qlora_linear_fwd(p, 64, bad, p, p, 16, 1.0f, p, QLORA_DTYPE_BF16, p, p, 0, NULL, NULL) ==
        QLORA_ERR_SHAPE);
  CHECK(qlora_linear_fwd(p, 0, w, p, p, 16, 1.0f, p, QLORA_DTYPE_BF16, p, p, 0, NULL, NULL) == QLORA_OK);
  CHECK(qlora_linear_fwd(p, 64, w, p, p, 16, 1.0f, p, 7, p, p, 0, NULL, NULL) == QLORA_ERR_DTYPE);
  CHECK(qlora_adamw8_step(p, p, p, p, p, p, 10, 1e-3f, 0.9f, 0.999f, 1e-8f, 0.0f, 0, NULL, NULL) ==
        QLORA_ERR_SHAPE); /* step 0 */
  CHECK(qlora_adamw8_step(p, p, p, p, p, p, 10, 1e-3f, 1.0f, 0.999f, 1e-8f, 0.0f, 1, NULL, NULL) ==
        QLORA_ERR_SHAPE); /* beta1 = 1 */
  CHECK(qlora_adamw8_step(p, p, p, p, p, p, 10, NAN, 0.9f, 0.999f, 1e-8f, 0.0f, 1, NULL, NULL) ==
        QLORA_ERR_SHAPE);
  CHECK(qlora_adamw8_step(p, p, p, p, p, p, 0, 1e-3f, 0.9f, 0.999f, 1e-8f, 0.0f, 1, NULL, NULL) == QLORA_OK);
  CHECK(qlora_adamw8_step(NULL, p, p, p, p, p, 10, 1e-3f, 0.9f, 0.999f, 1e-8f, 0.0f, 1, NULL, NULL) ==
        QLORA_ERR_NULL);
  CHECK(qlora_adamw8_step(odd, p, p, p, p, p, 10, 1e-3f, 0.9f, 0.999f, 1e-8f, 0.0f, 1, NULL, NULL) ==
        QLORA_ERR_ALIGN);
  /* LoRA dropout: p outside [0, 1) and a missing X_drop are rejected first. */
  CHECK(qlora_linear_fwd_dropout(p, 64, w, p, p, 16, 1.0f, 1.0f, 7u, p, p, QLORA_DTYPE_BF16, p, p, 1u << 20, NULL,
                                 NULL) == QLORA_ERR_SHAPE);
  CHECK(qlora_linear_fwd_dropout(p, 64, w, p, p, 16, 1.0f, 0.05f, 7u, NULL, p, QLORA_DTYPE_BF16, p, p, 1u << 20,
                                 NULL, NULL) == QLORA_ERR_NULL);
  CHECK(qlora_linear_bwd_dropout(p, p, p, 64, w, p, p, 16, 1.0f, -0.5f, 7u, p, QLORA_DTYPE_BF16, p, p, p, 1u << 20,
                                 NULL, NULL) == QLORA_ERR_SHAPE);
  CHECK(qlora_bwd_dropout_workspace_size(4096, 4096, 4096, 64) ==
        qlora_bwd_workspace_size(4096, 4096, 4096, 64) + (size_t)4096 * 4096 * 4);
  /* Allocation-free forward: the forward's checks, then the fixed-scratch limit. */
  nf4_weight w128 = {(const uint8_t*)p, (const uint8_t*)p, (const float*)p, 128, 128};
  CHECK(qlora_linear_fwd_noalloc(p, 70000, w128, p, p, 64, 0.25f, p, QLORA_DTYPE_BF16, p, NULL, NULL) ==
        QLORA_ERR_WORKSPACE);
  CHECK(qlora_linear_fwd_noalloc(p, 64, w, p, p, 8, 0.25f, p, QLORA_DTYPE_BF16, p, NULL, NULL) == QLORA_ERR_SHAPE);
  CHECK(qlora_linear_fwd_noalloc(p, 0, w, p, p, 16, 0.25f, p, 7, p, NULL, NULL) == QLORA_ERR_DTYPE);
  /* Mean-centred double quantisation: argument checks. */
  CHECK(nf4_centered_workspace_size(0) == 0);
  CHECK(nf4_quantize_centered(p, 64, p, p, p, NULL, p, 1u << 20, NULL, NULL) == QLORA_ERR_NULL);
  CHECK(nf4_quantize_centered(p, 64, p, p, p, p, p, 16, NULL, NULL) == QLORA_ERR_WORKSPACE);
  CHECK(nf4_dequantize_centered(p, p, p, NULL, 64, p, NULL) == QLORA_ERR_NULL);
  /* Bounded-wait self-test: argument checks only (no device here). */
  CHECK(qlora_selftest_timeout(NULL, 5000000, NULL) == QLORA_ERR_NULL);
  CHECK(qlora_selftest_timeout(p, 10, NULL) == QLORA_ERR_SHAPE);
  CHECK(qlora_paged_alloc(NULL, 16) == QLORA_ERR_NULL);
  CHECK(qlora_paged_free(NULL) == QLORA_OK);
  printf("c abi consumer ok\n");
  return 0;
}
