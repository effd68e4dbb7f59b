/* Host-only use of the C ABI from plain C (no CUDA headers, no GPU): create a handle,
 * validate well-formed and malformed calls, read back the plan and the configuration,
 * and release it. Prints one line per check and exits non-zero on the first failure.
 * The device pointers are never dereferenced on the host: validation only inspects their
 * values (alignment, overlap), so aligned dummy addresses stand in for device memory. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fused_norm.h"

static int failures = 0;

static void check(int ok, const char* what) {
  printf("%s %s\n", ok ? "ok  " : "FAIL", what);
  if (!ok) ++failures;
}

/* Disjoint, 16-byte aligned dummy addresses for each tensor of a (B, L, D) problem. */
static void fill_args(fn_args* a, int64_t B, int64_t L, int64_t D) {
  const uintptr_t base = (uintptr_t)1 << 40;
  const uintptr_t span = (uintptr_t)(B * L * D * 2 + 4096);
  memset(a, 0, sizeof(*a));
  a->B = B;
  a->L = L;
  a->x.ptr = (const void*)(base + 0 * span);
  a->x.stride_b = L * D;
  a->x.stride_l = D;
  a->residual = a->x;
  a->residual.ptr = (const void*)(base + 1 * span);
  a->gate.ptr = (const void*)(base + 2 * span);   /* (1, D) broadcast: strides 0 */
  a->scale = a->x;
  a->scale.ptr = (const void*)(base + 3 * span);
  a->shift = a->x;
  a->shift.ptr = (const void*)(base + 4 * span);
  a->y = (void*)(base + 5 * span);
  a->y_stride_b = L * D;
  a->y_stride_l = D;
  a->r = (void*)(base + 6 * span);
  a->r_stride_b = L * D;
  a->r_stride_l = D;
}

int main(void) {
  fn_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.D = 5120;
  cfg.has_gate = 1;
  cfg.eps = 1e-6;

  fused_norm_t h = NULL;
  check(fused_norm_create(&h, &cfg) == FN_OK && h != NULL, "create LayerNorm, gate, D=5120");

  fn_config back;
  check(fused_norm_get_config(h, &back) == FN_OK && back.D == 5120 && back.has_gate == 1 &&
            back.eps == 1e-6, "get_config returns the configuration");

  fn_args a;
  fill_args(&a, 1, 176400, 5120);
  check(fused_norm_validate(h, &a) == FN_OK, "validate the WAN2.2 shape");

  int64_t grid = 0;
  int block = 0;
  size_t smem = 1;
  check(fused_norm_plan(h, &a, &grid, &block, &smem) == FN_OK && grid == 176400 &&
            block > 0 && block % 32 == 0 && smem == 0, "plan: one CTA per row, whole warps");

  fn_args bad = a;
  bad.x.ptr = (const void*)((uintptr_t)a.x.ptr + 2);
  check(fused_norm_validate(h, &bad) == FN_ERR_MISALIGNED, "misaligned x is rejected");

  bad = a;
  bad.gate.ptr = NULL;
  check(fused_norm_validate(h, &bad) == FN_ERR_INVALID_ARG, "missing gate is rejected");

  bad = a;
  bad.r = a.y;
  check(fused_norm_validate(h, &bad) == FN_ERR_INVALID_ARG, "r overlapping y is rejected");

  bad = a;
  bad.tokens_per_frame = 11;  /* 176400 = 2^4 3^2 5^2 7^2: 11 does not divide it */
  check(fused_norm_validate(h, &bad) == FN_ERR_INVALID_ARG, "frame length not dividing L is rejected");

  bad = a;
  bad.B = 0;
  check(fused_norm_validate(h, &bad) == FN_OK, "an empty problem is valid");
  check(fused_norm_launch(h, &bad, NULL) == FN_OK, "launching an empty problem is a no-op");

  fn_config wrong = cfg;
  wrong.D = 4096;
  fused_norm_t h2 = NULL;
  check(fused_norm_create(&h2, &wrong) == FN_ERR_UNSUPPORTED && h2 == NULL, "D=4096 is unsupported");

  check(strlen(fused_norm_status_string(FN_ERR_MISALIGNED)) > 0, "status strings");
  check(fused_norm_version() > 0, "version");
  check(fused_norm_destroy(h) == FN_OK && fused_norm_destroy(NULL) == FN_OK, "destroy");

  printf("%d failure(s)\n", failures);
  return failures ? 1 : 0;
}
