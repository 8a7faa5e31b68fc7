/* A plain C99 client of the ISA library, built and run by
 * tests/test_c_abi.py on a machine without a GPU.  It includes only
 * include/isa.h, takes the address of every entry point (so each one links
 * with the declared C name) and calls those that need no device: the
 * version string, the workspace sizes, the plan view of a fake workspace
 * address and the host-side argument checks.  Exit status 0 means every
 * check held; otherwise it prints the first one that failed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "isa.h"

typedef void (*any_fn)(void);

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s (%s)\n", __LINE__, \
              #cond, isa_last_error());                               \
      return 1;                                                       \
    }                                                                 \
  } while (0)

int main(void) {
  const any_fn entry_points[] = {
      (any_fn)isa_plan_workspace_size, (any_fn)isa_plan, (any_fn)isa_plan_rope, (any_fn)isa_plan_view_get,
      (any_fn)isa_forward, (any_fn)isa_dense, (any_fn)isa_forward_static,
      (any_fn)isa_forward_static_status, (any_fn)isa_backward_workspace_size, (any_fn)isa_backward, (any_fn)isa_coarse_residual,
      (any_fn)isa_coarse_residual_backward_workspace_size, (any_fn)isa_coarse_residual_backward,
      (any_fn)isa_rope_workspace_size, (any_fn)isa_rope, (any_fn)isa_last_error, (any_fn)isa_version,
      (any_fn)isa_set_wait_timeout_ns, (any_fn)isa_set_fault_injection};
  size_t i;
  for (i = 0; i < sizeof(entry_points) / sizeof(entry_points[0]); ++i) CHECK(entry_points[i] != NULL);

  CHECK(isa_version() != NULL && strstr(isa_version(), "sm_100a") != NULL);

  /* 1000 + 500 tokens in blocks of 64: T_src = 16, T_ctx = 8, K_sel =
   * ceil(0.125 * 8) = 1, T_kv = 17, n_flat = floor(0.5 * 24) = 12,
   * n_exact = ceil(0.0625 * 17) = 2 */
  isa_params p = {1, 2, 128, 1000, 500, 64, 0.125f, 0.5f, 0.0625f, 0.0f};
  size_t plan_bytes = 0, bwd_bytes = 0, rope_bytes = 0, coarse_bytes = 0;
  CHECK(isa_plan_workspace_size(&p, &plan_bytes) == ISA_OK && plan_bytes > 0);
  CHECK(isa_backward_workspace_size(&p, &bwd_bytes) == ISA_OK && bwd_bytes > 0);
  CHECK(isa_rope_workspace_size(&p, &rope_bytes) == ISA_OK && rope_bytes > 0);
  CHECK(isa_coarse_residual_backward_workspace_size(&p, &coarse_bytes) == ISA_OK);

  const uintptr_t fake_ws = (uintptr_t)1 << 20; /* never dereferenced */
  isa_plan_view v;
  memset(&v, 0, sizeof(v));
  CHECK(isa_plan_view_get(&p, (const void*)fake_ws, plan_bytes, &v) == ISA_OK);
  CHECK(v.T_src == 16 && v.T_ctx == 8 && v.T == 24 && v.K_sel == 1 && v.T_kv == 17);
  CHECK(v.n_flat == 12 && v.n_sharp == 12 && v.n_exact == 2 && v.T_kv_pad == 128 && v.bitmap_words == 1);
  CHECK((uintptr_t)v.Qc >= fake_ws && (uintptr_t)v.status < fake_ws + plan_bytes);
  CHECK(isa_plan_view_get(&p, (const void*)fake_ws, plan_bytes - 1, &v) == ISA_ERR_WORKSPACE);

  /* host-side refusals, each with a message */
  isa_params bad = p;
  bad.D = 96;
  CHECK(isa_plan_workspace_size(&bad, &plan_bytes) == ISA_ERR_UNSUPPORTED && strlen(isa_last_error()) > 0);
  bad = p;
  bad.alpha_s = 0.0f;
  CHECK(isa_plan_workspace_size(&bad, &plan_bytes) == ISA_ERR_INVALID_ARG);
  CHECK(isa_plan_workspace_size(NULL, &plan_bytes) == ISA_ERR_INVALID_ARG);
  CHECK(isa_set_fault_injection(7) == ISA_ERR_INVALID_ARG);
  CHECK(isa_set_fault_injection(0) == ISA_OK && isa_set_wait_timeout_ns(0) == ISA_OK);

  printf("c abi ok: %s, plan workspace %zu bytes\n", isa_version(), plan_bytes);
  return 0;
}
