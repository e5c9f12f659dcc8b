/* Host-side use of the Prism C ABI from plain C (C11): the header compiles as
 * C, the library links and loads, and every call below returns before any
 * CUDA work (no GPU needed).  Prints "ok" and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "prism.h"

static int failures = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static prism_params grid(int T, int H, int W, int heads, int D) {
  prism_params p;
  memset(&p, 0, sizeof p);
  p.T = T; p.H = H; p.W = W; p.heads = heads; p.head_dim = D;
  p.tau128 = 0.5f; p.tau256 = 0.25f; p.eps = 1e-6f;
  p.topk_frac = 0.04f; p.top_p = 0.9f;
  return p;
}

int main(void) {
  /* the version string is "major.minor.patch" */
  const char *v = prism_version();
  int dots = 0;
  for (const char *c = v; *c; ++c) dots += *c == '.';
  CHECK(dots == 2);

  /* workspace sizes: positive for a valid grid, growing with it, 0 on bad params */
  prism_params small = grid(8, 16, 16, 1, 64), big = grid(56, 96, 160, 24, 128);
  size_t ws_small = prism_plan_workspace_size(&small), ws_big = prism_plan_workspace_size(&big);
  CHECK(ws_small > 0 && ws_big > ws_small);
  CHECK(prism_select_workspace_size(&big) > prism_select_workspace_size(&small));
  CHECK(prism_attn_workspace_size(&big, 1) > 0 && prism_attn_workspace_size(&big, 0) > 0);
  prism_params bad = grid(12, 16, 16, 1, 64);            /* T not a multiple of 8 */
  CHECK(prism_plan_workspace_size(&bad) == 0);

  /* argument errors come back as status codes with a message */
  CHECK(prism_plan(&bad, NULL, NULL, NULL, NULL, 0, NULL) == PRISM_ERR_UNSUPPORTED);
  CHECK(strstr(prism_last_error(), "multiples") != NULL);
  prism_params d96 = grid(8, 16, 16, 1, 96);
  CHECK(prism_plan(&d96, NULL, NULL, NULL, NULL, 0, NULL) == PRISM_ERR_UNSUPPORTED);
  CHECK(prism_plan(&small, NULL, NULL, NULL, NULL, 0, NULL) == PRISM_ERR_INVALID_ARG);
  CHECK(prism_plan(NULL, NULL, NULL, NULL, NULL, 0, NULL) == PRISM_ERR_INVALID_ARG);
  prism_params neg = small;
  neg.top_p = -1.0f;
  CHECK(prism_select(&neg, NULL, NULL, NULL, NULL, NULL, 0, NULL) == PRISM_ERR_INVALID_ARG);

  /* pointers are never dereferenced before the checks: dummies stand in */
  uint16_t *V = (uint16_t *)(uintptr_t)256, *V_odd = (uint16_t *)(uintptr_t)264;
  int32_t *p256 = (int32_t *)(uintptr_t)256;
  prism_plan_t plan = {(uint8_t *)p256, NULL, NULL, p256, p256, p256, NULL};
  CHECK(prism_plan(&small, V_odd, NULL, &plan, (void *)(uintptr_t)256, ws_small, NULL) == PRISM_ERR_INVALID_ARG);
  CHECK(strstr(prism_last_error(), "aligned") != NULL);
  CHECK(prism_plan(&small, V, NULL, &plan, (void *)(uintptr_t)256, ws_small - 1, NULL) == PRISM_ERR_CAPACITY);
  CHECK(prism_plan(&small, V, NULL, &plan, (void *)(uintptr_t)260, ws_small, NULL) == PRISM_ERR_INVALID_ARG);
  prism_params dens = small;
  dens.density = 3;                                      /* needs the A2V norms */
  CHECK(prism_plan(&dens, V, NULL, &plan, (void *)(uintptr_t)256, ws_small, NULL) == PRISM_ERR_INVALID_ARG);

  /* the backward requires the selection's transpose */
  prism_select_t sel = {p256, p256, 10, 0, NULL, NULL};
  size_t ws_b = prism_attn_workspace_size(&small, 1);
  CHECK(prism_attn_bwd(&small, &plan, &sel, V, V, V, V, NULL, V, (const float *)p256, V, V, V, 0,
                       0, (void *)(uintptr_t)256, ws_b, NULL) == PRISM_ERR_INVALID_ARG);
  /* and its path selector is 0 (fused) or 1 (deterministic) */
  sel.col_ptr = p256;
  sel.row = p256;
  CHECK(prism_attn_bwd(&small, &plan, &sel, V, V, V, V, NULL, V, (const float *)p256, V, V, V, 0,
                       2, (void *)(uintptr_t)256, ws_b, NULL) == PRISM_ERR_INVALID_ARG);
  CHECK(strstr(prism_last_error(), "deterministic") != NULL);

  /* a2v_norm: n = 0 is a no-op, a width that is not a multiple of 8 is refused */
  CHECK(prism_a2v_norm(V, 0, 64, 64, (float *)p256, NULL) == PRISM_OK);
  CHECK(prism_a2v_norm(V, 4, 12, 16, (float *)p256, NULL) == PRISM_ERR_INVALID_ARG);

  /* timing ids outside 0..PRISM_KERNEL_TIMING_IDS-1 are refused */
  int n = 0;
  double ms = 0.0;
  const char *name = NULL;
  CHECK(prism_kernel_timing_read(PRISM_KERNEL_TIMING_IDS, &n, &ms, &name) == PRISM_ERR_INVALID_ARG);

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
