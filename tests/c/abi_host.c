/* Host-side checks of the C ABI from plain C (no Python, no GPU): the header
 * compiles as C99, the library links, and every check that runs before a
 * launch gives the status the header documents.  No call here reaches the
 * device: each one fails (or answers) on its arguments first. */
#include <stdio.h>
#include <string.h>

#include "msign_b200.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  /* a fake device address: host-side checks never dereference it */
  void *p = (void *)(uintptr_t)256;
  msign_coeffs auto_route = {0, NULL, -1.0f, 0, 1};
  const float jordan2[6] = {3.4445f, -4.7750f, 2.0315f, 3.4445f, -4.7750f, 2.0315f};
  msign_coeffs two_steps = {2, jordan2, -1.0f, 0, 0};
  msign_coeffs bad_steps = {0, jordan2, -1.0f, 0, 0};

  CHECK(msign_abi_version() == 106);
  CHECK(strcmp(msign_status_string(MSIGN_OK), "ok") == 0);
  CHECK(strlen(msign_status_string(MSIGN_ERR_TIMEOUT)) > 0);

  /* workspace queries: zero for empty problems, growing with the batch */
  CHECK(msign_ns_workspace_size(0, 64, 64, MSIGN_BF16) == 0);
  CHECK(msign_ns_workspace_size(1, 64, 64, MSIGN_BF16) > 0);
  CHECK(msign_ns_workspace_size(2, 512, 1024, MSIGN_BF16) > msign_ns_workspace_size(1, 512, 1024, MSIGN_BF16));
  CHECK(msign_ns_workspace_size(1, 512, 1024, MSIGN_FP32) > msign_ns_workspace_size(1, 512, 1024, MSIGN_BF16));
  CHECK(msign_ns_workspace_size(1, 300, 100, MSIGN_BF16) == msign_ns_workspace_size(1, 100, 300, MSIGN_BF16));
  CHECK(gram_ns_workspace_size(1, 1024, 16384) > 0);
  {
    int64_t rows[2] = {4096, 1024}, cols[2] = {4096, 4096};
    CHECK(muon_step_workspace_size(2, rows, cols) >= muon_step_workspace_size(1, rows, cols));
  }
  CHECK(msign_ns_noalloc_max_bytes() == (size_t)32 << 20);

  /* routes: host-only queries */
  CHECK(msign_ns_route(1, 1024, 16384, MSIGN_BF16, &auto_route) == 1);
  CHECK(msign_ns_route(1, 16384, 1024, MSIGN_BF16, &auto_route) == 1);
  CHECK(msign_ns_route(1, 4096, 4096, MSIGN_BF16, &auto_route) == 0);
  CHECK(msign_ns_route(1, 1024, 16384, MSIGN_FP32, &auto_route) == 0);
  CHECK(msign_ns_route(1, 1024, 16384, MSIGN_BF16, NULL) == 0);
  CHECK(msign_ns_route(-1, 4, 4, MSIGN_BF16, NULL) == -MSIGN_ERR_INVALID_ARG);
  CHECK(muon_step_route(4096, 14336, &auto_route) == 1);
  CHECK(muon_step_route(1024, 4096, &auto_route) == 0);

  /* argument checks before any launch */
  CHECK(msign_ns(NULL, NULL, MSIGN_BF16, MSIGN_BF16, 0, 4, 4, 0, 0, NULL, NULL, 0, NULL) == MSIGN_OK);
  CHECK(msign_ns(NULL, NULL, MSIGN_BF16, MSIGN_BF16, -1, 4, 4, 0, 0, NULL, NULL, 0, NULL) == MSIGN_ERR_INVALID_ARG);
  CHECK(msign_ns(NULL, NULL, MSIGN_BF16, MSIGN_BF16, 1, 4, 4, 0, 0, NULL, NULL, 0, NULL) == MSIGN_ERR_INVALID_ARG);
  CHECK(msign_ns(p, p, MSIGN_BF16, MSIGN_BF16, 1, 4, 4, 0, 0, NULL, NULL, 0, NULL) == MSIGN_ERR_WORKSPACE);
  CHECK(msign_ns(p, p, MSIGN_BF16, MSIGN_BF16, 1, 4, 4, 0, 0, &two_steps, NULL, 0, NULL) == MSIGN_ERR_WORKSPACE);
  CHECK(msign_ns(p, p, MSIGN_BF16, MSIGN_BF16, 1, 4, 4, 0, 0, &bad_steps, NULL, 0, NULL) == MSIGN_ERR_INVALID_ARG);
  CHECK(msign_ns(p, p, MSIGN_BF16, MSIGN_BF16, 2, 4, 4, 15, 0, NULL, NULL, 0, NULL) == MSIGN_ERR_INVALID_ARG);
  CHECK(msign_ns(p, p, MSIGN_BF16, MSIGN_BF16, 70000, 4, 4, 0, 0, NULL, NULL, 0, NULL) == MSIGN_ERR_UNSUPPORTED);
  CHECK(gram_ns(p, p, MSIGN_BF16, 1, 4, 8, 0, 0, &auto_route, NULL, -1, NULL, 0, NULL) == MSIGN_ERR_INVALID_ARG);
  CHECK(gram_xxt(p, MSIGN_FP32, p, MSIGN_FP32, 1, 4, 8, NULL, 0, NULL) == MSIGN_ERR_UNSUPPORTED);
  CHECK(msign_ns_noalloc(p, p, MSIGN_BF16, 1, 2048, 2048, NULL, NULL) == MSIGN_ERR_WORKSPACE);
  CHECK(msign_ns_host(p, p, MSIGN_BF16, MSIGN_BF16, 1, 4, 4, NULL, NULL, 0, NULL) == MSIGN_ERR_WORKSPACE);
  {
    void *w[1] = {p}, *g[1] = {p};
    float *m[1] = {(float *)p};
    const void *gc[1] = {g[0]};
    int64_t rows[1] = {8}, cols[1] = {8};
    CHECK(muon_step(1, w, m, gc, rows, cols, MSIGN_BF16, MSIGN_BF16, 0.95f, 0.02f, NULL, NULL, 0, NULL) ==
          MSIGN_ERR_WORKSPACE);
    CHECK(muon_step(1, w, m, gc, rows, cols, MSIGN_FP16, MSIGN_BF16, 0.95f, 0.02f, NULL, NULL, 0, NULL) ==
          MSIGN_ERR_UNSUPPORTED);
  }
  CHECK(msign_selftest_timeout(0, NULL) == MSIGN_ERR_INVALID_ARG);

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
