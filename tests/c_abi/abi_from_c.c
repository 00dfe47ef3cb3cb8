/* Links libflce.so from plain C (no C++, no Python, no torch) and exercises
 * the entry points that need no GPU: workspace sizing, FLOP count, status
 * strings and host-side argument refusal.  Exit status 0 = all checks held. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "flce.h"

static int failures = 0;
#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                            \
    }                                                        \
  } while (0)

int main(void) {
  /* bench workload sizes: N = 4096, H = 4096, V = Vp = 128256, BF16 head */
  size_t ws = flce_workspace_size(4096, 4096, 128256, 128256, FLCE_BF16);
  size_t ws_min = flce_workspace_min_size(4096, 4096, 128256, 128256, FLCE_BF16);
  CHECK(ws > 0 && ws_min > 0 && ws_min <= ws);
  CHECK(ws < (size_t)4096 * 128256);               /* never an [N, V] buffer */
  CHECK(flce_workspace_size(10, 7, 100, 100, FLCE_BF16) == 0);   /* H % 8 != 0 */
  CHECK(flce_ce_workspace_size(4096) > 0 && flce_ce_workspace_size(-1) == 0);
  CHECK(flce_flops_fwd_bwd(4096, 4096, 128256) == 8.0 * 4096.0 * 4096.0 * 128256.0);
  CHECK(strcmp(flce_status_string(FLCE_OK), "ok") == 0);
  CHECK(strlen(flce_status_string(FLCE_ERR_BAD_LABEL)) > 0);
  /* a bad argument is refused on the host before anything touches a device */
  float loss = 0.0f, lse = 0.0f;
  CHECK(flce_forward(NULL, NULL, FLCE_BF16, NULL, 1, 8, 16, 16, -100, 0.0f, FLCE_SUM, 0, &loss,
                     &lse, NULL, 0, NULL) == FLCE_ERR_INVALID_ARG);
  CHECK(flce_ce_forward(NULL, FLCE_BF16, NULL, NULL, 4, 10, 5 /* ld < V */, -100, FLCE_SUM, 0,
                        &loss, &lse, NULL, 0, NULL) == FLCE_ERR_INVALID_ARG);
  if (failures == 0) printf("C ABI ok: workspace %zu bytes (min %zu)\n", ws, ws_min);
  return failures == 0 ? 0 : 1;
}
