/* Calls libcrisp.so from plain C through include/crisp.h: status strings, workspace sizing, and
 * argument checks that refuse a call before anything is launched (no GPU needed). Prints one
 * line per check and exits non-zero on the first mismatch. */
#include <stdio.h>
#include <string.h>

#include "crisp.h"

static int fails = 0;
#define CHECK(cond, what)                          \
  do {                                             \
    if (cond) {                                    \
      printf("ok   %s\n", what);                   \
    } else {                                       \
      printf("FAIL %s\n", what);                   \
      ++fails;                                     \
    }                                              \
  } while (0)

int main(void) {
  crisp_params p;
  memset(&p, 0, sizeof p); /* rule switches 0 = CRISP */
  p.block = 128;
  p.anchors = 128;
  p.tau_proxy = 0.5f;
  p.alpha = 1.0f;
  p.gamma = 0.95f;
  p.min_blocks = 0;

  CHECK(strcmp(crisp_status_string(CRISP_OK), "CRISP_OK") == 0, "status string of CRISP_OK");
  CHECK(strcmp(crisp_status_string(CRISP_ERR_WORKSPACE), "CRISP_ERR_WORKSPACE") == 0, "status string of WORKSPACE");

  size_t small = crisp_workspace_size(1, 1, 4096, 128, &p);
  size_t big = crisp_workspace_size(32, 8, 131072, 128, &p);
  CHECK(small > 0 && big > small && big % 256 == 0, "workspace sizes grow with the shape, 256-byte multiples");
  CHECK(crisp_workspace_size(1, 1, 4096, 64, &p) == 0, "d != 128 is unsupported");
  CHECK(crisp_workspace_size(1, 1, 1000, 128, NULL) > 0, "attention alone sizes any length");

  /* refusals before any launch: fake but aligned device addresses are never dereferenced */
  void* fake = (void*)0x10000;
  void* ws = (void*)0x100000;
  crisp_index ix = {(int32_t*)0x1000, (float*)0x1000, (int32_t*)0x1000, (int32_t*)0x1000, NULL};
  CHECK(crisp_select(NULL, fake, 1, 1, 4096, 128, &p, &ix, ws, big, NULL) == CRISP_ERR_INVALID_ARG, "null q");
  CHECK(crisp_select(fake, fake, 3, 2, 4096, 128, &p, &ix, ws, big, NULL) == CRISP_ERR_UNSUPPORTED,
        "h_q not a multiple of h_kv");
  CHECK(crisp_select(fake, fake, 1, 1, 4096, 128, &p, &ix, ws, 1024, NULL) == CRISP_ERR_WORKSPACE,
        "workspace too small");
  p.route_rule = 7;
  CHECK(crisp_select(fake, fake, 1, 1, 4096, 128, &p, &ix, ws, big, NULL) == CRISP_ERR_INVALID_ARG,
        "unknown route rule");
  p.route_rule = 0;
  int32_t cu[3] = {0, 50, 512};
  CHECK(crisp_prefill_varlen(fake, fake, fake, 2, 1, 512, cu, 2, 128, &p, fake, NULL, ws, big, NULL) ==
            CRISP_ERR_UNSUPPORTED,
        "varlen sequence shorter than 128 tokens");
  CHECK(crisp_get_status(NULL, NULL) == CRISP_ERR_INVALID_ARG, "status of a null workspace");
  return fails ? 1 : 0;
}
