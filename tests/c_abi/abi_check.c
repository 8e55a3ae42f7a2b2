/* Plain-C client of the library: include/moe.h must compile as C11 and the shared
 * library must link and answer its host-only entry points without a GPU.  Prints one
 * line per check and exits non-zero on the first failure. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int fails = 0;
#define CHECK(cond, what)                                  \
  do {                                                     \
    if (cond) {                                            \
      printf("ok   %s\n", what);                           \
    } else {                                               \
      printf("FAIL %s\n", what);                           \
      fails++;                                             \
    }                                                      \
  } while (0)

int main(void) {
  moe_config c;
  memset(&c, 0, sizeof c);
  c.T = 128;
  c.d_model = 7168;
  c.E = 256;
  c.top_k = 8;
  c.d_ff = 2048;
  c.n_shared = 1;
  c.d_ff_shared = 2048;
  c.score = MOE_SCORE_SIGMOID_BIAS;
  c.act = MOE_BF16;
  c.weight = MOE_BF16;
  c.out = MOE_BF16;

  size_t bytes = 0;
  CHECK(moe_workspace_size(&c, &bytes) == MOE_OK && bytes > 0, "workspace size of the R1 decode layer");
  CHECK(moe_workspace_size(&c, NULL) == MOE_ERR_INVALID_ARG, "null size pointer rejected");

  moe_config bad = c;
  bad.top_k = 17;
  CHECK(moe_workspace_size(&bad, &bytes) == MOE_ERR_UNSUPPORTED, "top_k > 16 rejected");
  bad = c;
  bad.d_model = 7000;
  CHECK(moe_workspace_size(&bad, &bytes) == MOE_ERR_UNSUPPORTED, "d_model % 128 rejected");

  moe_config empty = c;
  empty.T = 0;
  CHECK(moe_workspace_size(&empty, &bytes) == MOE_OK, "workspace size of an empty batch");
  CHECK(moe_route(&empty, NULL, NULL, NULL, NULL, 0) == MOE_OK, "empty batch route is a no-op");

  CHECK(moe_route(&c, NULL, NULL, NULL, NULL, 0) == MOE_ERR_INVALID_ARG, "null logits rejected");
  CHECK(strcmp(moe_status_string(MOE_OK), "ok") == 0, "status string of MOE_OK");
  CHECK(strstr(moe_status_string(MOE_ERR_DEVICE_VALUE), "power of two") != NULL,
        "status string of MOE_ERR_DEVICE_VALUE");
  return fails ? 1 : 0;
}
