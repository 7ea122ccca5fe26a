/* A plain C program against the C ABI (include/moe.h, libmoe.so): the host-side entry
 * points, callable without a GPU.  Prints "ok" and returns 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int failures = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static moe_config base_config(void) {
  moe_config c;
  memset(&c, 0, sizeof(c));
  c.N = 4096;
  c.d = 2048;
  c.E = 64;
  c.k = 6;
  c.I = 1408;
  c.n_shared = 2;
  c.P = 8;
  c.n_groups = 1;
  c.topk_groups = 1;
  c.score = MOE_SCORE_SOFTMAX;
  c.renormalize = 0;
  c.dtype = MOE_BF16;
  c.bias_mode = MOE_BIAS_LOGITS;
  return c;
}

int main(void) {
  CHECK(moe_version() > 0);
  const char* s = moe_status_string(MOE_ERR_TIMEOUT);
  CHECK(s != NULL && s[0] != '\0');

  moe_config c = base_config();
  CHECK(moe_check_config(&c) == MOE_OK);
  CHECK(moe_workspace_bytes(&c) > 0);
  CHECK(moe_layout_workspace_bytes(&c) > 0);
  CHECK(moe_check_config(NULL) == MOE_ERR_INVALID_ARG);
  moe_config bad = c;
  bad.k = 9;
  CHECK(moe_check_config(&bad) == MOE_ERR_UNSUPPORTED);
  bad = c;
  bad.E = 513;
  CHECK(moe_check_config(&bad) == MOE_ERR_UNSUPPORTED);
  bad = c;
  bad.N = -1;
  CHECK(moe_check_config(&bad) == MOE_ERR_INVALID_ARG);
  bad = c;
  bad.d = 2050; /* a bf16 row of 4100 bytes is not a multiple of 16 */
  CHECK(moe_check_config(&bad) == MOE_ERR_UNSUPPORTED);
  CHECK(moe_workspace_bytes(&bad) == 0);

  /* the expert-parallel window: parts in order, inside the window */
  size_t off[11];
  CHECK(moe_ep_window_layout(&c, 6144, off) == MOE_OK);
  for (int i = 1; i < 11; ++i) CHECK(off[i] > off[i - 1]);
  CHECK(moe_ep_window_bytes(&c, 6144) > off[10]);
  CHECK(moe_ep_window_bytes(&c, 0) == 0);

  /* EPLB plan on the host: 8 experts, 4 extra copies, 4 owners */
  const int32_t E = 8, R = 4, P = 4;
  const int64_t load[8] = {100, 10, 10, 10, 10, 10, 10, 50};
  int32_t copies[8], replica_off[9], replica_slots[12], slot_expert[12], slot_owner[12];
  int64_t owner_load[4];
  CHECK(moe_eplb_plan(E, R, P, load, copies, replica_off, replica_slots, slot_expert, slot_owner, owner_load) ==
        MOE_OK);
  int sum = 0;
  for (int e = 0; e < E; ++e) {
    CHECK(copies[e] >= 1);
    sum += copies[e];
    CHECK(replica_off[e + 1] - replica_off[e] == copies[e]);
    for (int c2 = replica_off[e]; c2 < replica_off[e + 1]; ++c2) CHECK(slot_expert[replica_slots[c2]] == e);
  }
  CHECK(sum == E + R);
  CHECK(copies[0] > copies[1]); /* the hottest expert gets copies */
  int64_t total = 0, per_owner[4] = {0, 0, 0, 0};
  for (int j = 0; j < P; ++j) total += owner_load[j];
  CHECK(total == 100 + 6 * 10 + 50);
  for (int q = 0; q < E + R; ++q) per_owner[slot_owner[q]] += 1;
  for (int j = 0; j < P; ++j) CHECK(per_owner[j] == (E + R) / P);
  CHECK(moe_eplb_plan(E, 3, P, load, copies, replica_off, replica_slots, slot_expert, slot_owner, owner_load) ==
        MOE_ERR_INVALID_ARG); /* (E + R) % P != 0 */

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
