/*
 * libdsa from plain C99, with no Python and no torch: the header compiles as
 * C, the library links, and the calls that need no device answer as
 * include/dsa.h documents them (version and status names, workspace and split
 * arithmetic, the grouped-attention plan, host argument checks that return
 * before any device work, and the two-tier cache's host planner).
 * Exit status 0 on success; a failed check prints its line and exits 1.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "dsa.h"

#define CHECK(c)                                                        \
  do {                                                                  \
    if (!(c)) {                                                         \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c);  \
      return 1;                                                         \
    }                                                                   \
  } while (0)

int main(void) {
  int head = -1, tail = -1, splits = -1;
  size_t ws, st_bytes;
  void* st;
  int32_t idx[8], q_off[3], copies[16 * 3], table[2 * 8];
  const int32_t idx5[2 * 5] = {0, 16, 32, 48, 64, 112, -1, -1, -1, -1};
  int n = -1, i;
  int64_t stats[3];

  CHECK(dsa_version() > 0);
  CHECK(strcmp(dsa_status_string(DSA_OK), "DSA_OK") == 0);
  CHECK(strcmp(dsa_status_string(DSA_ERR_DEVICE_BOUNDS), "DSA_ERR_DEVICE_BOUNDS") == 0);
  CHECK(dsa_status_string(12345) != NULL);

  /* workspace: the fp32 score rows at least; invalid sizes give 0 */
  ws = dsa_workspace_bytes(32, 131072, DSA_MAX_TOPK, 0);
  CHECK(ws >= (size_t)32 * 131072 * sizeof(float));
  CHECK(dsa_workspace_bytes(0, 131072, DSA_MAX_TOPK, 0) == 0);
  CHECK(dsa_workspace_bytes(32, 131072, DSA_MAX_TOPK + 1, 0) == 0);
  CHECK(dsa_workspace_bytes(32, 131072, DSA_MAX_TOPK, DSA_MAX_SPLITS + 1) == 0);

  /* split-K parts: the requested count, or the library's choice for 0 */
  CHECK(dsa_choose_splits(32, 2048, 3) == 3);
  CHECK(dsa_choose_splits(32, 2048, 0) == 2);  /* 64 units fill 64 of 74 SM pairs */
  CHECK(dsa_choose_splits(4, 2048, 0) == 16);

  /* grouped attention of 4 layers x 64 queries: three whole waves, then 34
     units cut in two */
  CHECK(dsa_mla_group_plan(256, 2048, &head, &tail, &splits) == 1);
  CHECK(head == 222 && tail == 34 && splits == 2);
  CHECK(dsa_mla_group_plan(0, 2048, &head, &tail, &splits) == 0);

  /* host argument checks: nothing is enqueued, no device is needed */
  CHECK(dsa_indexer_topk(NULL, NULL, NULL, 0, NULL, NULL, NULL, 1, 1, DSA_IDX_HEADS, 1, 2048, 0,
                         NULL, NULL, NULL, 0, NULL) == DSA_ERR_INVALID_ARG);
  CHECK(dsa_sparse_mla_decode(NULL, NULL, 1, DSA_PAGE_SIZE, NULL, 1, NULL, NULL, NULL, 1, 1,
                              DSA_HEADS, 2048, 0.1f, 0, NULL, NULL, NULL, 0, NULL) ==
        DSA_ERR_INVALID_ARG);

  /* two-tier cache, host planner: 2 sequences, 4 device slots each, 8
     logical pages of 16 tokens */
  st_bytes = dsa_tier_state_bytes(2, 4, 8);
  CHECK(st_bytes > 0 && dsa_tier_state_bytes(0, 4, 8) == 0);
  st = malloc(st_bytes);
  CHECK(st != NULL);
  CHECK(dsa_tier_init(st, st_bytes, 2, 4, 8) == DSA_OK);
  q_off[0] = 0; q_off[1] = 1; q_off[2] = 2;
  /* sequence 0 selects pages 0, 1 and 2; sequence 1 page 7 (twice) */
  idx[0] = 0; idx[1] = 17; idx[2] = 33; idx[3] = -1;
  idx[4] = 112; idx[5] = 127; idx[6] = -1; idx[7] = -1;
  CHECK(dsa_tier_plan(st, idx, 2, 4, q_off, table, copies, 16, &n, stats) == DSA_OK);
  CHECK(n == 4 && stats[0] == 0 && stats[1] == 4 && stats[2] == 0);
  for (i = 0; i < n; ++i) CHECK(copies[3 * i + 2] == -1);   /* nothing evicted yet */
  CHECK(table[0] >= 0 && table[1] >= 0 && table[2] >= 0 && table[3] == -1);
  CHECK(table[8 + 7] >= 0 && table[8 + 0] == -1);
  /* the same step again: every page is resident */
  CHECK(dsa_tier_plan(st, idx, 2, 4, q_off, table, copies, 16, &n, stats) == DSA_OK);
  CHECK(n == 0 && stats[0] == 4 && stats[1] == 0);
  /* five distinct pages of one sequence do not fit its 4 slots: refused,
     and the state is unchanged (the first step's pages are still resident) */
  CHECK(dsa_tier_plan(st, idx5, 2, 5, q_off, NULL, copies, 16, &n, stats) == DSA_ERR_UNSUPPORTED);
  CHECK(dsa_tier_plan(st, idx, 2, 4, q_off, NULL, copies, 16, &n, stats) == DSA_OK);
  CHECK(n == 0 && stats[0] == 4);
  free(st);

  printf("libdsa C ABI: host calls ok (version %d)\n", dsa_version());
  return 0;
}
