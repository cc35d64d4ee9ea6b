/* A plain C99 consumer of include/moe.h, built and run by tests/test_c_consumer.py on a
 * machine without a GPU: it links libmoe.so and calls only the entry points that answer on
 * the host (layout and workspace queries, status strings, the tile-mode switch, argument
 * checks that reject before anything is enqueued).  It prints one "name value" line per
 * result; the test compares them with the Python binding's answers. */
#include <stdio.h>
#include <stdint.h>

#include "moe.h"

#define FAKE ((void*)4096) /* never dereferenced: every call below fails its host checks */

int main(void) {
  moe_plan_layout L;
  int st = moe_plan_get_layout(64, 8, 8, &L);
  printf("layout_status %d\n", st);
  printf("layout_words %lld\n", (long long)L.words);
  printf("layout_groups %lld\n", (long long)L.groups);
  printf("layout_max_groups_per_rank %d\n", (int)L.max_groups_per_rank);
  printf("dispatch_workspace_words %lld\n", (long long)moe_dispatch_workspace_words(4096, 64));
  printf("route_plan_workspace_words %lld\n", (long long)moe_route_plan_workspace_words(64));
  printf("route_plan_workspace_words_bad %lld\n", (long long)moe_route_plan_workspace_words(0));
  printf("ffn_tile_mode %d\n", moe_ffn_tile_mode());
  printf("set_ffn_tile_mode_bad %d\n", moe_set_ffn_tile_mode(7));
  /* argument checks */
  printf("topk_null_logits %d\n",
         moe_topk(NULL, 16, 8, 2, (int32_t*)FAKE, (float*)FAKE, (int32_t*)FAKE, NULL));
  printf("topk_k_above_E %d\n",
         moe_topk((const float*)FAKE, 16, 8, 9, (int32_t*)FAKE, (float*)FAKE, (int32_t*)FAKE, NULL));
  printf("plan_rows_not_divisible %d\n",
         moe_plan_balanced((const int32_t*)FAKE, 15, 1, 8, 4, 2, (int32_t*)FAKE, (int32_t*)FAKE, NULL));
  printf("route_plan_null_workspace %d\n",
         moe_route_plan((const float*)FAKE, NULL, 16, 8, 2, 4, 2, (int32_t*)FAKE, (float*)FAKE,
                        (int32_t*)FAKE, (int32_t*)FAKE, (double*)FAKE, (double*)FAKE,
                        (int32_t*)FAKE, NULL, (int32_t*)FAKE, NULL));
  printf("status_ok_string %s\n", moe_status_string(MOE_OK));
  printf("status_arg %d\n", (int)MOE_ERR_ARG);
  printf("status_shape %d\n", (int)MOE_ERR_SHAPE);
  return 0;
}
