/* A plain C99 client of the C-ABI, built and run by tests/test_c_client.py
 * without a GPU: it exercises only entry points that do their work on the
 * host (version, error text, argument checks, the shard planner). */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "shampoo.h"

static int failures = 0;

static void check(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  const char* v = shampoo_version();
  check(v != NULL && strlen(v) >= 5, "shampoo_version");

  /* the planner: 3 parameters over 2 ranks, every owner in range, costs > 0 */
  const int64_t shapes[6] = {1024, 1024, 512, 4096, 1, 777};
  const int32_t ndims[3] = {2, 2, 1};
  int32_t owner[3] = {-1, -1, -1};
  double cost[2] = {0.0, 0.0};
  shampoo_status st = shampoo_plan_shards(3, shapes, ndims, 512, 20, 2, owner, cost);
  check(st == SHAMPOO_OK, "plan_shards status");
  for (int i = 0; i < 3; ++i) check(owner[i] == 0 || owner[i] == 1, "owner in range");
  check(cost[0] > 0.0 && cost[1] > 0.0, "both ranks loaded");

  /* argument errors come back as SHAMPOO_EINVAL with a message, no abort */
  st = shampoo_plan_shards(3, shapes, ndims, 512, 20, 0, owner, cost);
  check(st == SHAMPOO_EINVAL, "plan_shards with 0 ranks");
  shampoo_ctx* ctx = NULL;
  const int64_t one[2] = {64, 32};
  st = shampoo_create(&ctx, 1, one, NULL, 100, 0.99f, 1e-6f, 4, SHAMPOO_GRAFT_ADAGRAD, 0.0f, SHAMPOO_F32, NULL);
  check(st == SHAMPOO_EINVAL && ctx == NULL, "create with block_size 100");
  check(strlen(shampoo_last_error(NULL)) > 0, "error text");
  check(shampoo_compute_roots(NULL) == SHAMPOO_EINVAL, "null context");
  shampoo_destroy(NULL);

  printf("owners %d %d %d costs %.3g %.3g\n", owner[0], owner[1], owner[2], cost[0], cost[1]);
  return failures ? 1 : 0;
}
