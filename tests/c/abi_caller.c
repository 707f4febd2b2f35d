/*
 * A plain C caller of the library: includes include/moe.h, links
 * libmoe_b200.so, and exercises the host-side paths that need no GPU (status
 * strings, size queries, argument and placement checks, empty batches).
 * Built and run by tests/test_c_caller.py; prints "ok" and exits 0 when
 * every check holds, else names the failing check and exits 1.
 */
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int fails = 0;
#define CHECK(cond)                                   \
  do {                                                \
    if (!(cond)) {                                    \
      printf("FAIL line %d: %s\n", __LINE__, #cond); \
      ++fails;                                        \
    }                                                 \
  } while (0)

int main(void) {
  moe_shape s = {16384, 256, 64, 4, 64, 8, MOE_BF16};
  size_t scratch = 0, fwd = 0, packed = 0;
  CHECK(moe_scratch_size(&s, &scratch) == MOE_OK && scratch > 0);
  CHECK(moe_forward_workspace_size(&s, &fwd) == MOE_OK && fwd > scratch);
  CHECK(moe_packed_weights_size(&s, &packed) == MOE_OK);
  /* router W_r^T padded to 16 experts, then 3 matrices of E*d*f bf16 */
  CHECK(packed >= (size_t)2 * (64 * 256 + 3 * 64 * 256 * 64));
  CHECK(strcmp(moe_status_string(MOE_OK), "MOE_OK") == 0);
  CHECK(strcmp(moe_status_string(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE") == 0);

  /* shape limits */
  moe_shape bad = s;
  bad.k = 17;
  CHECK(moe_scratch_size(&bad, &scratch) == MOE_ERR_INVALID_ARG);
  bad = s;
  bad.d = 100;
  CHECK(moe_scratch_size(&bad, &scratch) == MOE_ERR_UNSUPPORTED);
  CHECK(moe_scratch_size(NULL, &scratch) == MOE_ERR_INVALID_ARG);
  CHECK(moe_scratch_size(&s, NULL) == MOE_ERR_INVALID_ARG);

  /* the forward: a too small workspace and missing tensors are refused
     before any launch; an empty batch is a no-op */
  void* fake = (void*)(uintptr_t)4096; /* never dereferenced on these paths */
  CHECK(moe_forward(&s, fake, fake, NULL, NULL, fake, NULL, fake, 16, NULL) == MOE_ERR_WORKSPACE);
  CHECK(moe_forward(&s, NULL, fake, NULL, NULL, fake, NULL, fake, fwd, NULL) == MOE_ERR_INVALID_ARG);
  CHECK(moe_forward_routed(&s, fake, fake, NULL, NULL, NULL, fake, NULL, fake, fwd, NULL) ==
        MOE_ERR_INVALID_ARG);
  moe_shape empty = s;
  empty.T = 0;
  size_t fwd0 = 0;
  CHECK(moe_forward_workspace_size(&empty, &fwd0) == MOE_OK);
  CHECK(moe_forward(&empty, NULL, NULL, NULL, NULL, NULL, NULL, fake, fwd0, NULL) == MOE_OK);

  /* the expert -> rank map must give every rank E/ep experts */
  int32_t map[64];
  for (int e = 0; e < 64; ++e) map[e] = e / 8;
  map[0] = 1; /* rank 0 now owns 7 experts, rank 1 owns 9 */
  CHECK(moe_forward(&s, fake, fake, NULL, map, fake, NULL, fake, fwd, NULL) == MOE_ERR_INVALID_ARG);

  if (fails) return 1;
  printf("ok\n");
  return 0;
}
