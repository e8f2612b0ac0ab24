/* The C ABI used from plain C: the header compiles as C99, its structs have
 * the sizes the Python binding assumes, and the host-only entry points
 * (descriptor validation, workspace size, stage names, init without a GPU)
 * answer through the shared library without touching a device. */
#include <stdio.h>
#include <string.h>

#include "moe_sparse.h"

_Static_assert(sizeof(moe_sparse_desc) == 16 * 4, "moe_sparse_desc layout");
_Static_assert(sizeof(moe_stats) == 15 * 8, "moe_stats layout");

static int fails = 0;
#define CHECK(c)                                  \
  do {                                            \
    if (!(c)) {                                   \
      printf("FAIL line %d: %s\n", __LINE__, #c); \
      ++fails;                                    \
    }                                             \
  } while (0)

int main(void) {
  moe_sparse_desc d;
  memset(&d, 0, sizeof d);
  d.d_model = 4096;
  d.d_ff = 14336;
  d.n_experts = 8;
  d.top_k_max = 2;
  d.max_tokens = 64;
  d.renormalize = 1;
  d.dtype = MOE_BF16;
  d.path = MOE_PATH_AUTO;
  d.score = MOE_SCORE_H;
  d.out_f32 = 0;
  CHECK(moe_sparse_validate_desc(&d) == MOE_OK);

  size_t bytes = 0;
  CHECK(moe_sparse_workspace_bytes(&d, &bytes) == MOE_OK);
  CHECK(bytes > 0);
  d.max_tokens = 128;
  size_t bytes2 = 0;
  CHECK(moe_sparse_workspace_bytes(&d, &bytes2) == MOE_OK);
  CHECK(bytes2 > bytes);

  moe_sparse_desc bad = d;
  bad.d_model = 100; /* not a multiple of 256 for bf16 */
  CHECK(moe_sparse_validate_desc(&bad) != MOE_OK);
  bad = d;
  bad.score = 7;
  CHECK(moe_sparse_validate_desc(&bad) == MOE_ERR_INVALID);
  bad = d;
  bad.out_f32 = 2;
  CHECK(moe_sparse_validate_desc(&bad) == MOE_ERR_INVALID);
  CHECK(moe_sparse_validate_desc(NULL) == MOE_ERR_INVALID);

  CHECK(moe_sparse_stage_name(0) != NULL && strlen(moe_sparse_stage_name(0)) > 0);
  CHECK(moe_sparse_stage_name(-1) == NULL || strlen(moe_sparse_stage_name(-1)) == 0);

  moe_sparse_ctx* ctx = (moe_sparse_ctx*)&d; /* must be reset to NULL on failure */
  if (moe_sparse_init(&d, &ctx) == MOE_OK) {
    /* a GPU was present: init worked, so tear down */
    CHECK(ctx != NULL);
    CHECK(moe_sparse_destroy(ctx) == MOE_OK);
  } else {
    CHECK(ctx == NULL);
  }
  printf("%s\n", fails ? "FAIL" : "OK");
  return fails ? 1 : 0;
}
