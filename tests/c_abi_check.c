/* Calls the C ABI of libmcs.so from plain C (no Python, no torch): argument checks that return
 * before any device work, so it runs without a GPU.  Built and run by tests/test_abi_cpu.py. */
#include <stdio.h>
#include <string.h>

#include "mcs.h"

static int failures = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main(void) {
  CHECK(mcs_abi_version() == 1);
  CHECK(strcmp(mcs_status_string(MCS_OK), "MCS_OK") == 0);
  mcs_shape bad_d = {1, 2, 1024, 96, 0.0f};
  mcs_shape bad_n = {1, 1, 0, 64, 0.0f};
  mcs_shape big_n = {1, 1, (1 << 24) + 128, 128, 0.0f};
  mcs_shape ok = {1, 24, 32256, 128, 0.0f};
  CHECK(mcs_dense_attn(bad_d, NULL, NULL, NULL, NULL, NULL, NULL) == MCS_ERR_SHAPE);
  CHECK(mcs_dense_attn(bad_n, NULL, NULL, NULL, NULL, NULL, NULL) == MCS_ERR_INVALID_ARG);
  CHECK(mcs_dense_attn(big_n, NULL, NULL, NULL, NULL, NULL, NULL) == MCS_ERR_SHAPE);
  CHECK(mcs_group(ok, NULL, 96, NULL, NULL, 0, NULL) == MCS_ERR_SHAPE);            /* C not in {64,128} */
  CHECK(mcs_sparse_attn(ok, NULL, NULL, NULL, NULL, 128, NULL, 0, NULL, NULL, NULL) == MCS_ERR_INVALID_ARG);
  CHECK(mcs_sparse_attn(ok, NULL, NULL, NULL, NULL, 128, NULL, 16, NULL, NULL, NULL) == MCS_ERR_INVALID_ARG);
  CHECK(mcs_workspace_size(bad_d, 128, 16) == 0);
  CHECK(mcs_host_staging_size(ok, 2) == (size_t)2 * 4 * 2 * 32256 * 128 * 2);
  CHECK(mcs_host_staging_size(ok, 0) == 0);
  CHECK(mcs_sparse_attn_host(ok, NULL, NULL, NULL, NULL, 128, NULL, 16, NULL, NULL, 0, NULL, 0, NULL) ==
        MCS_ERR_INVALID_ARG);
  if (failures == 0) printf("c abi ok\n");
  return failures == 0 ? 0 : 1;
}
