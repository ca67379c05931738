/* A plain C99 client of libkvpop: the header compiles as C, the library
 * links without Python or PyTorch, and every call below validates its
 * arguments on the host before touching a device, so this runs anywhere.
 * Exit status 0 when every expectation holds; each failure is printed. */
#include <stdio.h>
#include <string.h>

#include "kvpop.h"

static int failures = 0;

static void expect_status(const char* what, kvpop_status got, kvpop_status want) {
  if (got != want) {
    printf("FAIL %s: %s (%d), expected %s (%d); last error: %s\n", what, kvpop_status_string(got), (int)got,
           kvpop_status_string(want), (int)want, kvpop_last_error());
    ++failures;
  }
}

static void expect_size(const char* what, size_t got, size_t want) {
  if (got != want) {
    printf("FAIL %s: %zu bytes, expected %zu\n", what, got, want);
    ++failures;
  }
}

int main(void) {
  /* Any non-null, 16-byte aligned address: validation fails before it is used. */
  static unsigned char fake[64] __attribute__((aligned(16)));
  void* p = fake;
  const int32_t cu[2] = {0, 100};
  const int32_t cu_empty[2] = {0, 0};
  const int32_t budget[1] = {50};
  const kvpop_shape sh = {1, 100, 4, 2, 128};
  const kvpop_shape empty = {1, 0, 4, 2, 128};
  kvpop_shape bad_dim = sh;
  bad_dim.head_dim = 96;
  const size_t rows = kvpop_target_workspace_bytes(sh);

  if (kvpop_abi_version() != KVPOP_ABI_VERSION) {
    printf("FAIL abi version %d, header says %d\n", (int)kvpop_abi_version(), KVPOP_ABI_VERSION);
    ++failures;
  }
  if (strcmp(kvpop_status_string(KVPOP_OK), "ok") != 0) ++failures;

  expect_status("row_lse, q NULL", kvpop_row_lse(NULL, p, cu, sh, 0.1f, (float*)p, NULL, NULL),
                KVPOP_ERR_INVALID_ARG);
  expect_status("row_lse, head_dim 96", kvpop_row_lse(p, p, cu, bad_dim, 0.1f, (float*)p, NULL, NULL),
                KVPOP_ERR_UNSUPPORTED);
  expect_status("row_lse, T = 0", kvpop_row_lse(p, p, cu_empty, empty, 0.1f, (float*)p, NULL, NULL), KVPOP_OK);
  expect_status("future_target, window < 0",
                kvpop_future_target(p, p, cu, sh, 0.1f, -1, (const float*)p, (float*)p, p, rows, NULL, NULL),
                KVPOP_ERR_INVALID_ARG);
  expect_status("future_target, workspace too small",
                kvpop_future_target(p, p, cu, sh, 0.1f, 4, (const float*)p, (float*)p, p, rows - 16, NULL, NULL),
                KVPOP_ERR_INVALID_ARG);
  expect_status("keep_mask, budget below sinks + window",
                kvpop_keep_mask((const float*)p, cu, sh, 64, 4, budget, (uint8_t*)p, NULL), KVPOP_ERR_INVALID_ARG);
  expect_status("check_device_status, NULL", kvpop_check_device_status(NULL, NULL), KVPOP_ERR_INVALID_ARG);

  expect_size("target workspace", rows, 4u * 100u * 16u);   /* 6400 = 25 x 256 */
  expect_size("fused workspace", kvpop_fused_workspace_bytes(cu, sh), 256u + 6400u);
  {
    const kvpop_cache_shape cs = {1, 8, 2, 128, 1000};
    expect_size("decode workspace", kvpop_decode_workspace_bytes(cs), 1u * 8u * 8u * 130u * 4u);
  }

  if (failures == 0) printf("c client ok: abi %d\n", (int)kvpop_abi_version());
  return failures == 0 ? 0 : 1;
}
