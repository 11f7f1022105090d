/* Links against libhkv.so from plain C (C99) and exercises host-side paths
 * that need no GPU: the version string, argument errors and their messages,
 * and zero-sized calls.  Exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "hkv.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s (last error: %s)\n", what, hkv_last_error());
    ++failures;
  }
}

int main(void) {
  expect(strstr(hkv_version(), "sm_100a") != NULL, "version names the target");
  /* Hq not a multiple of Hkv */
  expect(hkv_retrieve_topk(1, 6, 4, 128, NULL, NULL, 10, 10, 0, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) ==
             HKV_ERR_INVALID_ARG,
         "group mismatch rejected");
  expect(strstr(hkv_last_error(), "multiple") != NULL, "message names the mismatch");
  /* unsupported code width */
  expect(hkv_retrieve_topk(1, 4, 4, 96, NULL, NULL, 10, 10, 0, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) ==
             HKV_ERR_UNSUPPORTED,
         "96-bit codes rejected");
  /* empty batch: nothing to do, nothing launched */
  expect(hkv_retrieve_topk(0, 4, 4, 128, NULL, NULL, 10, 10, 0, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) == HKV_OK,
         "empty batch is a no-op");
  /* workspace sizing rejects a bad group before it asks the device anything */
  expect(hkv_workspace_bytes(1, 6, 4, 1024, 128, 16, 0, 0) == 0, "workspace of a bad shape is 0");
  /* paged: too few pages for the tokens */
  expect(hkv_retrieve_topk_paged(1, 4, 2, 128, NULL, NULL, NULL, 2, 4, 4, 10, 0, 0, 4, NULL, NULL, NULL, 0, NULL, NULL) ==
             HKV_ERR_INVALID_ARG,
         "short page table rejected");
  /* norm-weighted retrieval past 65536 candidates without a workspace */
  expect(hkv_retrieve_topk_normw(1, 4, 2, 128, (const uint32_t*)16, (const uint32_t*)16, (const uint16_t*)16, 70000,
                                 70000, 0, 0, 4, (int32_t*)16, NULL, NULL, 0, NULL) == HKV_ERR_UNSUPPORTED,
         "long normw window without a workspace rejected");
  /* norm-weighted decode step: sign codes are 128 bits */
  expect(hkv_decode_step_normw(1, 4, 2, HKV_BF16, 64, NULL, NULL, NULL, NULL, NULL, 10, 10, 0, 0, 4, 0.1f, NULL, NULL,
                               NULL, NULL, NULL, NULL, 0, NULL, NULL) == HKV_ERR_UNSUPPORTED,
         "64-bit codes rejected by the norm-weighted decode step");
  /* G-way merge with no partials */
  expect(hkv_lse_merge_n(0, 4, NULL, NULL, NULL, NULL, NULL) == HKV_ERR_INVALID_ARG, "G = 0 rejected");
  if (failures == 0) printf("c abi ok\n");
  return failures == 0 ? 0 : 1;
}
