/* A plain C11 client of liblkv: includes only include/lkv.h (no CUDA or
 * PyTorch headers), links liblkv.so and makes the calls that need no GPU --
 * status strings, sizes, and argument checks that fail on the host before
 * anything is launched.  Prints "ok" and exits 0 when every result is the
 * documented one. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "lkv.h"

static int failures = 0;

static void expect(int cond, const char *what) {
  if (!cond) {
    printf("FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  const lkv_qspec k6v4 = {6, 4, 64};
  const lkv_qspec bad_bits = {5, 4, 64};
  void *fake = (void *)(uintptr_t)0x7F0000000000ull; /* 16-byte aligned, never dereferenced */
  void *misaligned = (void *)(uintptr_t)0x7F0000000008ull;

  expect(lkv_version() > 0, "version");
  expect(strlen(lkv_status_string(LKV_OK)) > 0, "status string");
  expect(lkv_row_bytes(6, 128) == 96 && lkv_row_bytes(4, 128) == 64, "row bytes");
  expect(lkv_sz_row_bytes(128, 64) == 16, "(scale, zero) row bytes");
  expect(lkv_decode_workspace_bytes(k6v4, 16, 32, 8, 8192, 128) > 0, "workspace size");
  expect(lkv_quantize_kv(bad_bits, 1, 1, 256, 128, fake, fake, fake, fake, fake, fake, fake, NULL) ==
             LKV_ERR_UNSUPPORTED,
         "bad bit width rejected");
  expect(lkv_quantize_kv(k6v4, 1, 1, 256, 128, fake, misaligned, fake, fake, fake, fake, fake, NULL) ==
             LKV_ERR_INVALID_ARG,
         "misaligned pointer rejected");
  expect(lkv_decode_attention(k6v4, 1, 3, 2, 256, 128, fake, fake, fake, fake, fake, fake, 0.1f, 0.0f, fake, NULL,
                              NULL, fake, 1 << 30, NULL) == LKV_ERR_INVALID_ARG,
         "Hq not a multiple of Hkv rejected");
  expect(lkv_decode_attention(k6v4, 1, 4, 2, 256, 128, fake, fake, fake, fake, fake, fake, 0.1f, 0.0f, fake, NULL,
                              NULL, fake, 256, NULL) == LKV_ERR_WORKSPACE,
         "short workspace rejected");
  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
