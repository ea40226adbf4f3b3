/* A plain C11 host program against the library's C ABI: it includes only
 * dualflow.h, links libdualflow.so, and makes host-only calls (every compute
 * call carries an invalid argument, so nothing reaches the device). Exit code
 * 0 when every documented answer comes back. */
#include <stdio.h>
#include <string.h>

#include "dualflow.h"

static int fails = 0;

static void expect(int got, int want, const char* what) {
  if (got != want) {
    fprintf(stderr, "%s: got %d, want %d\n", what, got, want);
    ++fails;
  }
}

int main(void) {
  void* fake = (void*)0x7f0000000000ull;
  expect(dualflow_abi_version(), 1, "abi version");
  expect(strncmp(dualflow_status_string(DF_ERR_SHAPE), "DF_", 3), 0, "status string");
  expect(dualflow_decode_attn(NULL, NULL, NULL, 0, fake, fake, fake, 4, fake, 200, fake, NULL, 0,
                              2, 8, 2, 128, 64, 8, 0.f, DF_BF16, 0, NULL, 0, NULL, NULL),
         DF_ERR_NULL, "decode attention without q1");
  expect(dualflow_kv_append(fake, fake, 0, fake, fake, fake, 4, fake, 2, 3, 128, 64, 8, 7, NULL,
                            NULL),
         DF_ERR_UNSUPPORTED, "append with an unknown dtype");
  expect(dualflow_prefill(fake, 0, fake, fake, 0, NULL, NULL, fake, fake, fake, 8, fake, NULL, 256,
                          400, fake, 0, NULL, 2, 300, 8, 2, 128, 64, 16, 0.f, DF_FP32, NULL, 0,
                          NULL, NULL),
         DF_ERR_UNSUPPORTED, "prefill in fp32");
  expect(dualflow_prefill_num_launches(1, 1), 4, "prefill launches");
  expect(dualflow_prefill_kernel(128, 300, fake, 0, 8), DF_PREFILL_KERNEL_TCGEN05,
         "prefill kernel choice");
  expect(dualflow_mixture_head(fake, 0, 2, 4095, DF_BF16, fake, 0, fake, NULL),
         DF_ERR_UNSUPPORTED, "mixture head with V not a multiple of 8");
  if (fails == 0) printf("c abi ok\n");
  return fails == 0 ? 0 : 1;
}
