/*
 * A plain C99 client of libwvae.so: compiled against include/wvae.h alone (no
 * CUDA headers, no C++), it exercises the calls that need no GPU - version,
 * status names, buffer sizes and host-side argument validation - and prints
 * one "name value" line per result for the test that runs it.
 */
#include <stdint.h>
#include <stdio.h>

#include "wvae.h"

static void* fake_ptr(uintptr_t v) { return (void*)v; }

int main(void) {
  const void* a = fake_ptr(0x10000); /* 16-byte aligned, never dereferenced */
  void* y = fake_ptr(0x20000);
  const float* g = (const float*)fake_ptr(0x30000);
  int s;

  printf("version %d\n", wvae_version());
  for (s = 0; s <= 7; ++s) printf("status%d %s\n", s, wvae_status_string(s));
  printf("conv_packed_512x512x27_bf16 %zu\n", wvae_conv_packed_bytes(512, 512, 3, 3, 3, WVAE_BF16));
  printf("conv_packed_unsupported %zu\n", wvae_conv_packed_bytes(512, 512, 2, 3, 3, WVAE_BF16));
  printf("resblock_ws_256_bf16 %zu\n", wvae_resblock_workspace_bytes(4, 176, 312, 256, 256, WVAE_BF16));
  printf("trunk_launches %d\n", wvae_decode_trunk_launches());
  /* rejected on the host, before any device call */
  printf("norm_null_x %d\n",
         (int)wvae_norm_silu(NULL, y, g, g, 1, 1, 1, 64, 1e-12f, WVAE_BF16, NULL));
  printf("norm_bad_c %d\n", (int)wvae_norm_silu(a, y, g, g, 1, 1, 1, 60, 1e-12f, WVAE_BF16, NULL));
  printf("norm_misaligned %d\n",
         (int)wvae_norm_silu(fake_ptr(0x10004), y, g, g, 1, 1, 1, 64, 1e-12f, WVAE_BF16, NULL));
  printf("selftest_bad_limit %d\n", (int)wvae_selftest_wait_timeout(0u, NULL));
  return 0;
}
