/*
 * c_client.c - a plain C99 caller of libqwen3attn.so, built by tests/test_c_client.py with
 * gcc against include/qwen3_attn.h alone (no CUDA headers, no C++).  It exercises only
 * calls that need no GPU: the version and status strings, the size helpers and the host
 * argument checks, which reject a call before anything is launched.  Prints "ok" and
 * exits 0 when every expectation holds; otherwise names the first failed one and exits 1.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "qwen3_attn.h"

static int failures = 0;

#define EXPECT(cond)                                  \
  do {                                                \
    if (!(cond)) {                                    \
      fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                     \
    }                                                 \
  } while (0)

int main(void) {
  /* Fake device addresses: 16-byte aligned, never dereferenced because every call below
   * fails its host-side checks first. */
  qwen3_bf16* const fake = (qwen3_bf16*)(uintptr_t)(1u << 20);
  float* const fakef = (float*)(uintptr_t)(1u << 20);
  int32_t* const fakei = (int32_t*)(uintptr_t)(1u << 20);

  EXPECT(strstr(qwen3_attn_version(), "sm_100a") != NULL);
  EXPECT(strlen(qwen3_attn_status_string(QWEN3_OK)) > 0);
  EXPECT(strcmp(qwen3_attn_status_string(QWEN3_ERR_WORKSPACE), qwen3_attn_status_string(QWEN3_OK)) != 0);

  /* 2 * Hkv * d bf16 values per cached token: 1024 values (2048 bytes) for Hkv = 4. */
  EXPECT(qwen3_attn_kv_cache_bytes(1, 4, 1, 128) == 2 * 1024);
  EXPECT(qwen3_attn_kv_cache_bytes(64, 8, 32769, 128) == (size_t)64 * 32769 * 2 * 8 * 128 * 2);
  EXPECT(qwen3_attn_prefill_workspace_size(2, 2048, 16, 8, 128) >= (size_t)2 * 2048 * (16 + 8) * 256);
  EXPECT(qwen3_attn_decode_workspace_size(64, 32, 128, 32769) > 0);

  /* Host argument checks: non-positive sizes, unsupported head layouts, a missing workspace. */
  EXPECT(qwen3_attn_prefill_ex(fake, fake, fake, fakef, fakef, fakei, fake, NULL, NULL, NULL, 0, NULL, 0,
                               0, 128, 16, 8, 128, 1e6f, 1e-6f, NULL) == QWEN3_ERR_INVALID_ARG);
  EXPECT(qwen3_attn_prefill_ex(fake, fake, fake, fakef, fakef, fakei, fake, NULL, NULL, NULL, 0, NULL, 0,
                               1, 128, 16, 8, 64, 1e6f, 1e-6f, NULL) == QWEN3_ERR_UNSUPPORTED);
  EXPECT(qwen3_attn_prefill_ex(fake, fake, fake, fakef, fakef, fakei, fake, NULL, NULL, NULL, 0, NULL, 0,
                               1, 128, 24, 8, 128, 1e6f, 1e-6f, NULL) == QWEN3_ERR_UNSUPPORTED);
  EXPECT(qwen3_attn_prefill_ex(fake, fake, fake, fakef, fakef, fakei, fake, NULL, NULL, NULL, 0, NULL, 0,
                               1, 128, 16, 8, 128, 1e6f, 1e-6f, NULL) == QWEN3_ERR_WORKSPACE);
  EXPECT(qwen3_attn_decode(fake, fake, fake, fakef, fakef, fake, fake, fakei, fake, NULL, 0, 32, 8, 128, 4096,
                           1e6f, 1e-6f, NULL, 0, NULL) == QWEN3_ERR_INVALID_ARG);
  EXPECT(qwen3_attn_decode(fake, fake, fake, fakef, fakef, fake, fake, fakei, fake, NULL, 4, 32, 8, 128, 4096,
                           1e6f, 1e-6f, NULL, 0, NULL) == QWEN3_ERR_WORKSPACE);

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
