/*
 * A C99 caller of the KDA library: the headers under include/ compile as plain C (no CUDA or
 * C++ headers), the library links, and its host-side checks answer without touching a device.
 * Built and run by tests/test_abi_cpu.py; prints "ok <version>" and exits 0 when every check
 * holds.
 */
#include <stdio.h>
#include <string.h>

#include "kda.h"
#include "kda_selftest.h"

/* the no-allocation entry point's declaration and its scratch limit are part of the C ABI */
typedef char kda_noalloc_limit_is_64_mib[(KDA_NOALLOC_SCRATCH_BYTES == ((size_t)64 << 20)) ? 1 : -1];
static kda_status_t (*const kda_noalloc_entry)(const void*, const void*, const void*, kda_dtype_t,
                                               const float*, const float*, const float*,
                                               const int32_t*, int32_t, int32_t, int32_t, int32_t,
                                               int32_t, int32_t, int32_t, void*, float*,
                                               kda_stream_t) = kda_chunk_fwd_noalloc;

static int fails = 0;
#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      printf("FAIL line %d: %s\n", __LINE__, #cond);         \
      ++fails;                                               \
    }                                                        \
  } while (0)

int main(void) {
  size_t bytes = 0;
  kda_fusion_t fz;
  memset(&fz, 0, sizeof(fz));
  CHECK(strcmp(kda_status_string(KDA_OK), "KDA_OK") == 0);
  CHECK(kda_chunk_fwd_workspace_size(2, 4096, 32, 128, 128, 64, 2, KDA_DTYPE_BF16, &bytes) ==
        KDA_OK);
  CHECK(bytes > 0 && bytes % 256 == 0);
  CHECK(kda_chunk_fwd_workspace_size(1, 256, 1, 96, 128, 64, 1, KDA_DTYPE_BF16, &bytes) ==
        KDA_ERR_UNSUPPORTED);
  CHECK(kda_chunk_bwd_workspace_size(2, 4096, 32, 128, 128, 2, KDA_DTYPE_BF16, &bytes) == KDA_OK);
  /* null tensors with tokens present: refused on the host */
  CHECK(kda_chunk_fwd(NULL, NULL, NULL, KDA_DTYPE_BF16, NULL, NULL, NULL, NULL, 1, 1, 64, 1, 128,
                      128, 64, NULL, NULL, NULL, 0, NULL) == KDA_ERR_INVALID_ARG);
  CHECK(kda_chunk_fwd_fused(NULL, NULL, NULL, KDA_DTYPE_BF16, NULL, NULL, NULL, NULL, 1, 1, 64, 1,
                            128, 128, 64, NULL, NULL, NULL, 0, &fz, NULL) == KDA_ERR_INVALID_ARG);
  CHECK(kda_recurrent_step(NULL, NULL, NULL, KDA_DTYPE_BF16, NULL, NULL, NULL, NULL, 4, 2, 128, 128,
                           NULL) == KDA_ERR_INVALID_ARG);
  CHECK(kda_recurrent_step(NULL, NULL, NULL, KDA_DTYPE_BF16, NULL, NULL, NULL, NULL, 4, 2, 256, 128,
                           NULL) == KDA_ERR_UNSUPPORTED);
  /* nothing to do: no tokens, no sequences */
  CHECK(kda_chunk_fwd(NULL, NULL, NULL, KDA_DTYPE_F32, NULL, NULL, NULL, NULL, 0, 0, 0, 1, 32, 32,
                      32, NULL, NULL, NULL, 0, NULL) == KDA_OK);
  CHECK(kda_selftest_wait_timeout(0, NULL) == KDA_ERR_INVALID_ARG);
  CHECK(kda_noalloc_entry != NULL);
  if (fails == 0) printf("ok %s\n", kda_version());
  return fails != 0;
}
