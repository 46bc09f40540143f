/* The C ABI from plain C: include/zf.h compiles as C11 with every warning
 * an error, and the host-side parts of libzf.so (version, status strings,
 * size queries, argument errors) answer as the header documents without any
 * CUDA device. */
#include <stdio.h>
#include <string.h>

#include "zf.h"

#define CHECK(c)                                                  \
  do {                                                            \
    if (!(c)) {                                                   \
      fprintf(stderr, "failed: %s (line %d)\n", #c, __LINE__);    \
      return 1;                                                   \
    }                                                             \
  } while (0)

int main(void) {
  CHECK(zf_version() >= 100);
  CHECK(strcmp(zf_status_string(ZF_OK), "ZF_OK") == 0);
  CHECK(strcmp(zf_status_string(ZF_ERR_TIMEOUT), "ZF_ERR_TIMEOUT") == 0);

  /* sizes: worst case 2 bytes per value; 48-byte header + 32 raw blocks per chunk */
  CHECK(zf_compressed_bound(640) == 1280);
  CHECK(zf_compressed_bound(63) == 0);
  CHECK(zf_paged_bound(3) == 3 * (48 + 4096));
  CHECK(zf_append_staging_bytes(2, 8) == 2 * 8 * 4144);
  const size_t ws = zf_decode_workspace_size(32, 32, 8, 4096, 148);
  CHECK(ws > 0);
  CHECK(zf_decode_host_workspace_size(32, 32, 8, 256, 4096, 148) > ws);
  CHECK(zf_decode_workspace_size(-1, 32, 8, 4096, 148) == 0);

  /* argument errors come back before anything touches CUDA */
  zf_kv_compressed kv;
  memset(&kv, 0, sizeof kv);
  CHECK(zf_decode_attention(NULL, &kv, &kv, 8, NULL, 4, NULL, 64, 2, 8, 2, 64, 0.088f, NULL, NULL, NULL, 0,
                            NULL) == ZF_ERR_UNSUPPORTED);
  CHECK(zf_decode_attention(NULL, &kv, &kv, 8, NULL, 4, NULL, 64, 2, 8, 2, 128, 0.088f, NULL, NULL, NULL, 0,
                            NULL) == ZF_ERR_INVALID_ARG);
  CHECK(zf_decode_attention(NULL, &kv, &kv, 8, NULL, 4, NULL, 64, 0, 8, 2, 128, 0.088f, NULL, NULL, NULL, 0,
                            NULL) == ZF_OK);
  CHECK(zf_fp8_quantize(NULL, 7, 1.0f, NULL, NULL) == ZF_ERR_INVALID_ARG);
  CHECK(zf_check_bounded_wait(ZF_WAITCHECK_PLAIN_TIMEOUT + 1, NULL, NULL, NULL) == ZF_ERR_INVALID_ARG);
  puts("ok");
  return 0;
}
