/* A plain C caller of the library: include/fa.h must compile as C (not only
 * C++) and the host-side entry points must behave as declared. Only calls that
 * need no GPU are made: workspace-size queries, status strings, and argument
 * checks that return an error before anything is launched. Prints "ok". */
#include <stdio.h>
#include <string.h>

#include "fa.h"

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed line %d: %s\n", __LINE__, #cond); \
      return 1;                                                  \
    }                                                            \
  } while (0)

int main(void) {
  void* const P = (void*)0x100000; /* aligned, never dereferenced by these calls */
  CHECK(strcmp(fa_status_string(FA_OK), "FA_OK") == 0);
  CHECK(strcmp(fa_status_string(FA_ERR_WORKSPACE), "FA_ERR_WORKSPACE") == 0);
  CHECK(fa_bwd_workspace_size(1, 2, 2, 128, 64) > 0);
  CHECK(fa_bwd_workspace_size(1, 3, 2, 128, 64) == 0);            /* Hq % Hkv != 0 */
  CHECK(fa_fp8_workspace_size(1, 2, 2, 256, 128) > 0);
  CHECK(fa_mxfp8_workspace_size(1, 2, 2, 256, 128) > 0);
  CHECK(fa_mxfp8_workspace_size(1, 2, 2, 256, 64) == 0);             /* d = 128 only */
  CHECK(strcmp(fa_status_string(FA_ERR_BOUNDS), "FA_ERR_BOUNDS") == 0);
  CHECK(fa_decode_workspace_size(16, 32, 8, 1, 16384, 128, 0) > 0);
  CHECK(fa_decode_workspace_size(1, 8, 1, 4, 100, 128, 0) == 0);  /* 32 query rows per KV head */
  CHECK(fa_fwd(NULL, P, P, P, (float*)P, 1, 2, 2, 128, 64, 0, 0.125f, 0) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(P, P, P, P, (float*)P, 1, 2, 2, 128, 80, 0, 0.125f, 0) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd((char*)P + 2, P, P, P, (float*)P, 1, 2, 2, 128, 64, 0, 0.125f, 0) == FA_ERR_MISALIGNED);
  {
    size_t ws = fa_bwd_workspace_size(1, 2, 2, 128, 64);
    CHECK(fa_bwd(P, P, P, P, (const float*)P, P, P, P, P, P, ws - 1, 1, 2, 2, 128, 64, 0, 0.125f, 0) ==
          FA_ERR_WORKSPACE);
  }
  CHECK(fa_fwd_decode(P, P, P, P, (float*)P, P, 0, 2, 8, 2, 8, 4, 128, 1, 0.1f, 0, 0) == FA_ERR_INVALID_ARG);
  printf("ok\n");
  return 0;
}
