/* A plain C client of liblwm_blockattn.so: includes only the public header,
 * links only the library, and exercises what needs no GPU (version, status
 * strings, workspace sizing, argument rejection before any launch). Built
 * and run by tests/test_abi.py. Exit code 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "lwm_blockattn.h"

#define CHECK(cond)                                             \
  do {                                                          \
    if (!(cond)) {                                              \
      fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                                 \
    }                                                           \
  } while (0)

int main(void) {
  /* any 16-byte aligned address: never dereferenced on these paths */
  void* p = (void*)(uintptr_t)(1u << 20);
  const size_t ws = lwm_blockattn_fwd_workspace_size(
      1, 4096, 8, 128, 128, 128, 4096, LWM_DTYPE_BF16, LWM_QK_BF16);
  CHECK(lwm_blockattn_version() == 1);
  CHECK(strcmp(lwm_status_string(LWM_OK), "ok") == 0);
  CHECK(ws > (size_t)4096 * 128 * 4);  /* holds at least the RoPE table */
  /* unsupported head dim, null q, too little workspace, empty problem */
  CHECK(lwm_blockattn_fwd(p, p, p, p, p, 1e4, 128, 128, 4096, 1, 4096, 8, 64,
                          LWM_DTYPE_BF16, LWM_QK_BF16, LWM_ROPE_INTERLEAVED,
                          p, p, p, ws, NULL) == LWM_ERR_UNSUPPORTED);
  CHECK(lwm_blockattn_fwd(NULL, p, p, p, p, 1e4, 128, 128, 4096, 1, 4096, 8,
                          128, LWM_DTYPE_BF16, LWM_QK_BF16,
                          LWM_ROPE_INTERLEAVED, p, p, p, ws,
                          NULL) == LWM_ERR_INVALID_ARG);
  CHECK(lwm_blockattn_fwd(p, p, p, p, p, 1e4, 128, 128, 4096, 1, 4096, 8, 128,
                          LWM_DTYPE_BF16, LWM_QK_BF16, LWM_ROPE_HALF, p, p, p,
                          ws - 1, NULL) == LWM_ERR_WORKSPACE);
  CHECK(lwm_blockattn_fwd(NULL, NULL, NULL, NULL, NULL, 1e4, 128, 128, 1, 1,
                          0, 8, 128, LWM_DTYPE_BF16, LWM_QK_BF16,
                          LWM_ROPE_INTERLEAVED, NULL, NULL, NULL, 0,
                          NULL) == LWM_OK);
  CHECK(lwm_blockffn_fwd(p, p, p, p, 256, 100, 256, 128, LWM_DTYPE_BF16, p, p,
                         (size_t)1 << 30, NULL) == LWM_ERR_UNSUPPORTED);
  printf("c client ok: version %d, fwd workspace %zu bytes\n",
         lwm_blockattn_version(), ws);
  return 0;
}
