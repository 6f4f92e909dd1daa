/*
 * A plain C99 caller of the library: compiled against include/s2attn.h and linked with
 * libs2attn.so, it checks the calls that answer on the host -- version, status strings,
 * workspace sizes, argument validation -- without touching a GPU.  Exit status 0 means
 * every check passed; otherwise the failing check is printed.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "s2attn.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  CHECK(s2attn_version() == 100);
  CHECK(strcmp(s2attn_status_string(S2ATTN_OK), "ok") == 0);
  CHECK(strncmp(s2attn_status_string(S2ATTN_ERR_UNSUPPORTED), "unsupported", 11) == 0);

  /* workspace sizes: fp32 dQ accumulator + delta; decode partials of at most 64 splits */
  CHECK(s2attn_bwd_workspace_bytes(1, 32768, 32, 128) == (size_t)1 * 32768 * 32 * 128 * 4 + (size_t)32 * 32768 * 4);
  CHECK(s2attn_bwd_workspace_bytes(0, 32768, 32, 128) == 0);
  CHECK(s2attn_decode_workspace_bytes(1, 4, 32768, 32, 128) == (size_t)32 * 64 * 4 * (128 + 2) * 4);
  CHECK(s2attn_decode_workspace_bytes(1, 2, 1, 2, 128) == 0);
  /* LoRA projections: padded adapters and the rank-64 intermediate; none without an adapter */
  CHECK(lora_proj_workspace_bytes(32768, 4096, 4096, 3, 8) == (size_t)(3 * 32768 + 3 * 4096) * 64 * 2 + (size_t)3 * 64 * 4096 * 2);
  CHECK(lora_proj_workspace_bytes(32768, 4096, 4096, 1, 0) == 0);

  /* argument errors are returned before anything is enqueued (no device needed) */
  CHECK(s2attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1000, 2, 128, 300, 0, NULL) == S2ATTN_ERR_INVALID_ARG);
  CHECK(s2attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1024, 2, 64, 512, 0, NULL) == S2ATTN_ERR_UNSUPPORTED);
  CHECK(s2attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1024, 2, 128, 512, 1, NULL) == S2ATTN_ERR_INVALID_ARG);
  {
    void* p = (void*)(uintptr_t)0x10000;
    CHECK(s2attn_bwd(p, p, p, p, p, (const float*)p, p, p, p, 1, 1024, 2, 128, 512, 0, p, 16, NULL) ==
          S2ATTN_ERR_WORKSPACE);
    CHECK(s2attn_decode(p, p, p, p, (float*)p, 1, 129, 200, 2, 128, p, 1 << 20, NULL) == S2ATTN_ERR_UNSUPPORTED);
    CHECK(rope_pi_apply_offset(p, NULL, 1, 16, 2, 128, -1, 0.5f, 10000.0f, NULL) == S2ATTN_ERR_INVALID_ARG);
    CHECK(lora_proj_fwd(p, p, p, p, p, 300, 520, 384, 3, 8, 2.0f, 0, 128, 100, 0.5f, 10000.0f, p, 1 << 26, NULL) ==
          S2ATTN_ERR_UNSUPPORTED);
    CHECK(lora_proj_fwd(p, p, p, p, p, 300, 520, 256, 3, 8, 2.0f, 0, 128, 100, 0.5f, 10000.0f, p, 64, NULL) ==
          S2ATTN_ERR_WORKSPACE);
  }
  CHECK(s2attn_fwd_f32(NULL, NULL, NULL, NULL, NULL, 1, 90, 3, 256, 18, 1, NULL) == S2ATTN_ERR_UNSUPPORTED);
  CHECK(rope_pi_apply(NULL, NULL, 1, 16, 2, 128, 0.5f, 10000.0f, NULL) == S2ATTN_ERR_INVALID_ARG);

  if (failures == 0) printf("C ABI boundary: all checks passed\n");
  return failures == 0 ? 0 : 1;
}
