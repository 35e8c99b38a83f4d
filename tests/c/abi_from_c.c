/* Uses the library from plain C through include/dit_attn.h: version, status strings and
 * host-side argument validation.  Every attention call below has an invalid argument, so
 * nothing reaches the GPU (the program runs on machines without one).  Exit status 0 when
 * every check holds; prints the first failing check otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "dit_attn.h"

#define CHECK(cond)                                   \
  do {                                                \
    if (!(cond)) {                                    \
      fprintf(stderr, "check failed: %s\n", #cond);   \
      return 1;                                       \
    }                                                 \
  } while (0)

int main(void) {
  /* fake, aligned, non-null device addresses; never dereferenced (see above) */
  const uintptr_t base = (uintptr_t)1 << 40;
  void* q = (void*)base;
  void* k = (void*)(base + ((uintptr_t)1 << 30));
  void* v = (void*)(base + ((uintptr_t)2 << 30));
  void* out = (void*)(base + ((uintptr_t)3 << 30));
  float* lse = (float*)(base + ((uintptr_t)4 << 30));

  CHECK(dit_version() >= 100);
  CHECK(strcmp(dit_status_str(DIT_OK), "DIT_OK") == 0);
  CHECK(strcmp(dit_status_str(DIT_ERR_TIMEOUT | (3 << 8)), "DIT_ERR_TIMEOUT") == 0);

  CHECK(dit_attn_fwd(NULL, k, v, out, lse, 1, 2, 256, 128, 0.1f, DIT_BF16, NULL, NULL) == DIT_ERR_INVALID_ARG);
  CHECK(dit_attn_fwd(q, k, v, out, lse, 1, 2, 256, 96, 0.1f, DIT_BF16, NULL, NULL) == DIT_ERR_UNSUPPORTED);
  CHECK(dit_attn_fwd((char*)q + 8, k, v, out, lse, 1, 2, 256, 128, 0.1f, DIT_BF16, NULL, NULL) ==
        DIT_ERR_MISALIGNED);
  CHECK(dit_attn_fwd_chunk(q, k, v, out, lse, 1, 2, 256, 256, 128, 10, 5, 0.1f, DIT_BF16, DIT_FP32, NULL, NULL) ==
        DIT_ERR_INVALID_ARG);
  CHECK(dit_attn_fwd(q, k, v, out, lse, 1, 2, 256, 128, 0.1f, DIT_FP8_E4M3, NULL, NULL) == DIT_ERR_INVALID_ARG);

  const void* outs[2] = {k, v};
  const float* lses[2] = {lse, lse + 1024};
  CHECK(dit_attn_merge(outs, lses, 0, out, NULL, 1, 2, 8, 64, DIT_FP32, DIT_BF16, NULL) == DIT_ERR_INVALID_ARG);
  CHECK(dit_na3d_fwd(q, k, v, out, lse, 1, 2, 3, 4, 5, 64, 2, 3, 3, 0.1f, NULL) == DIT_ERR_INVALID_ARG);
  CHECK(dit_quant_fp8_workspace_bytes(1) == 4);
  CHECK(dit_set_sm_reserve(-1) == DIT_ERR_INVALID_ARG);
  CHECK(dit_set_wait_timeout_us(0) == DIT_OK);
  printf("abi_from_c ok (version %d)\n", dit_version());
  return 0;
}
