/* A plain C99 caller of the library: only nvfp4.h and libnvfp4.so, no CUDA
 * or torch headers.  It exercises the host-side contract (status codes,
 * messages, empty calls, workspace sizing); device pointers would come from
 * the caller's allocator in real use. */
#include <stdio.h>
#include <string.h>

#include "nvfp4.h"

int main(void) {
  int bad = 0;
  const float one = 1.0f; /* stands in for a device pointer: never dereferenced */

  /* nothing to quantize: OK without touching a device */
  nvfp4_status s = nvfp4_quantize(NULL, NVFP4_DT_BF16, 0, 4096, NULL, NULL, NULL, NVFP4_LAYOUT_SWIZZLED, NULL);
  if (s != NVFP4_OK) bad |= 1;

  /* one global scale without the other is refused on the host */
  s = qqmm(NVFP4_MODE_NVFP4, 128, 128, 256, NULL, NULL, NULL, NULL, &one, NULL, NULL, NVFP4_DT_BF16, NULL);
  if (s != NVFP4_ERR_INVALID_ARG || strstr(nvfp4_last_error_message(), "or neither") == NULL) bad |= 2;
  printf("qqmm: %s: %s\n", nvfp4_status_string(s), nvfp4_last_error_message());

  /* the MoE workspace for 4096 tokens, top-8, 64 experts */
  if (gather_qmm_workspace_size(4096, 8, 64) == 0 || gather_qmm_workspace_size(4096, 8, 2048) != 0) bad |= 4;

  /* padded scale bytes of a [200, 4096] NVFP4 operand in the MMA layout */
  if (nvfp4_scale_bytes(200, 4096 / 16, NVFP4_LAYOUT_SWIZZLED) != (size_t)256 * 256) bad |= 8;

  printf("%s\n", bad ? "FAILED" : "ok");
  return bad;
}
