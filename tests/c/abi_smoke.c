/* Plain C use of the library's host-side calls: sizes, argument checks and the weight pack.
 * Built and run by tests/test_abi_c.py with gcc against include/svdq.h and libsvdq.so. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "svdq.h"

static int fail(const char* what) {
  fprintf(stderr, "FAIL: %s\n", what);
  return 1;
}

int main(void) {
  svdq_sizes sz;
  if (svdq_buffer_sizes(SVDQ_FMT_NVFP4_G16, 300, 256, 512, 16, &sz) != SVDQ_OK) return fail("sizes nvfp4");
  if (sz.a_codes != (size_t)300 * 256 || sz.a_scales != (size_t)384 * 512 / 16) return fail("nvfp4 sizes values");
  if (svdq_buffer_sizes(SVDQ_FMT_W8A8, 300, 256, 512, 16, &sz) != SVDQ_OK) return fail("sizes w8a8");
  if (sz.a_codes != (size_t)300 * 512 || sz.a_scales != (size_t)384 * 4) return fail("w8a8 sizes values");
  if (svdq_buffer_sizes(SVDQ_FMT_NVFP4_G16, 300, 200, 512, 16, &sz) != SVDQ_ERR_INVALID_ARG) return fail("N % 128");
  if (strcmp(svdq_status_string(SVDQ_OK), "ok") != 0) return fail("status string");

  /* pack a 128 x 128 residual whose first column is 127 and the rest small: W8A8 gives
   * s = 1 per row and codes rint(x) */
  const int64_t N = 128, K = 128;
  float* R = (float*)calloc((size_t)(N * K), sizeof(float));
  for (int64_t n = 0; n < N; ++n) {
    R[n * K + 0] = 127.0f;
    R[n * K + 1] = 2.5f;    /* tie -> 2 */
    R[n * K + 2] = -3.5f;   /* tie -> -4 */
  }
  if (svdq_buffer_sizes(SVDQ_FMT_W8A8, 1, N, K, 0, &sz) != SVDQ_OK) return fail("sizes pack");
  uint8_t* codes = (uint8_t*)malloc(sz.w_codes);
  float* scales = (float*)malloc(sz.w_scales);
  float gw = 0.f;
  if (svdq_pack_weight(SVDQ_FMT_W8A8, N, K, 0, 1.0f, R, NULL, NULL, codes, scales, &gw, NULL, NULL) != SVDQ_OK)
    return fail("pack w8a8");
  if (gw != 1.0f || scales[0] != 1.0f) return fail("w8a8 scale");
  if ((int8_t)codes[0] != 127 || (int8_t)codes[1] != 2 || (int8_t)codes[2] != -4 || codes[3] != 0)
    return fail("w8a8 codes");
  /* a non power-of-two activation scale is rejected before any work */
  if (svdq_pack_weight(SVDQ_FMT_NVFP4_G16, N, K, 0, 3.0f, R, NULL, NULL, codes, scales, &gw, NULL, NULL) !=
      SVDQ_ERR_INVALID_ARG)
    return fail("pack rejects");
  free(R);
  free(codes);
  free(scales);
  printf("ok\n");
  return 0;
}
