/* A C program against include/svdq.h and libsvdq_b200.so: host-only calls of
 * the ABI (sizes, weight binding, layout conversions, argument validation),
 * which need no GPU.  Prints "ok" and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "svdq.h"

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                                       \
    }                                                                 \
  } while (0)

int main(void) {
  const int N = 256, K = 512, r = 32;
  CHECK(strstr(svdq_version(), "sm_100a") != NULL);
  CHECK(strcmp(svdq_status_string(SVDQ_ERR_MISALIGNED), "SVDQ_ERR_MISALIGNED") == 0);

  /* weight binding is pointer arithmetic on a caller buffer */
  const size_t wb = svdq_weight_bytes(N, K, r, 1);
  CHECK(wb > 0);
  CHECK(svdq_weight_bytes(100, K, r, 1) == 0); /* N % 128 != 0 */
  void* fake = (void*)(uintptr_t)0x7F0000000000ull;
  svdq_weight w;
  CHECK(svdq_weight_bind(fake, wb, N, K, r, 1, &w) == SVDQ_OK);
  CHECK(w.format == SVDQ_FORMAT_NVFP4 && w.N == N && w.K == K && w.r == r);
  CHECK(svdq_weight_bind(fake, wb - 1, N, K, r, 1, &w) == SVDQ_ERR_WORKSPACE_TOO_SMALL);
  CHECK(svdq_weight_bind_format(fake, wb, N, K, r, 1, SVDQ_FORMAT_INT4, &w) == SVDQ_OK);
  CHECK(w.format == SVDQ_FORMAT_INT4);
  CHECK(svdq_weight_bind_format(fake, wb, N, K, r, 1, 9, &w) == SVDQ_ERR_INVALID_ARG);

  /* argument validation happens before any device work */
  void* dev = (void*)(uintptr_t)0x7E0000000000ull;
  CHECK(svdq_quantize_act(NULL, 64, &w, dev, dev, dev, NULL) == SVDQ_ERR_INVALID_ARG);
  CHECK(svdq_quantize_act((const uint16_t*)((char*)dev + 8), 64, &w, dev, dev, dev, NULL) ==
        SVDQ_ERR_MISALIGNED);
  CHECK(svdq_linear_forward(dev, 0, &w, dev, dev, 0, NULL) == SVDQ_OK); /* M == 0 */

  /* NVFP4 scale layout round trip (rows padded to 128 in the native layout) */
  const int rows = 130;
  const size_t nat_bytes = svdq_act_scales_bytes(rows, K);
  CHECK(nat_bytes == (size_t)256 * (K / 16));
  uint8_t* logical = malloc((size_t)rows * (K / 16));
  uint8_t* back = malloc((size_t)rows * (K / 16));
  uint8_t* native = malloc(nat_bytes);
  for (size_t i = 0; i < (size_t)rows * (K / 16); ++i) logical[i] = (uint8_t)((i * 37u) % 127u);
  CHECK(svdq_scales_to_native(logical, rows, K, native) == SVDQ_OK);
  CHECK(svdq_act_scales_to_logical(native, rows, K, back) == SVDQ_OK);
  CHECK(memcmp(logical, back, (size_t)rows * (K / 16)) == 0);

  /* INT4 fp16 scales: group-major [K/64][rows_pad] */
  const int ng = K / 64, rows_pad = 256;
  uint16_t* l16 = malloc(sizeof(uint16_t) * rows * ng);
  uint16_t* b16 = malloc(sizeof(uint16_t) * rows * ng);
  uint16_t* n16 = malloc(sizeof(uint16_t) * rows_pad * ng);
  for (int i = 0; i < rows * ng; ++i) l16[i] = (uint16_t)(0x3C00 + i);
  CHECK(svdq_int4_scales_to_native(l16, rows, rows_pad, K, n16) == SVDQ_OK);
  CHECK(n16[3 * rows_pad + 5] == l16[5 * ng + 3]); /* row 5, group 3 */
  CHECK(n16[0 * rows_pad + rows] == 0);            /* padding row */
  CHECK(svdq_int4_scales_to_logical(n16, rows, rows_pad, K, b16) == SVDQ_OK);
  CHECK(memcmp(l16, b16, sizeof(uint16_t) * rows * ng) == 0);

  free(logical); free(back); free(native); free(l16); free(b16); free(n16);
  printf("ok\n");
  return 0;
}
