/* A plain C11 program against include/nvfp4.h and libnvfp4.so: the boundary
 * is usable without C++ or Python.  Only host-side checks run (every call
 * below is rejected before any launch), so no GPU is needed. */
#include <stdio.h>
#include <string.h>

#include "nvfp4.h"

static int fails = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      printf("FAIL line %d: %s\n", __LINE__, #cond);                  \
      ++fails;                                                        \
    }                                                                 \
  } while (0)

int main(void) {
  void* fake = (void*)0x10000; /* never dereferenced */
  uint8_t* fb = (uint8_t*)fake;
  nvfp4_qtensor_t out;
  memset(&out, 0, sizeof out);

  CHECK(nvfp4_version() >= 10000);
  CHECK(strcmp(nvfp4_status_string(NVFP4_OK), "ok") == 0);
  CHECK(nvfp4_launch_count() == 0);
  CHECK(nvfp4_workspace_size(16, 16, NVFP4_ROWWISE) > 0);
  CHECK(nvfp4_workspace_size(16, 16, NVFP4_ROWWISE | NVFP4_ALPHA_PROVIDED) == 0);
  /* bad mode, bad flags, missing outputs, shapes */
  CHECK(nvfp4_quantize(fake, 16, 16, 16, (nvfp4_mode_t)7, NVFP4_ROWWISE, 0, 0, NULL, &out, NULL, 0, NULL) ==
        NVFP4_ERR_ARG);
  CHECK(nvfp4_quantize(fake, 16, 16, 16, NVFP4_RTN, 0x8000u, 0, 0, NULL, &out, NULL, 0, NULL) == NVFP4_ERR_ARG);
  CHECK(nvfp4_quantize(fake, 16, 16, 16, NVFP4_RHT_SR_HW, NVFP4_ROWWISE, 0, 0, NULL, &out, NULL, 0, NULL) ==
        NVFP4_ERR_ARG);
  CHECK(nvfp4_quantize(fake, 16, 24, 24, NVFP4_RTN, NVFP4_ROWWISE, 0, 0, NULL, &out, NULL, 0, NULL) ==
        NVFP4_ERR_SHAPE);
  CHECK(nvfp4_quantize(NULL, 0, 16, 16, NVFP4_RTN, NVFP4_ROWWISE, 0, 0, NULL, &out, NULL, 0, NULL) == NVFP4_OK);
  CHECK(nvfp4_dequantize(fb, fb, (const float*)fake, 16, 24, 0, 0, fake, NULL) == NVFP4_ERR_SHAPE);
  CHECK(nvfp4_gemm(fb, fb, (const float*)fake, fb, fb, (const float*)fake, 100, 128, 128, fake,
                   NVFP4_OUT_DTYPE_BF16, 128, NULL, 0, NULL) == NVFP4_ERR_SHAPE);
  CHECK(nvfp4_gemm_quantize(fb, fb, (const float*)fake, fb, fb, (const float*)fake, 256, 256, 128, NULL, 256,
                            NVFP4_MS_EDEN, 0, (const float*)fake, fb, fb, NULL, NULL, 0, NULL) == NVFP4_ERR_ARG);
  /* amax pass: bad flags, missing output, shapes; AMAX_PROVIDED needs amax input and excludes ALPHA_PROVIDED */
  CHECK(nvfp4_amax(fake, 16, 16, 16, NVFP4_BLOCK2D, 0, (float*)fake, NULL, NULL) == NVFP4_ERR_ARG);
  CHECK(nvfp4_amax(fake, 16, 16, 16, 0, 0, NULL, NULL, NULL) == NVFP4_ERR_ARG);
  CHECK(nvfp4_amax(fake, 16, 24, 24, 0, 0, (float*)fake, NULL, NULL) == NVFP4_ERR_SHAPE);
  CHECK(nvfp4_amax(fake, 24, 16, 16, NVFP4_COLWISE | NVFP4_RHT, 0, (float*)fake, NULL, NULL) == NVFP4_ERR_SHAPE);
  CHECK(nvfp4_workspace_size(16, 16, NVFP4_ROWWISE | NVFP4_AMAX_PROVIDED) == 0);
  CHECK(nvfp4_quantize(fake, 16, 16, 16, NVFP4_RTN, NVFP4_ROWWISE | NVFP4_AMAX_PROVIDED, 0, 0, NULL, &out, NULL, 0,
                       NULL) == NVFP4_ERR_ARG);
  CHECK(nvfp4_quantize(fake, 16, 16, 16, NVFP4_RTN, NVFP4_ROWWISE | NVFP4_AMAX_PROVIDED | NVFP4_ALPHA_PROVIDED, 0, 0,
                       (const float*)fake, &out, NULL, 0, NULL) == NVFP4_ERR_ARG);
  /* MXFP4 */
  CHECK(mxfp4_quantize(fake, 32, 48, 48, NVFP4_ROWWISE, 0, fb, fb, NULL, NULL, NULL, NULL) == NVFP4_ERR_SHAPE);
  CHECK(mxfp4_quantize(fake, 32, 32, 32, 0, 0, fb, fb, NULL, NULL, NULL, NULL) == NVFP4_ERR_ARG);
  CHECK(mxfp4_dequantize(fb, fb, 16, 48, 0, 0, fake, NULL) == NVFP4_ERR_SHAPE);
  CHECK(mxfp4_gemm(fb, fb, fb, fb, 128, 256, 128, fake, NVFP4_OUT_DTYPE_BF16, 256, NULL, 0, NULL) ==
        NVFP4_ERR_SHAPE);
  CHECK(nvfp4_launch_count() == 0); /* nothing was launched */
  printf(fails ? "FAILED\n" : "OK\n");
  return fails != 0;
}
