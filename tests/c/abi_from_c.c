/* A plain C consumer of the library's C ABI (no Python, no torch): builds
 * descriptors, sizes and packs small weight tensors of every packed format
 * on the host, and checks the documented argument errors.  Compiled and run
 * on the host by tests/test_c_abi.py; needs no GPU.  Prints "ok" and
 * returns 0 when every check holds, else names the first failed check. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "hq.h"

#define CHECK(cond)                                                 \
  do {                                                              \
    if (!(cond)) {                                                  \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                     \
    }                                                               \
  } while (0)

static int pack_case(int32_t fmt, int32_t n, int32_t k, int32_t group, int32_t zp, size_t code_bytes,
                     size_t scale_bytes, size_t expect_size) {
  hq_quant_desc d;
  CHECK(hq_quant_desc_init(&d, fmt, n, k, group, zp, 1) == HQ_OK);
  CHECK(d.layout_version == hq_layout_version());
  const size_t size = hq_packed_size(&d);
  CHECK(size == expect_size);
  uint8_t* codes = (uint8_t*)calloc(code_bytes, 1);
  uint8_t* scales = (uint8_t*)calloc(scale_bytes, 1);
  uint8_t* zeros = zp ? (uint8_t*)calloc((size_t)n * (k / group), 1) : NULL;
  uint8_t* out = (uint8_t*)malloc(size);
  CHECK(codes && scales && out && (!zp || zeros));
  for (size_t i = 0; i < code_bytes; ++i) codes[i] = (uint8_t)(i * 37u + 11u);
  for (size_t i = 0; i < scale_bytes; ++i) scales[i] = (uint8_t)(100u + i % 20u);
  CHECK(hq_pack_weights(&d, codes, scales, zeros, 0.5f, out, size) == HQ_OK);
  CHECK(hq_pack_weights(&d, codes, scales, zeros, 0.5f, out, size - 1) == HQ_ERR_WORKSPACE_TOO_SMALL);
  CHECK(hq_pack_weights(&d, NULL, scales, zeros, 0.5f, out, size) == HQ_ERR_INVALID_ARG);
  free(codes);
  free(scales);
  free(zeros);
  free(out);
  return 0;
}

int main(void) {
  const int32_t n = 256, k = 512;
  const size_t nt = n / 128, kb = k / 128;
  /* INT4 (scales fp16, zero points) */
  if (pack_case(HQ_FMT_INT4, n, k, 128, 1, (size_t)n * k / 2, (size_t)n * kb * 2, nt * kb * (8192 + 256 + 128)))
    return 1;
  /* INT3 (bit-stream codes) and INT2 */
  if (pack_case(HQ_FMT_INT3, n, k, 128, 0, (size_t)n * k * 3 / 8, (size_t)n * kb * 2, nt * kb * (6144 + 256)))
    return 1;
  if (pack_case(HQ_FMT_INT2, n, k, 128, 1, (size_t)n * k / 4, (size_t)n * kb * 2, nt * kb * (4096 + 256 + 128)))
    return 1;
  /* MXFP4 for the W4A16 kernels, MXFP4 and NVFP4 for the block-scaled ones */
  if (pack_case(HQ_FMT_MXFP4_A16, n, k, 32, 0, (size_t)n * k / 2, (size_t)n * k / 32, nt * kb * 8704)) return 1;
  if (pack_case(HQ_FMT_MXFP4, n, k, 32, 0, (size_t)n * k / 2, (size_t)n * k / 32,
                (size_t)n * k / 2 + nt * (k / 128) * 512))
    return 1;
  if (pack_case(HQ_FMT_NVFP4, n, k, 16, 0, (size_t)n * k / 2, (size_t)n * k / 16,
                (size_t)n * k / 2 + nt * (k / 64) * 512 + 16))
    return 1;

  /* descriptor and call errors, before anything is launched */
  hq_quant_desc d;
  CHECK(hq_quant_desc_init(&d, HQ_FMT_INT4, n, 100, 128, 0, 1) == HQ_ERR_UNSUPPORTED);
  CHECK(hq_quant_desc_init(&d, 42, n, k, 128, 0, 1) == HQ_ERR_INVALID_ARG);
  CHECK(hq_quant_desc_init(NULL, HQ_FMT_INT4, n, k, 128, 0, 1) == HQ_ERR_INVALID_ARG);
  /* exact-integer weights need a 128-K group scale: MXFP4 (one per 32 K) has none */
  CHECK(hq_quant_desc_init(&d, HQ_FMT_MXFP4_A16, n, k, 32, 0, 1) == HQ_OK);
  hq_tuning t;
  memset(&t, 0, sizeof t);
  t.variant = 2;
  CHECK(hq_gemm_w4a16(&d, (void*)16, (void*)16, 4, (void*)32, &t, (void*)256, 1 << 20, NULL) ==
        HQ_ERR_UNSUPPORTED);
  CHECK(hq_quant_desc_init(&d, HQ_FMT_INT3, n, k, 128, 1, 1) == HQ_OK);
  CHECK(hq_gemm_w4a16(&d, NULL, NULL, 0, NULL, NULL, NULL, 0, NULL) == HQ_OK); /* m == 0 */
  CHECK(hq_gemm_w4a16(&d, (void*)16, (void*)18, 4, (void*)32, NULL, (void*)256, 1 << 20, NULL) ==
        HQ_ERR_ALIGNMENT);
  d.layout_version = 0;
  CHECK(hq_packed_size(&d) == 0);
  CHECK(hq_status_string(HQ_ERR_DEVICE_TIMEOUT) != NULL && strlen(hq_status_string(HQ_ERR_DEVICE_TIMEOUT)) > 0);
  printf("ok\n");
  return 0;
}
