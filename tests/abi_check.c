/* A plain C99 program against include/bonsai.h and libbonsai.so: sizes,
 * status strings and the argument checks that return before any device
 * work (so it runs without a GPU).  Exits 0 and prints "ok" when every
 * answer is the documented one. */
#include <stdio.h>
#include <string.h>

#include "bonsai.h"

static int failures = 0;

static void expect(int got, int want, const char* what) {
  if (got != want) {
    fprintf(stderr, "%s: got %d, want %d\n", what, got, want);
    ++failures;
  }
}

int main(void) {
  /* sizes: 2 bits per INT2 weight, 1 per binary weight, 112 bytes per 512 base-3 weights */
  expect((int)(bonsai_packed_bytes(3072, 9216, BONSAI_TERNARY_INT2) == (size_t)3072 * 9216 / 4), 1, "INT2 bytes");
  expect((int)(bonsai_packed_bytes(3072, 9216, BONSAI_BINARY) == (size_t)3072 * 9216 / 8), 1, "binary bytes");
  expect((int)(bonsai_packed_bytes(3072, 9216, BONSAI_TERNARY_B3) == (size_t)3072 * 112 * 18), 1, "base-3 bytes");
  expect((int)(bonsai_scale_bytes(3072, 9216) == (size_t)3072 * 72 * 2), 1, "scale bytes");
  expect((int)bonsai_packed_bytes(8, 100, BONSAI_TERNARY_INT2), 0, "partial group");
  expect(strcmp(bonsai_status_string(BONSAI_OK), "ok"), 0, "status string");

  /* argument errors, reported before anything touches a device */
  expect(bonsai_pack(NULL, 4, 128, 9, NULL, NULL), BONSAI_ERR_INVALID_ARG, "pack: mode");
  expect(bonsai_pack(NULL, 4, 100, BONSAI_TERNARY_INT2, NULL, NULL), BONSAI_ERR_SHAPE, "pack: K % 128");
  expect(bonsai_pack(NULL, 0, 128, BONSAI_TERNARY_INT2, NULL, NULL), BONSAI_OK, "pack: empty");
  expect(bonsai_lowbit_gemm(NULL, NULL, NULL, 4, 4, 128, BONSAI_TERNARY_INT2, NULL, NULL), BONSAI_ERR_INVALID_ARG,
         "gemm: null");
  expect(bonsai_lowbit_gemm(NULL, NULL, NULL, 4, 4, 128, BONSAI_TERNARY_INT2, (uint16_t*)8, NULL), BONSAI_ERR_ALIGN,
         "gemm: misaligned out");
  expect(bonsai_lowbit_gemm(NULL, NULL, NULL, 0, 4, 128, BONSAI_BINARY, NULL, NULL), BONSAI_OK, "gemm: empty");

  bonsai_gemm_problem batch[2];
  memset(batch, 0, sizeof(batch));
  batch[0].M = 4;
  batch[0].N = 8;
  batch[0].K = 100; /* not a multiple of 128 */
  expect(bonsai_lowbit_gemm_batch(batch, 1, BONSAI_TERNARY_INT2, NULL), BONSAI_ERR_SHAPE, "batch: K % 128");
  expect(bonsai_lowbit_gemm_batch(batch, -1, BONSAI_TERNARY_INT2, NULL), BONSAI_ERR_INVALID_ARG, "batch: count");
  expect(bonsai_lowbit_gemm_batch(NULL, 0, BONSAI_TERNARY_INT2, NULL), BONSAI_OK, "batch: empty");
  expect(bonsai_lowbit_gemm_batch(NULL, 2, BONSAI_TERNARY_INT2, NULL), BONSAI_ERR_INVALID_ARG, "batch: null list");
  expect(bonsai_lowbit_gemm_batch(batch, 1, 7, NULL), BONSAI_ERR_INVALID_ARG, "batch: mode");
  batch[0].K = 128; /* shapes fine, output missing */
  expect(bonsai_lowbit_gemm_batch(batch, 1, BONSAI_BINARY, NULL), BONSAI_ERR_INVALID_ARG, "batch: null out");
  batch[0].M = 0; /* an empty problem needs no buffers */
  expect(bonsai_lowbit_gemm_batch(batch, 1, BONSAI_BINARY, NULL), BONSAI_OK, "batch: only empty problems");

  /* 4-bit group-affine weights: half a byte per weight, same argument rules */
  expect((int)(bonsai_hqq4_packed_bytes(3072, 9216) == (size_t)3072 * 9216 / 2), 1, "4-bit bytes");
  expect(bonsai_hqq4_pack(NULL, 4, 100, NULL, NULL), BONSAI_ERR_SHAPE, "4-bit pack: K % 128");
  expect(bonsai_hqq4_pack(NULL, 4, 128, NULL, NULL), BONSAI_ERR_INVALID_ARG, "4-bit pack: null");
  expect(bonsai_hqq4_gemm(NULL, NULL, NULL, NULL, 4, 4, 128, NULL, NULL), BONSAI_ERR_INVALID_ARG, "4-bit gemm: null");

  /* plan query: an empty GEMM plans nothing and needs no device */
  int bt = -1, ks = -1, ctas = -1, tiles = -1;
  expect(bonsai_gemm_plan(0, 8, 128, BONSAI_BINARY, &bt, &ks, &ctas, &tiles), BONSAI_OK, "plan: empty");
  expect(bt | ks | ctas | tiles, 0, "plan: empty is all zeros");
  expect(bonsai_gemm_plan(4, 8, 100, BONSAI_BINARY, &bt, &ks, &ctas, &tiles), BONSAI_ERR_SHAPE, "plan: K % 128");

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
