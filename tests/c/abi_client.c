/* A plain C99 client of the fused linear layer's C ABI (include/fused_linear.h), built
 * with gcc and linked against libfused_linear.so.  It runs without a GPU: it asks for the
 * configuration of the 4096^3 RELU_AUX_BIAS layer and of a 32-row tail on a 148-SM device,
 * and checks that bad arguments come back as status codes with a message, never an abort.
 * Prints one line per check; exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "fused_linear.h"

static int failures = 0;

static void expect(int ok, const char* what) {
  printf("%s %s\n", ok ? "ok  " : "FAIL", what);
  if (!ok) ++failures;
}

static fl_epilogue_desc epilogue(fl_epi_kind kind, fl_dtype out) {
  fl_epilogue_desc e;
  memset(&e, 0, sizeof(e));
  e.kind = kind;
  e.out_dtype = out;
  e.bias_dtype = FL_BF16;
  e.residual_dtype = FL_BF16;
  e.scale = 1.0f;
  return e;
}

int main(void) {
  fl_plan_info info;
  fl_epilogue_desc e = epilogue(FL_EPI_RELU_AUX_BIAS, FL_BF16);
  fl_status st = fl_plan_preview(4096, 4096, 4096, FL_BF16, FL_COMPUTE_32F, &e, 148, 232448, &info);
  expect(st == FL_OK, "preview of the 4096^3 RELU_AUX_BIAS layer");
  expect(info.cta_pair == 1 && info.tile_m == 256 && info.grid == 148, "  CTA pairs, 256-row tiles, 148 CTAs");
  expect(info.stages >= 2 && info.smem_bytes <= 232448, "  fits shared memory with at least two stages");

  e = epilogue(FL_EPI_GELU_BIAS, FL_F32);
  e.has_residual = 1;
  e.scale = 0.5f;
  st = fl_plan_preview(32, 4096, 4096, FL_BF16, FL_COMPUTE_32F, &e, 148, 232448, &info);
  expect(st == FL_OK && info.swap_ab == 1 && info.split_k == 4, "32-row tail: swap-AB with split-K 4");

  e = epilogue(FL_EPI_NONE, FL_BF16);
  st = fl_plan_preview(64, 256, 256, FL_F32, FL_COMPUTE_32F, &e, 148, 232448, &info);
  expect(st == FL_ERR_UNSUPPORTED && strlen(fl_last_error()) > 0, "fp32 operands with FL_COMPUTE_32F rejected");
  e.ldo = 260; /* 520-byte rows */
  st = fl_plan_preview(64, 256, 256, FL_BF16, FL_COMPUTE_32F, &e, 148, 232448, &info);
  expect(st == FL_ERR_ALIGNMENT, "row pitch that is not a multiple of 16 bytes rejected");
  expect(fl_plan_preview(64, 256, 256, FL_BF16, FL_COMPUTE_32F, NULL, 148, 232448, &info) == FL_ERR_INVALID_ARG,
         "null descriptor rejected");
  expect(fl_free(NULL) == FL_OK, "fl_free(NULL) is a no-op");
  expect(fl_layernorm(NULL, NULL, NULL, NULL, 4, 4, 0, 0, FL_F32, FL_F32, FL_F32, 1e-5f, NULL) == FL_ERR_INVALID_ARG,
         "LayerNorm with null x and z rejected before any device call");

  printf("%d failure(s)\n", failures);
  return failures == 0 ? 0 : 1;
}
