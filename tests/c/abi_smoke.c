/* A plain C99 caller of libconvrot.so: the header compiles as C, the library
 * links and loads without Python or PyTorch, and argument validation answers
 * before any device work (no GPU is needed for these calls). */
#include <stdio.h>
#include <string.h>

#include "convrot.h"

static int fails = 0;

static void expect(const char* what, convrot_status got, convrot_status want) {
  if (got != want) {
    printf("FAIL %s: %d (%s), want %d\n", what, (int)got, convrot_status_string(got), (int)want);
    ++fails;
  }
}

int main(void) {
  /* fake, 16-byte aligned device addresses: validation rejects before launching */
  void* A = (void*)0x10000;
  int8_t* Q = (int8_t*)0x10000;
  float* F = (float*)0x10000;

  if (convrot_version() <= 0) {
    printf("FAIL version\n");
    ++fails;
  }
  expect("group 128", convrot_rotate_quant_act(A, 4, 512, 128, NULL, 1e-6f, Q, F, NULL),
         CONVROT_ERR_UNSUPPORTED);
  expect("K % group", convrot_rotate_quant_act(A, 4, 384, 256, NULL, 1e-6f, Q, F, NULL),
         CONVROT_ERR_SHAPE);
  expect("null x", convrot_rotate_quant_act(NULL, 4, 512, 256, NULL, 1e-6f, Q, F, NULL),
         CONVROT_ERR_NULL);
  expect("misaligned x",
         convrot_rotate_quant_act((void*)0x10008, 4, 512, 256, NULL, 1e-6f, Q, F, NULL),
         CONVROT_ERR_ALIGN);
  expect("M = 0", convrot_rotate_quant_act(NULL, 0, 512, 256, NULL, 1e-6f, NULL, NULL, NULL),
         CONVROT_OK);
  expect("N % 8", convrot_int8_linear(Q, F, Q, F, 4, 12, 512, A, NULL, 0, NULL), CONVROT_ERR_SHAPE);
  expect("K % 32 int4", convrot_w4a8_linear(Q, F, (const uint8_t*)A, F, 4, 16, 48, A, NULL, 0, NULL),
         CONVROT_ERR_SHAPE);
  expect("weight-only N % 8",
         convrot_weight_only_linear(A, Q, F, 4, 12, 512, A, NULL, 0, NULL), CONVROT_ERR_SHAPE);
  if (convrot_linear_workspace_bytes(4, 12, 512, 8) != 0) {
    printf("FAIL workspace size of an invalid shape\n");
    ++fails;
  }
  if (strstr(convrot_status_string(CONVROT_ERR_SHAPE), "CONVROT_ERR_SHAPE") == NULL) {
    printf("FAIL status string\n");
    ++fails;
  }
  printf("%s\n", fails ? "abi smoke: failures" : "abi smoke: ok");
  return fails ? 1 : 0;
}
