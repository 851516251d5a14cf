/* A plain C11 consumer of include/convrot.h: compiled with gcc
 * -Wall -Wextra -Werror -pedantic and linked against libconvrot_b200.so by
 * tests/test_c_consumer.py.  It uses only calls that need no GPU (status
 * strings, workspace sizes, arguments rejected before any device call), so it
 * runs on a machine without one.  Prints "ok" and exits 0 when every check
 * holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "convrot.h"

static int failures = 0;

static void check(int cond, const char *what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

static size_t r256(size_t v) { return (v + 255) / 256 * 256; }

int main(void) {
  /* 16-byte aligned stand-ins for device pointers: the calls below return
   * before they would be dereferenced. */
  static _Alignas(16) unsigned char buf[1 << 16];
  void *good = buf;
  void *bad = buf + 4;
  int code;

  check(strstr(convrot_version(), "sm_100a") != NULL, "version names sm_100a");
  for (code = CONVROT_OK; code <= CONVROT_ERR_TIMEOUT; ++code)
    check(convrot_status_string((convrot_status_t)code) != NULL, "status string");
  check(strcmp(convrot_status_string(CONVROT_ERR_SHAPE), convrot_status_string(CONVROT_OK)) != 0,
        "distinct status strings");

  /* workspace sizes: codes as bytes (M*K) then M scales, each 256-aligned */
  check(convrot_w4a4_workspace_size(76, 9728, 2560) == r256(76u * 2560u) + r256(76u * 4u), "w4a4 workspace");
  check(convrot_w4a4_workspace_size(76, 9728, 300) == 0, "w4a4 workspace: K % 256");
  check(w8a8_workspace_size(76, 1024, 2560, W8A8_CONVROT_INT8_ROW) == r256(76u * 2560u) + r256(76u * 4u) + 256,
        "w8a8 workspace");
  check(asym_w4a8_workspace_size(76, 1024, 2560) == r256(76u * 2560u) + r256(76u * 4u) + 256, "asym workspace");

  /* arguments rejected synchronously, before any device call */
  check(convrot_rotate_quant(NULL, 4, 256, good, good, NULL) == CONVROT_ERR_NULL, "rotate_quant NULL x");
  check(convrot_rotate_quant(good, 4, 300, good, good, NULL) == CONVROT_ERR_SHAPE, "rotate_quant K % 256");
  check(convrot_rotate_quant(bad, 4, 256, good, good, NULL) == CONVROT_ERR_ALIGN, "rotate_quant alignment");
  check(convrot_w4a4_linear(good, good, good, NULL, 4, 8, 256, good, good, 16, NULL) == CONVROT_ERR_WORKSPACE,
        "linear workspace too small");
  check(w8a8_gemm_s32(good, good, 4, 8, 300, good, NULL) == CONVROT_ERR_SHAPE, "w8a8 K % 256");
  check(asym_w4a8_gemm_s32(good, good, good, NULL, 4, 8, 256, good, NULL) == CONVROT_ERR_NULL, "asym NULL codebook");
  check(asym_w4a8_gemm_s32(good, good, good, good, 4, 12, 256, good, NULL) == CONVROT_ERR_SHAPE, "asym N % 8");

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
