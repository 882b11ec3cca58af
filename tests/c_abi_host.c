/* Plain C99 client of the library: includes the public header, links the shared library and
 * calls the entry points that need no GPU (sizes, version, host-side argument checks).  Built
 * and run by tests/test_c_client.py; prints one line per check and returns non-zero on a
 * failure. */
#include <stdio.h>
#include <string.h>

#include "nvfp4_moe.h"

static int failures = 0;

static void check(int ok, const char* what) {
  printf("%s %s\n", ok ? "ok  " : "FAIL", what);
  if (!ok) ++failures;
}

int main(void) {
  void* fake = (void*)(uintptr_t)(1u << 20); /* never dereferenced: every call fails its checks */
  check(nvfp4_abi_version() == 1, "abi version");
  check(nvfp4_quantize_workspace_size() == 256, "quantize workspace");
  check(moe_rows_max(16, 256, 8) == 128 + 127 * 128, "rows max, decode");
  check(moe_rows_max(0, 8, 2) == 0, "rows max, no tokens");
  check(nvfp4_rmsnorm_quantize_workspace_size(8192) == 256 + 8192 * 4, "rmsnorm workspace");
  check(nvfp4_linear_workspace_size(-1, 4096, 7168) == 0, "linear workspace, bad M");
  check(moe_ffn_workspace_size(-1, 7168, 2048, 256, 8) == 0, "ffn workspace, bad T");
  /* host validation: cols % 64 -> unsupported shape, before any launch */
  check(nvfp4_quantize(fake, 4, 65, 65, NULL, 1, 4, fake, fake, fake, 1, fake, 256, NULL,
                       NULL) == NVFP4_ERR_UNSUPPORTED_SHAPE, "quantize rejects cols % 64");
  check(nvfp4_linear(fake, 16, 128, 128, NULL, 0.0f, fake, fake, fake, 200, fake, fake,
                     (size_t)1 << 40, NULL, NULL) == NVFP4_ERR_UNSUPPORTED_SHAPE,
        "linear rejects N % 256");
  check(nvfp4_shared_expert(fake, 16, 256, 256, NULL, 0.0f, fake, fake, fake, fake, fake, fake,
                            128, fake, fake, fake, 100, NULL, NULL) ==
            NVFP4_ERR_WORKSPACE_TOO_SMALL,
        "shared expert rejects a small workspace");
  {
    int32_t map[64];
    check(moe_w1_row_map(32, map) == NVFP4_OK && map[0] == 0 && map[16] == 32 && map[32] == 16,
          "W1 row map");
  }
  /* the FFN's L2 form: slot rows below 32 routed rows per expert, token-row reductions from
     there unless the deterministic flag is given */
  check(moe_ffn_l2_form(16, 8, 256, 0) == 0 && moe_ffn_l2_form(8192, 8, 256, 0) == 1 &&
            moe_ffn_l2_form(8192, 8, 256, NVFP4_FFN_DETERMINISTIC) == 0,
        "FFN L2 form");
  check(moe_ffn_forward_ex(fake, fake, 16, 7168, 2048, 256, 8, fake, fake, fake, fake, fake, fake,
                           fake, 4, NULL, fake, fake, (size_t)1 << 40, NULL, NULL) ==
            NVFP4_ERR_INVALID_ARG,
        "FFN rejects unknown flags");
  check(mxfp4_quantize(fake, 4, 96, 96, fake, fake, NULL, NULL) == NVFP4_ERR_UNSUPPORTED_SHAPE,
        "MXFP4 quantize rejects cols % 128");
  check(mxfp4_grouped_gemm(fake, fake, fake, fake, fake, 2, 256, 192, 128, fake, 0, NULL, NULL) ==
            NVFP4_ERR_UNSUPPORTED_SHAPE,
        "MXFP4 GEMM rejects K % 128");
  check(nvfp4_last_error() != NULL, "last error string");
  return failures == 0 ? 0 : 1;
}
