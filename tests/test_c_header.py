"""include/w8a8.h as a C interface: a C11 program that includes only the
header compiles warning-free, links against libw8a8.so, takes the address of
every function the header declares, and gets the documented status codes
from calls whose host-side checks fail before any CUDA call (the pointers
are fake and never dereferenced)."""
import os
import shutil
import subprocess

import pytest

from int8_gemm_token_b200 import w8a8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_CHECKS = r"""
#define P ((void *)0x10000)
#define EXPECT(call, code)                                                             \
  do {                                                                                 \
    w8a8_status s_ = (call);                                                           \
    if (s_ != (code)) {                                                                \
      printf("%s -> %s, want %s\n", #call, w8a8_status_string(s_), w8a8_status_string(code)); \
      ++fails;                                                                         \
    }                                                                                  \
  } while (0)

static int run_checks(void) {
  int fails = 0;
  EXPECT(w8a8_quant_per_token(P, 4, 15, 16, P, P, NULL), W8A8_ERR_UNSUPPORTED_SHAPE);
  EXPECT(w8a8_quant_per_token(P, 0, 32, 32, NULL, NULL, NULL), W8A8_OK);
  EXPECT(w8a8_quant_per_tensor(P, 4, 64, 64, NULL, P, P, NULL), W8A8_ERR_INVALID_ARG);
  EXPECT(w8a8_gemm_dequant(P, P, 1, NULL, P, P, NULL, NULL, 8, 8, 64, (char *)P + 8, W8A8_BF16, NULL, 0, NULL),
         W8A8_ERR_MISALIGNED);
  EXPECT(w8a8_gemm_dequant(P, P, 1, NULL, P, P, NULL, NULL, 8, 8, 64, P, 7, NULL, 0, NULL),
         W8A8_ERR_UNSUPPORTED_DTYPE);
  EXPECT(w8a8_linear_static(P, 40, 64, 64, P, P, P, P, P, P, NULL, 8, P, W8A8_BF16, NULL, 0, NULL),
         W8A8_ERR_WORKSPACE);
  EXPECT(w8a8_linear_static_requant(P, 65, 64, 64, P, P, P, P, P, P, NULL, 8, P, P, P, NULL, 0, NULL),
         W8A8_ERR_UNSUPPORTED_SHAPE);
  EXPECT(w8a8_gemm_requant(P, P, 0, P, P, P, P, NULL, 8, 8, 64, NULL, P, P, NULL), W8A8_ERR_INVALID_ARG);
  EXPECT(w8a8_linear_static_noalloc(P, 33, 64, 64, P, P, P, P, P, P, NULL, 8, P, W8A8_BF16, NULL),
         W8A8_ERR_UNSUPPORTED_SHAPE);
  EXPECT(int8_mixed_decomp_gemm(P, P, P, P, P, 8, P, P, P, 8, NULL, 8, 8, 64, P, W8A8_I32, NULL),
         W8A8_ERR_UNSUPPORTED_DTYPE);
  EXPECT(w8a8_quant_weight_per_channel(P, 5, 64, 8, 8, P, P, P, NULL), W8A8_ERR_UNSUPPORTED_DTYPE);
  EXPECT(w8a8_dequant_per_tensor(P, 4, 64, 64, P, P, P, W8A8_I32, NULL), W8A8_ERR_UNSUPPORTED_DTYPE);
  EXPECT(w8a8_check_device_error(NULL, NULL), W8A8_ERR_INVALID_ARG);
  if (strcmp(w8a8_status_string(W8A8_ERR_OUTLIER_OVERFLOW), "W8A8_ERR_OUTLIER_OVERFLOW") != 0) ++fails;
  if (strcmp(w8a8_status_string(12345), "W8A8_ERR_UNKNOWN") != 0) ++fails;
  return fails;
}
"""


def _program(symbols):
    addrs = ",\n  ".join(f"(fn_t){s}" for s in symbols)
    return ("#include <stdio.h>\n#include <string.h>\n#include \"w8a8.h\"\n"
            "typedef void (*fn_t)(void);\n"
            f"static const fn_t every_entry_point[] = {{\n  {addrs}\n}};\n"
            + C_CHECKS +
            "int main(void) {\n"
            "  size_t n = sizeof every_entry_point / sizeof every_entry_point[0];\n"
            "  for (size_t i = 0; i < n; ++i)\n"
            "    if (!every_entry_point[i]) return 2;\n"
            "  int fails = run_checks();\n"
            "  printf(fails ? \"FAIL\\n\" : \"OK\\n\");\n"
            "  return fails != 0;\n"
            "}\n")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c_and_links(tmp_path):
    w8a8.lib()  # the library exists (raises otherwise)
    symbols = w8a8.header_symbols()
    src = tmp_path / "abi.c"
    src.write_text(_program(symbols))
    exe = tmp_path / "abi"
    libdir = os.path.dirname(w8a8.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                         "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                         "-L", libdir, "-l:" + os.path.basename(w8a8.LIB_PATH), "-Wl,-rpath," + libdir],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip().endswith("OK"), run.stdout + run.stderr
