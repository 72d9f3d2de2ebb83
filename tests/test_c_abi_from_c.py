"""The boundary is a plain C ABI: a C99 program that includes only
include/fp4.h links libfp4.so and calls its host-side entry points (no GPU
needed: sizes, status strings, a call refused by validation before any
launch)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp4.h"

int main(void)
{
    size_t q = 0, s = 0;
    if (fp4_quantize_sizes(200, 320, FP4_NVFP4, 16, &q, &s) != FP4_OK) return 1;
    if (q != 200 * 160 || s != 256 * 20) return 2;
    if (fp4_quantize_sizes(4, 64, FP4_MXFP4_16, 16, &q, &s) != FP4_OK || s != 128 * 4) return 3;
    if (strncmp(fp4_status_string(FP4_ERR_UNSUPPORTED), "FP4_ERR_UNSUPPORTED", 19) != 0) return 4;
    /* K not a multiple of 32: refused on the host, nothing launched */
    if (fp4_gemm(NULL, NULL, NULL, NULL, NULL, NULL, 4, 8, 100, FP4_MXFP4, FP4_OUT_BF16, NULL, 8, NULL, 0,
                 NULL) != FP4_ERR_UNSUPPORTED)
        return 5;
    printf("ok %llu\n", (unsigned long long)fp4_kernel_launches());
    return 0;
}
"""


def test_c_program_links_and_calls_the_abi(tmp_path):
    from fp4_microscaling_quantization_b200 import build
    lib = build.build()
    src = tmp_path / "use_fp4.c"
    src.write_text(PROGRAM)
    exe = str(tmp_path / "use_fp4")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-o", exe,
                           str(src), lib, "-Wl,-rpath," + os.path.dirname(lib)])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok 0")
