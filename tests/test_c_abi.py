"""The boundary is a C ABI: a plain C99 program includes include/fp8q.h,
links libfp8q.so and calls the host-only entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fp8_dynamic_quantization_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp8q.h"

int main(void) {
    int plan[11];
    size_t ws = 0;
    if (fp8q_abi_version() >> 16 != 1) return 1;
    if (strcmp(fp8q_status_string(FP8Q_ERR_MISALIGNED), "FP8Q_ERR_MISALIGNED") != 0) return 2;
    if (fp8q_gemm_plan(4096, 7168, 7168, 148, (size_t)-1, plan, &ws) != FP8Q_OK) return 3;
    if (fp8q_gemm_plan(4, 4, 100, 148, (size_t)-1, plan, &ws) != FP8Q_ERR_UNSUPPORTED_SHAPE) return 4;
    /* arguments are checked on the host before any device is touched */
    if (fp8_act_quant_group128((const void*)0, 4, 128, 128, (uint8_t*)0, 128, (float*)0, (void*)0)
        != FP8Q_ERR_INVALID_ARG) return 5;
    printf("pair=%d bn=%d splits=%d tail=%dx%d ws=%zu\n", plan[1], plan[2], plan[4], plan[9], plan[10], ws);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_links_and_calls_the_library(cuda_lib, tmp_path):
    src = tmp_path / "use_fp8q.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_fp8q"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", PKG, "-l:libfp8q.so", f"-Wl,-rpath,{PKG}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == f"pair=1 bn=256 splits=1 tail=4x18 ws={4 * 18 * 256 * 256 * 4}"
