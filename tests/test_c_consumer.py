"""A plain C program built against include/moe_qmm.h and linked to the library:
the header is valid C99 and every call below runs on the host only (validation
rejects the arguments before any CUDA call, or the call is host-side)."""

import os
import shutil
import subprocess

import pytest

import moe_expert_routed_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "moe_qmm.h"

int main(void) {
    moe_qmm_plan plan;
    static char ws[256] __attribute__((aligned(16)));  /* the workspace must be 16-byte aligned */
    int fails = 0;
    /* sizes */
    if (moe_packed_row_bytes(MOE_FMT_AFFINE, 4, 2816) != 1408) fails++;
    if (moe_packed_row_bytes(MOE_FMT_AFFINE, 6, 2048) != 1536) fails++;
    if (moe_packed_row_bytes(MOE_FMT_CODEBOOK, 3, 2816) != 1128) fails++;
    if (moe_packed_row_bytes(MOE_FMT_NVFP4, 4, 4096) != 2048) fails++;
    if (moe_packed_row_bytes(MOE_FMT_MXFP4, 4, 4096) != 2048) fails++;
    if (moe_qmm_id_workspace_bytes(1, 8, 128) == 0) fails++;
    /* validation before any CUDA call */
    if (moe_qmm_id(0, 0, 0, 0, 0, 0, 1, 64, 8, 32, 4, MOE_FMT_AFFINE, 1, 1, MOE_BF16, MOE_F32, ws, sizeof ws,
                   0) != MOE_ERR_INVALID_ARGUMENT) fails++;
    if (moe_qmm_id_glu(ws, (const uint32_t *)ws, ws, ws, ws, 0, ws, 1, 64, 7, 32, 4, MOE_FMT_AFFINE, 1, 1,
                       MOE_BF16, MOE_F32, MOE_F32, MOE_ACT_SILU, ws, sizeof ws, 0, MOE_PATH_AUTO)
        != MOE_ERR_INVALID_ARGUMENT) fails++;
    if (moe_qmm_plan_init(&plan, ws, ws, ws, 0, 1, 64, 8, 32, 4, MOE_FMT_AFFINE, 1, 1, MOE_BF16, MOE_F32,
                          MOE_F32, -1, ws, 16, (moe_path)(MOE_PATH_AUTO | MOE_LAUNCH_PDL))
        != MOE_ERR_WORKSPACE_TOO_SMALL) fails++;
    if (moe_qmm_plan_run(&plan, ws, (const uint32_t *)ws, ws, 0) != MOE_ERR_INVALID_ARGUMENT) fails++;
    printf("%s|%d\n", moe_status_str(MOE_ERR_BAD_EXPERT_POINTER), fails);
    return fails != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_against_header_and_library(tmp_path):
    M.lib()  # the library is built and loadable
    libdir = os.path.dirname(M.LIB_PATH)
    src = tmp_path / "consumer.c"
    exe = tmp_path / "consumer"
    src.write_text(PROGRAM)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), "-L", libdir, "-l:libmoe_qmm.so",
                           f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    msg, fails = out.stdout.strip().rsplit("|", 1)
    assert fails == "0" and "pointer-table" in msg
