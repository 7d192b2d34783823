"""The boundary is a C ABI: the header compiles as strict C99, and a plain C program
links against the library and calls its host-only entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import adapter_gemv_sgmv_b200 as L
from adapter_gemv_sgmv_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "lora_sgmv.h"

int main(void)
{
    lora_pool p;
    memset(&p, 0, sizeof p);
    /* host validation: a null pool is an invalid argument, nothing is launched */
    if (lora_bgmv(0, 64, 0, 64, 0, 0, 4, 1.0f, 0, 0, 0) != LORA_ERR_INVALID_ARG)
        return 1;
    if (lora_workspace_size(LORA_OP_LINEAR, 1000, 64, 4096, 14336, 64, 8, 0) < 1000u * 2u * 64u * 2u)
        return 2;
    if (lora_kernel_launches(LORA_OP_LINEAR, 1000, 64, 4096, 8) != 3)
        return 3;
    printf("%s\n", lora_version());
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_plain_c_program_links_and_calls_host_entry_points(tmp_path):
    B.build()
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(L.library_path())
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", lib_dir, "-llora_sgmv", f"-Wl,-rpath,{lib_dir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert "sm_100a" in out.stdout
