"""The boundary is a C ABI: a plain C99 program includes include/nvfp4.h, links against the
library and calls its host-side entry points (no GPU needed for these)."""
import os
import shutil
import subprocess

import pytest

from nvfp4_block_scaled_14_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "nvfp4.h"

int main(void)
{
    if (nvfp4_codes_bytes(3, 64) != 96) return 1;
    if (nvfp4_scales_bytes(3, 64, 0) != 12) return 2;
    if (nvfp4_scales_bytes(3, 64, 1) != 512) return 3;
    if (nvfp4_workspace_bytes(NVFP4_OP_LINEAR_LOWRANK, 4096, 128, 0) != 4096u * 128u * 2u) return 4;
    if (strlen(nvfp4_status_str(NVFP4_ERR_SHAPE)) == 0) return 5;
    /* cols not a multiple of 32: rejected on the host before any device work */
    if (nvfp4_quantize((const void *)0x10000, NVFP4_BF16, 8, 48, NULL, (uint8_t *)0x10000,
                       (uint8_t *)0x10000, NULL, (float *)0x10000, (void *)0x10000, 4096, 0)
        != NVFP4_ERR_SHAPE) return 6;
    printf("c-abi ok\n");
    return 0;
}
"""


def test_header_compiles_as_c99_and_links(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = L.load()
    libpath = L.lib_path()
    src = tmp_path / "t.c"
    src.write_text(C_SRC)
    exe = tmp_path / "t"
    cuda_inc = "/usr/local/cuda/include"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
           "-I" + cuda_inc, str(src), "-o", str(exe), libpath,
           "-Wl,-rpath," + os.path.dirname(libpath)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and "c-abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)
    assert lib is not None
