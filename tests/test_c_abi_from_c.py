"""The boundary is a plain C ABI: a C99 program includes include/nvfp4.h,
links libnvfp4.so and calls the host-only entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from nvfp4_bit_block_amax_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "nvfp4.h"
int main(void) {
    /* host-only calls: version, sizes, status names, and an argument error */
    printf("%d|%zu|%zu|%s|%d\n", nvfp4_version(), nvfp4_mma_scale_bytes(129, 256),
           nvfp4_workspace_size(16, 16), nvfp4_status_string(NVFP4_ERR_UNSUPPORTED_SHAPE),
           (int)nvfp4_quantize_1d(NULL, 16, 16, 16, 0, NVFP4_RNE, 0, NULL, NULL, NULL, NULL, NULL, 0, NULL));
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_c_program_links_and_calls(tmp_path):
    lib = B.build()
    src = tmp_path / "main.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "main"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), lib,
                           "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    version, mma, ws, name, status = out.stdout.strip().split("|")
    assert int(version) == 101 and int(mma) == 512 * 8 and int(ws) >= 4096 * 4
    assert "shape" in name.lower() or "unsupported" in name.lower()
    assert int(status) == 1          # NVFP4_ERR_INVALID_ARG: null input
