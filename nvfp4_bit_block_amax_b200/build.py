"""Build libnvfp4.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m nvfp4_bit_block_amax_b200.build [--force]

The quantizer translation unit is compiled with --fmad=false so that every
floating-point step stays a single IEEE binary32 operation (the quantized
codes are specified bit for bit).  No fast-math, no flush-to-zero.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libnvfp4.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "-I", os.path.join(ROOT, "include")]
UNITS = {
    "quant.cu": ["--fmad=false"],
    "gemm.cu": [],
    "mxfp4.cu": [],
    "api.cu": [],
}
HEADERS = ["common.cuh", "internal.h"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libnvfp4.so")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, u) for u in UNITS] + [os.path.join(CSRC, h) for h in HEADERS]
    srcs.append(os.path.join(ROOT, "include", "nvfp4.h"))
    srcs.append(os.path.abspath(__file__))
    return any(os.path.getmtime(s) > t for s in srcs)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    nvcc = _nvcc()
    with tempfile.TemporaryDirectory(prefix="nvfp4_build_") as tmp:
        objs = []
        for unit, extra in UNITS.items():
            obj = os.path.join(tmp, unit.replace(".cu", ".o"))
            cmd = [nvcc, *ARCH, *COMMON, *extra, "-c", os.path.join(CSRC, unit), "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
            objs.append(obj)
        out = os.path.join(tmp, "libnvfp4.so")
        subprocess.check_call([nvcc, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", out])
        tmp_lib = LIB + f".tmp{os.getpid()}"
        shutil.copyfile(out, tmp_lib)
        os.replace(tmp_lib, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
