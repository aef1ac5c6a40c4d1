"""A plain C program drives the path on the GPU through include/nvfp4.h: it
allocates device memory with cudaMalloc, quantizes the tiny linear's
activation (1D, RNE) and weight (2D, both code layouts), runs the
block-scaled GEMM and dequantizes, then writes the results to files.  Python
only generates the inputs and checks the outputs against the oracle
(quantizers bit for bit, GEMM within 2e-3 * sum |a b|).  No torch, no ctypes:
the C ABI alone."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from nvfp4_bit_block_amax_b200 import build as B
from nvfp4_bit_block_amax_b200 import inputs as G
from oracle import oracle as O

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime.h>
#include "nvfp4.h"

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
    fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 2; } } while (0)
#define NV(x) do { nvfp4_status s_ = (x); if (s_ != NVFP4_OK) { \
    fprintf(stderr, "%s: %s\n", #x, nvfp4_status_string(s_)); return 3; } } while (0)

static int rd(const char* dir, const char* name, void* p, size_t n) {
    char path[4096]; snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "rb"); if (!f) return 1;
    size_t got = fread(p, 1, n, f); fclose(f); return got != n;
}
static int wr(const char* dir, const char* name, const void* p, size_t n) {
    char path[4096]; snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "wb"); if (!f) return 1;
    size_t put = fwrite(p, 1, n, f); fclose(f); return put != n;
}

int main(int argc, char** argv) {
    const char* dir = argv[1];
    const int64_t M = 256, N = 256, K = 256;
    const size_t in_bytes = (size_t)M * K * 2;
    void* ha = malloc(in_bytes); void* hw = malloc(in_bytes);
    if (rd(dir, "a.bin", ha, in_bytes) || rd(dir, "w.bin", hw, in_bytes)) return 1;
    void *da, *dw, *ws, *dc, *dq;
    uint8_t *ac, *as, *asm_, *wc, *wcc, *wsc, *wsm;
    float* gs;
    const size_t wsb = nvfp4_workspace_size(M, K);
    const size_t mb = nvfp4_mma_scale_bytes(M, K);
    CK(cudaMalloc(&da, in_bytes)); CK(cudaMalloc(&dw, in_bytes)); CK(cudaMalloc(&ws, wsb));
    CK(cudaMalloc((void**)&ac, M * K / 2)); CK(cudaMalloc((void**)&as, M * K / 16)); CK(cudaMalloc((void**)&asm_, mb));
    CK(cudaMalloc((void**)&wc, N * K / 2)); CK(cudaMalloc((void**)&wcc, N * K / 2));
    CK(cudaMalloc((void**)&wsc, (N / 16) * (K / 16))); CK(cudaMalloc((void**)&wsm, mb));
    CK(cudaMalloc((void**)&gs, 2 * sizeof(float)));
    CK(cudaMalloc(&dc, (size_t)M * N * 4)); CK(cudaMalloc(&dq, (size_t)M * K * 4));
    CK(cudaMemcpy(da, ha, in_bytes, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(dw, hw, in_bytes, cudaMemcpyHostToDevice));
    NV(nvfp4_quantize_1d(da, M, K, K, 0, NVFP4_RNE, 0, ac, as, asm_, gs, ws, wsb, NULL));
    NV(nvfp4_quantize_2d(dw, N, K, K, wc, wcc, wsc, wsm, NULL, gs + 1, ws, wsb, NULL));
    NV(nvfp4_gemm(ac, asm_, gs, wc, wsm, gs + 1, M, N, K, NVFP4_OUT_F32, dc, N, NULL));
    NV(nvfp4_dequantize(ac, as, NVFP4_SCALE_1D, gs, M, K, NVFP4_OUT_F32, dq, NULL));
    NV(nvfp4_get_error(NULL));
    uint8_t* h = malloc((size_t)M * N * 4);
#define OUT(ptr, n, name) CK(cudaMemcpy(h, ptr, n, cudaMemcpyDeviceToHost)); if (wr(dir, name, h, n)) return 1
    OUT(ac, M * K / 2, "a_codes.bin");
    OUT(as, M * K / 16, "a_scales.bin");
    OUT(wc, N * K / 2, "w_codes.bin");
    OUT(wcc, N * K / 2, "w_codes_col.bin");
    OUT(wsc, (N / 16) * (K / 16), "w_scales.bin");
    OUT(gs, 2 * sizeof(float), "gs.bin");
    OUT(dc, (size_t)M * N * 4, "c.bin");
    OUT(dq, (size_t)M * K * 4, "a_deq.bin");
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_c_program_runs_the_path_on_the_gpu(tmp_path):
    lib = B.build()
    src = tmp_path / "linear.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "linear"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(CUDA, "include"), str(src), lib, "-L", os.path.join(CUDA, "lib64"),
                           "-lcudart", "-Wl,-rpath," + os.path.dirname(lib), "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
                           "-o", str(exe)])
    a_bits, w_bits = G.tiny_linear()
    a_bits.tofile(tmp_path / "a.bin")
    w_bits.tofile(tmp_path / "w.bin")
    out = subprocess.run([str(exe), str(tmp_path)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    ld = lambda name, dt, shape: np.fromfile(tmp_path / name, dtype=dt).reshape(shape)
    ca, sa, ga = O.quantize_1d(a_bits)
    cw, ccw, sw, gw = O.quantize_2d(w_bits)
    assert np.array_equal(ld("a_codes.bin", np.uint8, ca.shape), ca)
    assert np.array_equal(ld("a_scales.bin", np.uint8, sa.shape), sa)
    assert np.array_equal(ld("w_codes.bin", np.uint8, cw.shape), cw)
    assert np.array_equal(ld("w_codes_col.bin", np.uint8, ccw.shape), ccw)
    assert np.array_equal(ld("w_scales.bin", np.uint8, sw.shape), sw)
    gs = ld("gs.bin", np.float32, (2,))
    assert gs[0] == ga and gs[1] == gw
    deq = ld("a_deq.bin", np.float32, (256, 256))
    assert np.array_equal(deq.view(np.uint32), O.dequantize(ca, sa, 0, ga, 256, 256).view(np.uint32))
    ref, s = O.gemm_reference(O.dequantize_f64(ca, sa, 0, ga, 256, 256), O.dequantize_f64(cw, sw, 1, gw, 256, 256))
    c = ld("c.bin", np.float32, (256, 256)).astype(np.float64)
    assert (np.abs(c - ref) <= 2e-3 * s).all()
