"""The C-ABI library: loads without a GPU, exports every declared symbol, and
rejects bad arguments on the host before any launch (no compute here)."""
import ctypes
import os
import re

import pytest

from nvfp4_bit_block_amax_b200 import build as B
from nvfp4_bit_block_amax_b200 import nvfp4 as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return N.lib()


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ("nvfp4_quantize_1d", "nvfp4_quantize_2d", "nvfp4_rht_quantize_sr", "nvfp4_dequantize",
                 "nvfp4_gemm"):
        assert name in syms


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert set(declared_symbols()) <= set(N.EXPORTS) | {"nvfp4_status_string"}


def test_version_and_status_strings(L):
    assert N.nvfp4_version() == 101
    for s in range(7):
        assert N.nvfp4_status_string(s)
    assert "unknown" in N.nvfp4_status_string(99)


def test_sizes(L):
    assert N.nvfp4_workspace_size(1, 16) >= 4096 * 4
    assert N.nvfp4_mma_scale_bytes(1, 16) == 512
    assert N.nvfp4_mma_scale_bytes(128, 256) == 512 * 4
    assert N.nvfp4_mma_scale_bytes(129, 256) == 512 * 8
    assert N.nvfp4_mma_scale_bytes(256, 320) == 2 * 5 * 512
    assert N.nvfp4_mma_scale_bytes(16, 8) == 0


FAKE = 1 << 20          # a 16-byte aligned address that is never dereferenced: every call below
WS = 1 << 14            # fails validation before touching the device


def q1d(L, **kw):
    a = dict(x=FAKE, rows=32, cols=64, ld=64, tr=0, rnd=0, seed=0, codes=FAKE, scales=FAKE, mma=None,
             gs=FAKE, ws=FAKE, wsb=WS)
    a.update(kw)
    return L.nvfp4_quantize_1d(a["x"], a["rows"], a["cols"], a["ld"], a["tr"], a["rnd"], a["seed"], a["codes"],
                               a["scales"], a["mma"], a["gs"], a["ws"], a["wsb"], None)


def test_quantize_1d_validation(L):
    assert q1d(L, x=None) == 1
    assert q1d(L, codes=None) == 1
    assert q1d(L, scales=None, mma=None) == 1
    assert q1d(L, rows=0) == 1
    assert q1d(L, ld=32) == 1
    assert q1d(L, rnd=2) == 1
    assert q1d(L, tr=3) == 1
    assert q1d(L, cols=40, ld=40) == 2            # blocks of 16 along the row
    assert q1d(L, tr=1, rows=40) == 2             # transposed: rows hold the blocks
    assert q1d(L, x=FAKE + 2) == 3
    assert q1d(L, ld=68, cols=64) == 3
    assert q1d(L, ws=None) == 6
    assert q1d(L, wsb=16) == 6


def test_quantize_2d_and_rht_validation(L):
    assert L.nvfp4_quantize_2d(FAKE, 40, 64, 64, FAKE, None, FAKE, None, None, FAKE, FAKE, WS, None) == 2
    assert L.nvfp4_quantize_2d(FAKE, 32, 64, 64, None, None, FAKE, None, None, FAKE, FAKE, WS, None) == 1
    assert L.nvfp4_quantize_2d(FAKE, 32, 64, 64, FAKE + 8, None, FAKE, None, None, FAKE, FAKE, WS, None) == 3
    assert L.nvfp4_rht_quantize_sr(FAKE, 32, 64, 64, 0, 1, 5, 1, FAKE, FAKE, None, FAKE, FAKE, WS, None) == 1
    assert L.nvfp4_rht_quantize_sr(FAKE, 30, 64, 64, 1, 1, 1, 1, FAKE, FAKE, None, FAKE, FAKE, WS, None) == 2


def test_dequantize_gemm_validation(L):
    assert L.nvfp4_dequantize(FAKE, FAKE, 0, FAKE, 4, 40, 0, FAKE, None) == 2
    assert L.nvfp4_dequantize(FAKE, FAKE, 1, FAKE, 8, 32, 0, FAKE, None) == 2
    assert L.nvfp4_dequantize(FAKE, FAKE, 2, FAKE, 16, 32, 0, FAKE, None) == 1
    assert L.nvfp4_dequantize(FAKE, FAKE, 0, FAKE, 16, 32, 5, FAKE, None) == 1
    g = lambda **kw: L.nvfp4_gemm(kw.get("a", FAKE), FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("M", 128),
                                  kw.get("N", 128), kw.get("K", 256), kw.get("dt", 1), kw.get("c", FAKE),
                                  kw.get("ldc", 128), None)
    assert g(a=None) == 1
    assert g(M=0) == 1
    assert g(K=96) == 2
    assert g(ldc=64) == 1
    assert g(ldc=132) == 3
    assert g(c=FAKE + 4) == 3
    assert g(dt=7) == 1
    assert L.nvfp4_scales_to_mma(FAKE, 1, 20, 64, FAKE, None) == 2


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(N, "_lib", None)
    monkeypatch.setattr(N, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(OSError):
        N.lib()


def test_python_constants_match_header_enums():
    """The binding's status / mode constants carry the header's values."""
    import re
    hdr = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    for name, value in re.findall(r"\b(NVFP4_[A-Z0-9_]+) = (\d+)", hdr):
        assert getattr(N, name) == int(value), name


def rhtn(L, **kw):
    a = dict(x=FAKE, rows=256, cols=64, ld=64, tr=1, order=64, seed=0, rnd=0, sr=0, codes=FAKE, scales=FAKE,
             mma=None, gs=FAKE, ws=FAKE, wsb=WS)
    a.update(kw)
    return L.nvfp4_rht_quantize_n(a["x"], a["rows"], a["cols"], a["ld"], a["tr"], a["order"], a["seed"], a["rnd"],
                                  a["sr"], a["codes"], a["scales"], a["mma"], a["gs"], a["ws"], a["wsb"], None)


def test_rht_quantize_n_validation(L):
    for order in (0, 8, 48, 256, -16):
        assert rhtn(L, order=order) == N.NVFP4_ERR_INVALID_ARG, order
    assert rhtn(L, rows=192, order=128) == N.NVFP4_ERR_UNSUPPORTED_SHAPE      # tokens not a multiple of 128
    assert rhtn(L, tr=0, rows=32, cols=96, ld=96, order=64) == N.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert rhtn(L, x=None) == N.NVFP4_ERR_INVALID_ARG                            # common checks first
    assert rhtn(L, x=FAKE + 2) == N.NVFP4_ERR_MISALIGNED


def test_dual_from_amax_and_gemm_amax_validation(L):
    d = lambda **kw: L.nvfp4_quantize_dual(
        kw.get("x", FAKE), 32, 64, 64, kw.get("rnd", 1), 0, FAKE, FAKE, None, FAKE, 5, 6, kw.get("ct", FAKE), FAKE,
        None, kw.get("gt", FAKE), FAKE, kw.get("wsb", WS), None)
    assert d(x=None) == N.NVFP4_ERR_INVALID_ARG
    assert d(ct=None) == N.NVFP4_ERR_INVALID_ARG             # the transposed half is checked too
    assert d(gt=None) == N.NVFP4_ERR_INVALID_ARG
    assert d(rnd=3) == N.NVFP4_ERR_INVALID_ARG
    assert d(ct=FAKE + 4) == N.NVFP4_ERR_MISALIGNED
    assert d() == N.NVFP4_ERR_WORKSPACE                       # one workspace's worth is not enough for two
    q = lambda **kw: L.nvfp4_quantize_1d_from_amax(FAKE, 32, 64, 64, 0, 0, 0, kw.get("amax", FAKE), FAKE, FAKE,
                                                   None, FAKE, None)
    assert q(amax=None) == N.NVFP4_ERR_INVALID_ARG and q(amax=FAKE + 2) == N.NVFP4_ERR_MISALIGNED
    w = lambda **kw: L.nvfp4_quantize_2d_from_amax(FAKE, 32, 64, 64, kw.get("amax", FAKE), FAKE, None, FAKE, None,
                                                   None, FAKE, None)
    assert w(amax=None) == N.NVFP4_ERR_INVALID_ARG and w(amax=FAKE + 2) == N.NVFP4_ERR_MISALIGNED
    g = lambda **kw: L.nvfp4_gemm_amax(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 128, kw.get("K", 256), 1, FAKE, 128,
                                       kw.get("amax", FAKE), None)
    assert g(amax=None) == N.NVFP4_ERR_INVALID_ARG and g(amax=FAKE + 2) == N.NVFP4_ERR_MISALIGNED
    assert g(K=96) == N.NVFP4_ERR_UNSUPPORTED_SHAPE


def test_mxfp4_and_selftest_validation(L):
    assert L.nvfp4_mxfp4_quantize(FAKE, 4, 48, 48, FAKE, FAKE, None, None) == N.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_mxfp4_quantize(None, 4, 64, 64, FAKE, FAKE, None, None) == N.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_mxfp4_quantize(FAKE, 4, 64, 64, FAKE, None, None, None) == N.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_mxfp4_quantize(FAKE, 4, 64, 64, FAKE + 8, FAKE, None, None) == N.NVFP4_ERR_MISALIGNED
    assert L.nvfp4_mxfp4_dequantize(FAKE, FAKE, 4, 64, 9, FAKE, None) == N.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_mxfp4_dequantize(FAKE, FAKE, 4, 40, 0, FAKE, None) == N.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_mxfp4_gemm(FAKE, FAKE, FAKE, FAKE, 128, 128, 96, 1, FAKE, 128, None) == \
        N.NVFP4_ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_mxfp4_gemm(None, FAKE, FAKE, FAKE, 128, 128, 256, 1, FAKE, 128, None) == N.NVFP4_ERR_INVALID_ARG
    for limit in (0, 999, 2000000001):
        assert L.nvfp4_selftest_wait_timeout(limit, None) == N.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_quantize_1d_noalloc(None, 32, 64, 64, 0, 0, 0, FAKE, FAKE, None, FAKE, None) == \
        N.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_quantize_1d_noalloc(FAKE, 32, 40, 40, 0, 0, 0, FAKE, FAKE, None, FAKE, None) == \
        N.NVFP4_ERR_UNSUPPORTED_SHAPE


def test_noalloc_refuses_a_grid_beyond_its_scratch(L, monkeypatch):
    """The allocation-free quantizer holds 1024 amax partials; its amax pass
    takes up to 4 CTAs per SM.  With the SM count overridden to 300 a large
    tensor would need 1200 partials: the call must say NVFP4_ERR_WORKSPACE,
    enqueue nothing and leave its outputs untouched.  The outputs here are
    host buffers standing in for device ones (nothing may write them); the
    refusal happens before any CUDA call, so no GPU is needed."""
    import numpy as np
    rows, cols = 4096, 4096                   # 2M 16-byte vectors: 2048 CTAs wanted
    codes = np.full(rows * cols // 2 + 64, 0xAB, dtype=np.uint8)
    scales = np.full(rows * cols // 16 + 64, 0xAB, dtype=np.uint8)
    gs = np.full(16, 0xAB, dtype=np.uint8)
    al = lambda a: (a.ctypes.data + 15) & ~15
    before = L.nvfp4_kernel_launches()
    monkeypatch.setenv("NVFP4_SM_COUNT", "300")
    st = L.nvfp4_quantize_1d_noalloc(FAKE, rows, cols, cols, 0, 0, 0, al(codes), al(scales), None, al(gs), None)
    assert st == N.NVFP4_ERR_WORKSPACE
    assert L.nvfp4_kernel_launches() == before
    assert (codes == 0xAB).all() and (scales == 0xAB).all() and (gs == 0xAB).all()
