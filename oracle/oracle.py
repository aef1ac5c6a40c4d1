"""Python face of the CPU oracle for the NVFP4 path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
module.  It never imports the CUDA library or anything from the product
package; the quantizer arithmetic lives in ``nvfp4_oracle.c`` (plain scalar C,
binary32, no FMA contraction), the GEMM reference is a float64 matrix product.

Sources (page title, section) are cited on each function; see the C file for
the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, IEEE semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            i64, u64, vp, fp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_float
            ci = ctypes.c_int
            L.nvfp4o_e2m1_value.restype = ctypes.c_double
            L.nvfp4o_e2m1_value.argtypes = [ci]
            L.nvfp4o_e4m3_value.restype = ctypes.c_double
            L.nvfp4o_e4m3_value.argtypes = [ci]
            L.nvfp4o_e2m1_rne.restype = ci
            L.nvfp4o_e2m1_rne.argtypes = [fp]
            L.nvfp4o_e2m1_sr.restype = ci
            L.nvfp4o_e2m1_sr.argtypes = [fp, ctypes.c_uint32]
            L.nvfp4o_e4m3_rne_satfinite.restype = ci
            L.nvfp4o_e4m3_rne_satfinite.argtypes = [fp]
            L.nvfp4o_philox4x32_10.restype = None
            L.nvfp4o_philox4x32_10.argtypes = [vp, vp, vp]
            L.nvfp4o_sr_bits.restype = ctypes.c_uint32
            L.nvfp4o_sr_bits.argtypes = [u64, u64]
            L.nvfp4o_rht_signs.restype = None
            L.nvfp4o_rht_signs.argtypes = [u64, vp]
            L.nvfp4o_rht16.restype = None
            L.nvfp4o_rht16.argtypes = [vp, vp, vp]
            L.nvfp4o_rht_signs_n.restype = None
            L.nvfp4o_rht_signs_n.argtypes = [u64, ci, vp]
            L.nvfp4o_rht_norm.restype = fp
            L.nvfp4o_rht_norm.argtypes = [ci]
            L.nvfp4o_rht_n.restype = None
            L.nvfp4o_rht_n.argtypes = [vp, vp, ci, vp]
            L.nvfp4o_amax_n.restype = fp
            L.nvfp4o_amax_n.argtypes = [vp, i64, i64, i64, ci, ci, u64]
            L.nvfp4o_quantize_1d_rows_n.restype = None
            L.nvfp4o_quantize_1d_rows_n.argtypes = [vp, i64, i64, i64, ci, ci, u64, ci, u64, fp, i64, i64, vp, vp]
            L.nvfp4o_quantize_1d_n.restype = None
            L.nvfp4o_quantize_1d_n.argtypes = [vp, i64, i64, i64, ci, ci, u64, ci, u64, vp, vp, vp]
            L.nvfp4o_global_scale.restype = fp
            L.nvfp4o_global_scale.argtypes = [fp]
            L.nvfp4o_block_scale_code.restype = ci
            L.nvfp4o_block_scale_code.argtypes = [fp, fp]
            L.nvfp4o_encode_element.restype = ci
            L.nvfp4o_encode_element.argtypes = [fp, fp, fp, ci, ctypes.c_uint32]
            L.nvfp4o_amax.restype = fp
            L.nvfp4o_amax.argtypes = [vp, i64, i64, i64, ci, ci, u64]
            L.nvfp4o_quantize_1d_rows.restype = None
            L.nvfp4o_quantize_1d_rows.argtypes = [vp, i64, i64, i64, ci, ci, u64, ci, u64, fp, i64, i64, vp, vp]
            L.nvfp4o_quantize_1d.restype = None
            L.nvfp4o_quantize_1d.argtypes = [vp, i64, i64, i64, ci, ci, u64, ci, u64, vp, vp, vp]
            L.nvfp4o_quantize_2d_tiles.restype = None
            L.nvfp4o_quantize_2d_tiles.argtypes = [vp, i64, i64, i64, fp, i64, i64, vp, vp, vp]
            L.nvfp4o_quantize_2d.restype = None
            L.nvfp4o_quantize_2d.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
            L.nvfp4o_e2m1_rne_batch.restype = None
            L.nvfp4o_e2m1_rne_batch.argtypes = [vp, i64, vp]
            L.nvfp4o_e2m1_sr_batch.restype = None
            L.nvfp4o_e2m1_sr_batch.argtypes = [vp, i64, u64, u64, vp]
            L.nvfp4o_e4m3_batch.restype = None
            L.nvfp4o_e4m3_batch.argtypes = [vp, i64, vp]
            L.nvfp4o_dequantize.restype = None
            L.nvfp4o_dequantize.argtypes = [vp, vp, ci, fp, i64, i64, vp]
            L.nvfp4o_mx_scale_exp.restype = ci
            L.nvfp4o_mx_scale_exp.argtypes = [fp]
            L.nvfp4o_e8m0_value.restype = ctypes.c_double
            L.nvfp4o_e8m0_value.argtypes = [ci]
            L.nvfp4o_mx_encode_element.restype = ci
            L.nvfp4o_mx_encode_element.argtypes = [fp, ci]
            L.nvfp4o_mx_quantize.restype = None
            L.nvfp4o_mx_quantize.argtypes = [vp, i64, i64, i64, vp, vp]
            L.nvfp4o_mx_dequantize.restype = None
            L.nvfp4o_mx_dequantize.argtypes = [vp, vp, i64, i64, vp]
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return x


# ---------------------------------------------------------------- scalars --
def e2m1_value(code: int) -> float:
    """E2M1 code -> value ("数据格式:极简的 E2M1"; "Four bits do not provide many choices")."""
    return lib().nvfp4o_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    """E4M3 (FN) code -> value ("精度核心:两级分层缩放")."""
    return lib().nvfp4o_e4m3_value(int(code))


def e2m1_rne(v: float) -> int:
    return lib().nvfp4o_e2m1_rne(float(v))


def e2m1_sr(v: float, u16: int) -> int:
    return lib().nvfp4o_e2m1_sr(float(v), int(u16))


def e4m3_rne_satfinite(s: float) -> int:
    return lib().nvfp4o_e4m3_rne_satfinite(float(s))


def e2m1_rne_array(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.zeros(v.size, dtype=np.uint8)
    lib().nvfp4o_e2m1_rne_batch(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_sr_array(v, seed: int, first_index: int = 0) -> np.ndarray:
    """SR encode of v[i] with the Philox bits of output index first_index + i."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.zeros(v.size, dtype=np.uint8)
    lib().nvfp4o_e2m1_sr_batch(_ptr(v), v.size, int(seed), int(first_index), _ptr(out))
    return out


def e4m3_array(s) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(s, dtype=np.float32).ravel())
    out = np.zeros(s.size, dtype=np.uint8)
    lib().nvfp4o_e4m3_batch(_ptr(s), s.size, _ptr(out))
    return out


def global_scale(amax: float) -> float:
    """s_global = amax / (448 * 6) ("Anatomi NVFP4: empat bit dengan dua tingkat skala")."""
    return lib().nvfp4o_global_scale(float(amax))


def block_scale_code(block_amax: float, s_global: float) -> int:
    return lib().nvfp4o_block_scale_code(float(block_amax), float(s_global))


def encode_element(y: float, s_dec: float, s_global: float, rounding: int = 0, u16: int = 0) -> int:
    return lib().nvfp4o_encode_element(float(y), float(s_dec), float(s_global), int(rounding), int(u16))


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 (Salmon et al., SC'11)."""
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    lib().nvfp4o_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sr_bits(seed: int, index: int) -> int:
    return lib().nvfp4o_sr_bits(int(seed), int(index))


def rht_signs(rht_seed: int) -> np.ndarray:
    d = np.zeros(16, dtype=np.float32)
    lib().nvfp4o_rht_signs(int(rht_seed), _ptr(d))
    return d


def rht16(x, d) -> np.ndarray:
    """One 16-point chunk of the random Hadamard transform, (1/4) H16 (d . x)."""
    xx = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    dd = np.ascontiguousarray(np.asarray(d, dtype=np.float32))
    y = np.zeros(16, dtype=np.float32)
    lib().nvfp4o_rht16(_ptr(xx), _ptr(dd), _ptr(y))
    return y


RHT_ORDERS = (16, 32, 64, 128)


def rht_signs_n(rht_seed: int, n: int) -> np.ndarray:
    """The n-point sign vector (n <= 128): d_j = -1 iff bit j % 32 of Philox word j // 32."""
    if n not in RHT_ORDERS:
        raise ValueError("RHT order must be one of 16, 32, 64, 128")
    d = np.zeros(n, dtype=np.float32)
    lib().nvfp4o_rht_signs_n(int(rht_seed), int(n), _ptr(d))
    return d


def rht_norm(n: int) -> np.float32:
    """RN(1/sqrt(n)) in binary32, the factor applied after the butterflies."""
    return np.float32(lib().nvfp4o_rht_norm(int(n)))


def rht_n(x, d) -> np.ndarray:
    """One n-point chunk of the random Hadamard transform, RN(1/sqrt(n)) H_n (d . x), n = len(x)."""
    xx = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    dd = np.ascontiguousarray(np.asarray(d, dtype=np.float32))
    n = xx.size
    if n not in RHT_ORDERS or dd.size != n:
        raise ValueError("RHT order must be one of 16, 32, 64, 128")
    y = np.zeros(n, dtype=np.float32)
    lib().nvfp4o_rht_n(_ptr(xx), _ptr(dd), int(n), _ptr(y))
    return y


def _rht_n_arg(rht: bool, rht_order: int) -> int:
    if not rht:
        return 0
    if rht_order not in RHT_ORDERS:
        raise ValueError("RHT order must be one of 16, 32, 64, 128")
    return int(rht_order)


# ---------------------------------------------------------------- tensors --
def amax(x: np.ndarray, transpose: bool = False, rht: bool = False, rht_seed: int = 0,
         rht_order: int = 16) -> float:
    """Tensor amax of the quantized tensor Q (x or x^T, rotated when rht)."""
    x = _bf16(x)
    rows, cols = x.shape
    return lib().nvfp4o_amax_n(_ptr(x), rows, cols, x.strides[0] // 2, int(transpose),
                               _rht_n_arg(rht, rht_order), int(rht_seed))


def quantize_1d(x: np.ndarray, transpose: bool = False, rht: bool = False, rht_seed: int = 0,
                rounding: int = 0, sr_seed: int = 0, rht_order: int = 16):
    """Whole-tensor 1D NVFP4 quantization of bf16 x [rows x cols].

    Returns (codes [Qr x Qc/2] uint8, scales [Qr x Qc/16] uint8, s_global float32),
    Q = x^T when ``transpose``.  Rounding 0 = RNE, 1 = SR.  With ``rht`` the
    Q rows are rotated in chunks of ``rht_order`` points (Qc a multiple of it).
    """
    x = np.ascontiguousarray(_bf16(x))
    rows, cols = x.shape
    qr, qc = (cols, rows) if transpose else (rows, cols)
    n = _rht_n_arg(rht, rht_order)
    if qc % 16 or (n and qc % n):
        raise ValueError("quantized rows must hold a multiple of 16 (and of the RHT order) elements")
    codes = np.zeros((qr, qc // 2), dtype=np.uint8)
    scales = np.zeros((qr, qc // 16), dtype=np.uint8)
    sg = np.zeros(1, dtype=np.float32)
    lib().nvfp4o_quantize_1d_n(_ptr(x), rows, cols, cols, int(transpose), n, int(rht_seed),
                               int(rounding), int(sr_seed), _ptr(codes), _ptr(scales), _ptr(sg))
    return codes, scales, np.float32(sg[0])


def quantize_1d_rows(x: np.ndarray, s_global: float, row_ids, transpose: bool = False,
                     rht: bool = False, rht_seed: int = 0, rounding: int = 0, sr_seed: int = 0,
                     rht_order: int = 16):
    """1D quantization of selected rows of Q given the tensor's global scale.

    Returns dicts {row: (codes_row, scales_row)} for each row id (sampling of
    large tensors: the oracle computes those rows one element at a time)."""
    x = _bf16(x)
    if not x.flags.c_contiguous:
        raise ValueError("contiguous input expected")
    rows, cols = x.shape
    qr, qc = (cols, rows) if transpose else (rows, cols)
    n = _rht_n_arg(rht, rht_order)
    if n and qc % n:
        raise ValueError("quantized rows must hold a multiple of the RHT order")
    out = {}
    codes = np.zeros((1, qc // 2), dtype=np.uint8)
    scales = np.zeros((1, qc // 16), dtype=np.uint8)
    for r in row_ids:
        r = int(r)
        lib().nvfp4o_quantize_1d_rows_n(_ptr(x), rows, cols, cols, int(transpose), n, int(rht_seed),
                                        int(rounding), int(sr_seed), float(s_global), r, r + 1,
                                        _ptr(codes), _ptr(scales))
        out[r] = (codes[0].copy(), scales[0].copy())
    return out


def quantize_2d(w: np.ndarray, columnwise: bool = True):
    """2D (16x16 tile) NVFP4 quantization of a bf16 weight, RNE.

    Returns (codes_row [R x C/2], codes_col [C x R/2] or None, scales [R/16 x C/16], s_global)."""
    w = np.ascontiguousarray(_bf16(w))
    rows, cols = w.shape
    if rows % 16 or cols % 16:
        raise ValueError("2D quantization needs both dimensions multiples of 16")
    cr = np.zeros((rows, cols // 2), dtype=np.uint8)
    cc = np.zeros((cols, rows // 2), dtype=np.uint8) if columnwise else None
    sc = np.zeros((rows // 16, cols // 16), dtype=np.uint8)
    sg = np.zeros(1, dtype=np.float32)
    lib().nvfp4o_quantize_2d(_ptr(w), rows, cols, cols, _ptr(cr), _ptr(cc) if cc is not None else None,
                             _ptr(sc), _ptr(sg))
    return cr, cc, sc, np.float32(sg[0])


def quantize_2d_tiles(w: np.ndarray, s_global: float, tile_row_ids):
    """2D quantization of selected 16-row tile rows; returns {tile_row: (codes_row[16 x C/2], scales[C/16])}."""
    w = _bf16(w)
    rows, cols = w.shape
    out = {}
    cr = np.zeros((16, cols // 2), dtype=np.uint8)
    sc = np.zeros((1, cols // 16), dtype=np.uint8)
    for tr in tile_row_ids:
        tr = int(tr)
        lib().nvfp4o_quantize_2d_tiles(_ptr(w), rows, cols, cols, float(s_global), tr, tr + 1,
                                       _ptr(cr), None, _ptr(sc))
        out[tr] = (cr.copy(), sc[0].copy())
    return out


def dequantize(codes: np.ndarray, scales: np.ndarray, scale_mode: int, s_global: float,
               rows: int, cols: int) -> np.ndarray:
    """x = value(code) * s_block * s_global in binary32
    ("The smallest example: the same payload, two real values")."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.float32)
    lib().nvfp4o_dequantize(_ptr(codes), _ptr(scales), int(scale_mode), float(s_global), rows, cols, _ptr(out))
    return out


def dequantize_f64(codes: np.ndarray, scales: np.ndarray, scale_mode: int, s_global: float,
                   rows: int, cols: int) -> np.ndarray:
    """Exact float64 reconstruction value(code) * s_dec * s_global (all three
    factors have short significands, so the product is exact in float64)."""
    codes = np.asarray(codes, dtype=np.uint8)
    lo = (codes & 0xF).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    c = np.empty((rows, cols), dtype=np.int64)
    c[:, 0::2] = lo[:, : cols // 2]
    c[:, 1::2] = hi[:, : cols // 2]
    e2m1 = np.array([e2m1_value(i) for i in range(16)], dtype=np.float64)
    e4m3 = np.array([e4m3_value(i) if i != 0x7F and i != 0xFF else np.nan for i in range(256)], dtype=np.float64)
    sc = np.asarray(scales, dtype=np.int64)
    if scale_mode == 0:
        s = np.repeat(sc, 16, axis=1)[:, :cols]
    else:
        s = np.repeat(np.repeat(sc, 16, axis=0), 16, axis=1)[:rows, :cols]
    return e2m1[c] * e4m3[s] * np.float64(s_global)


def gemm_reference(a_hat: np.ndarray, b_hat: np.ndarray):
    """C_ref = A_hat . B_hat^T and S = |A_hat| . |B_hat|^T in float64, the
    block-scaled GEMM's plain definition over dequantized operands (the
    hot contraction of "Presisi sebagai tombol throughput").  Returns (C_ref, S)."""
    a = np.asarray(a_hat, dtype=np.float64)
    b = np.asarray(b_hat, dtype=np.float64)
    return a @ b.T, np.abs(a) @ np.abs(b).T


# ------------------------------------------------------------------ MXFP4 ----
def mx_scale_exp(block_amax: float) -> int:
    """Exponent e of the block's power-of-two scale 2^e (E8M0 code e + 127):
    floor(log2(amax)) - 2, clamped to [-127, 127]; -127 for an all-zero block
    ("MXFP4 和 NVFP4 的区别", "MXFP4:开放标准,但精度较粗"; the OCP rule)."""
    return lib().nvfp4o_mx_scale_exp(float(block_amax))


def e8m0_value(code: int) -> float:
    return lib().nvfp4o_e8m0_value(int(code))


def mx_encode_element(x: float, e: int) -> int:
    return lib().nvfp4o_mx_encode_element(float(x), int(e))


def mx_quantize(x: np.ndarray):
    """MXFP4 quantization of bf16 bits x [rows x cols] (cols % 32 == 0):
    (codes [rows x cols/2], E8M0 scale codes [rows x cols/32])."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    lib().nvfp4o_mx_quantize(_ptr(x), rows, cols, cols, _ptr(codes), _ptr(scales))
    return codes, scales


def mx_dequantize(codes: np.ndarray, scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.float32)
    lib().nvfp4o_mx_dequantize(_ptr(codes), _ptr(scales), rows, cols, _ptr(out))
    return out


def mx_gemm_reference(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int):
    """float64 C = A_hat . B_hat^T of two MXFP4 operands and S = |A_hat| . |B_hat|^T."""
    a_hat = mx_dequantize(a_codes, a_scales, M, K).astype(np.float64)
    b_hat = mx_dequantize(b_codes, b_scales, N, K).astype(np.float64)
    return a_hat @ b_hat.T, np.abs(a_hat) @ np.abs(b_hat).T
