"""Thin Python binding of libnvfp4.so (ctypes).

The functions named ``nvfp4_*`` mirror the C ABI in include/nvfp4.h one to
one: arguments are marshalled (torch tensors -> device pointers, the current
torch stream -> cudaStream_t) and the status is turned into an exception.
Every step of the NVFP4 path runs in the library's CUDA kernels; there is no
fallback of any kind -- if the library cannot be loaded, calls raise.

The lower-case helpers (``quantize_1d`` ...) only allocate the outputs with
torch (PyTorch is used for device memory and streams) and call the C ABI.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

NVFP4_OK = 0
(NVFP4_ERR_INVALID_ARG, NVFP4_ERR_UNSUPPORTED_SHAPE, NVFP4_ERR_MISALIGNED, NVFP4_ERR_CUDA, NVFP4_ERR_TIMEOUT,
 NVFP4_ERR_WORKSPACE) = 1, 2, 3, 4, 5, 6
NVFP4_RNE, NVFP4_SR = 0, 1
NVFP4_SCALE_1D, NVFP4_SCALE_2D = 0, 1
NVFP4_OUT_F32, NVFP4_OUT_BF16 = 0, 1

EXPORTS = (
    "nvfp4_version", "nvfp4_status_string", "nvfp4_workspace_size", "nvfp4_mma_scale_bytes",
    "nvfp4_quantize_1d", "nvfp4_rht_quantize_sr", "nvfp4_quantize_2d", "nvfp4_dequantize", "nvfp4_gemm",
    "nvfp4_scales_to_mma", "nvfp4_kernel_launches", "nvfp4_get_error", "nvfp4_quantize_1d_noalloc",
    "nvfp4_selftest_wait_timeout", "nvfp4_quantize_1d_from_amax", "nvfp4_quantize_2d_from_amax",
    "nvfp4_gemm_amax", "nvfp4_mxfp4_quantize", "nvfp4_mxfp4_dequantize", "nvfp4_mxfp4_gemm",
    "nvfp4_quantize_dual", "nvfp4_rht_quantize_n",
)

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {lib().nvfp4_status_string(status).decode()} (status {status})")


def lib():
    """Load libnvfp4.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libnvfp4.so not built (expected at {LIB_PATH}); run "
                          "`python -m nvfp4_bit_block_amax_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, u64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_size_t
        L.nvfp4_version.restype = ci
        L.nvfp4_version.argtypes = []
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_status_string.argtypes = [ci]
        L.nvfp4_workspace_size.restype = sz
        L.nvfp4_workspace_size.argtypes = [i64, i64]
        L.nvfp4_mma_scale_bytes.restype = sz
        L.nvfp4_mma_scale_bytes.argtypes = [i64, i64]
        L.nvfp4_quantize_1d.restype = ci
        L.nvfp4_quantize_1d.argtypes = [vp, i64, i64, i64, ci, ci, u64, vp, vp, vp, vp, vp, sz, vp]
        L.nvfp4_quantize_1d_noalloc.restype = ci
        L.nvfp4_quantize_1d_noalloc.argtypes = [vp, i64, i64, i64, ci, ci, u64, vp, vp, vp, vp, vp]
        L.nvfp4_rht_quantize_sr.restype = ci
        L.nvfp4_rht_quantize_sr.argtypes = [vp, i64, i64, i64, ci, u64, ci, u64, vp, vp, vp, vp, vp, sz, vp]
        L.nvfp4_rht_quantize_n.restype = ci
        L.nvfp4_rht_quantize_n.argtypes = [vp, i64, i64, i64, ci, ci, u64, ci, u64, vp, vp, vp, vp, vp, sz, vp]
        L.nvfp4_quantize_2d.restype = ci
        L.nvfp4_quantize_2d.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.nvfp4_dequantize.restype = ci
        L.nvfp4_dequantize.argtypes = [vp, vp, ci, vp, i64, i64, ci, vp, vp]
        L.nvfp4_gemm.restype = ci
        L.nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, ci, vp, i64, vp]
        L.nvfp4_scales_to_mma.restype = ci
        L.nvfp4_scales_to_mma.argtypes = [vp, ci, i64, i64, vp, vp]
        L.nvfp4_kernel_launches.restype = ctypes.c_longlong
        L.nvfp4_kernel_launches.argtypes = []
        L.nvfp4_get_error.restype = ci
        L.nvfp4_get_error.argtypes = [vp]
        L.nvfp4_selftest_wait_timeout.restype = ci
        L.nvfp4_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        L.nvfp4_quantize_1d_from_amax.restype = ci
        L.nvfp4_quantize_1d_from_amax.argtypes = [vp, i64, i64, i64, ci, ci, u64, vp, vp, vp, vp, vp, vp]
        L.nvfp4_quantize_2d_from_amax.restype = ci
        L.nvfp4_quantize_2d_from_amax.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp]
        L.nvfp4_gemm_amax.restype = ci
        L.nvfp4_gemm_amax.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, ci, vp, i64, vp, vp]
        L.nvfp4_mxfp4_quantize.restype = ci
        L.nvfp4_mxfp4_quantize.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
        L.nvfp4_mxfp4_dequantize.restype = ci
        L.nvfp4_mxfp4_dequantize.argtypes = [vp, vp, i64, i64, ci, vp, vp]
        L.nvfp4_quantize_dual.restype = ci
        L.nvfp4_quantize_dual.argtypes = [vp, i64, i64, i64, ci, u64, vp, vp, vp, vp, u64, u64, vp, vp, vp, vp, vp,
                                          sz, vp]
        L.nvfp4_mxfp4_gemm.restype = ci
        L.nvfp4_mxfp4_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, vp, i64, vp]
        _lib = L
    return _lib


def _p(t) -> Optional[int]:
    """Device pointer of a tensor (None / int pass through)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != NVFP4_OK:
        raise Nvfp4Error(fn, status)


# ------------------------------------------------------------- C ABI mirror --
def nvfp4_version() -> int:
    return lib().nvfp4_version()


def nvfp4_status_string(status: int) -> str:
    return lib().nvfp4_status_string(status).decode()


def nvfp4_workspace_size(rows: int, cols: int) -> int:
    return lib().nvfp4_workspace_size(rows, cols)


def nvfp4_mma_scale_bytes(rows: int, k: int) -> int:
    return lib().nvfp4_mma_scale_bytes(rows, k)


def nvfp4_kernel_launches() -> int:
    return lib().nvfp4_kernel_launches()


def nvfp4_quantize_1d(x, rows, cols, ld, transpose, rounding, sr_seed, codes, scales, scales_mma,
                      global_scale, workspace, ws_bytes, stream=None):
    _check("nvfp4_quantize_1d", lib().nvfp4_quantize_1d(
        _p(x), rows, cols, ld, transpose, rounding, sr_seed, _p(codes), _p(scales), _p(scales_mma),
        _p(global_scale), _p(workspace), ws_bytes, _stream(stream)))


def nvfp4_quantize_1d_noalloc(x, rows, cols, ld, transpose, rounding, sr_seed, codes, scales, scales_mma,
                              global_scale, stream=None):
    """nvfp4_quantize_1d without a workspace argument: for callers that cannot
    allocate device memory, the library uses its own static scratch."""
    _check("nvfp4_quantize_1d_noalloc", lib().nvfp4_quantize_1d_noalloc(
        _p(x), rows, cols, ld, transpose, rounding, sr_seed, _p(codes), _p(scales), _p(scales_mma),
        _p(global_scale), _stream(stream)))


def nvfp4_rht_quantize_sr(x, rows, cols, ld, transpose, rht_seed, rounding, sr_seed, codes, scales, scales_mma,
                          global_scale, workspace, ws_bytes, stream=None):
    _check("nvfp4_rht_quantize_sr", lib().nvfp4_rht_quantize_sr(
        _p(x), rows, cols, ld, transpose, rht_seed, rounding, sr_seed, _p(codes), _p(scales), _p(scales_mma),
        _p(global_scale), _p(workspace), ws_bytes, _stream(stream)))


def nvfp4_rht_quantize_n(x, rows, cols, ld, transpose, rht_order, rht_seed, rounding, sr_seed, codes, scales,
                         scales_mma, global_scale, workspace, ws_bytes, stream=None):
    _check("nvfp4_rht_quantize_n", lib().nvfp4_rht_quantize_n(
        _p(x), rows, cols, ld, transpose, rht_order, rht_seed, rounding, sr_seed, _p(codes), _p(scales),
        _p(scales_mma), _p(global_scale), _p(workspace), ws_bytes, _stream(stream)))


def nvfp4_quantize_dual(x, rows, cols, ld, rounding, sr_seed, codes, scales, scales_mma, global_scale, rht_seed,
                        sr_seed_t, codes_t, scales_t, scales_mma_t, global_scale_t, workspace, ws_bytes, stream=None):
    _check("nvfp4_quantize_dual", lib().nvfp4_quantize_dual(
        _p(x), rows, cols, ld, rounding, sr_seed, _p(codes), _p(scales), _p(scales_mma), _p(global_scale), rht_seed,
        sr_seed_t, _p(codes_t), _p(scales_t), _p(scales_mma_t), _p(global_scale_t), _p(workspace), ws_bytes,
        _stream(stream)))


def nvfp4_quantize_2d(w, rows, cols, ld, codes_row, codes_col, scales, scales_mma_row, scales_mma_col,
                      global_scale, workspace, ws_bytes, stream=None):
    _check("nvfp4_quantize_2d", lib().nvfp4_quantize_2d(
        _p(w), rows, cols, ld, _p(codes_row), _p(codes_col), _p(scales), _p(scales_mma_row), _p(scales_mma_col),
        _p(global_scale), _p(workspace), ws_bytes, _stream(stream)))


def nvfp4_dequantize(codes, scales, scale_mode, global_scale, rows, cols, out_dtype, out, stream=None):
    _check("nvfp4_dequantize", lib().nvfp4_dequantize(
        _p(codes), _p(scales), scale_mode, _p(global_scale), rows, cols, out_dtype, _p(out), _stream(stream)))


def nvfp4_gemm(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M, N, K, out_dtype, c, ldc,
               stream=None):
    _check("nvfp4_gemm", lib().nvfp4_gemm(
        _p(a_codes), _p(a_scales_mma), _p(a_gs), _p(b_codes), _p(b_scales_mma), _p(b_gs), M, N, K, out_dtype,
        _p(c), ldc, _stream(stream)))


def nvfp4_gemm_amax(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M, N, K, out_dtype, c, ldc, c_amax,
                    stream=None):
    _check("nvfp4_gemm_amax", lib().nvfp4_gemm_amax(
        _p(a_codes), _p(a_scales_mma), _p(a_gs), _p(b_codes), _p(b_scales_mma), _p(b_gs), M, N, K, out_dtype,
        _p(c), ldc, _p(c_amax), _stream(stream)))


def nvfp4_quantize_1d_from_amax(x, rows, cols, ld, transpose, rounding, sr_seed, amax, codes, scales, scales_mma,
                                global_scale, stream=None):
    _check("nvfp4_quantize_1d_from_amax", lib().nvfp4_quantize_1d_from_amax(
        _p(x), rows, cols, ld, transpose, rounding, sr_seed, _p(amax), _p(codes), _p(scales), _p(scales_mma),
        _p(global_scale), _stream(stream)))


def nvfp4_quantize_2d_from_amax(w, rows, cols, ld, amax, codes_row, codes_col, scales, scales_mma_row,
                                scales_mma_col, global_scale, stream=None):
    _check("nvfp4_quantize_2d_from_amax", lib().nvfp4_quantize_2d_from_amax(
        _p(w), rows, cols, ld, _p(amax), _p(codes_row), _p(codes_col), _p(scales), _p(scales_mma_row),
        _p(scales_mma_col), _p(global_scale), _stream(stream)))


def nvfp4_mxfp4_quantize(x, rows, cols, ld, codes, scales, scales_mma, stream=None):
    _check("nvfp4_mxfp4_quantize", lib().nvfp4_mxfp4_quantize(
        _p(x), rows, cols, ld, _p(codes), _p(scales), _p(scales_mma), _stream(stream)))


def nvfp4_mxfp4_dequantize(codes, scales, rows, cols, out_dtype, out, stream=None):
    _check("nvfp4_mxfp4_dequantize", lib().nvfp4_mxfp4_dequantize(
        _p(codes), _p(scales), rows, cols, out_dtype, _p(out), _stream(stream)))


def nvfp4_mxfp4_gemm(a_codes, a_scales_mma, b_codes, b_scales_mma, M, N, K, out_dtype, c, ldc, stream=None):
    _check("nvfp4_mxfp4_gemm", lib().nvfp4_mxfp4_gemm(
        _p(a_codes), _p(a_scales_mma), _p(b_codes), _p(b_scales_mma), M, N, K, out_dtype, _p(c), ldc,
        _stream(stream)))


def nvfp4_scales_to_mma(scales, scale_mode, rows, k, scales_mma, stream=None):
    _check("nvfp4_scales_to_mma", lib().nvfp4_scales_to_mma(
        _p(scales), scale_mode, rows, k, _p(scales_mma), _stream(stream)))


def nvfp4_get_error(stream=None) -> int:
    return lib().nvfp4_get_error(_stream(stream))


def nvfp4_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    return lib().nvfp4_selftest_wait_timeout(int(limit_ns), _stream(stream))


# --------------------------------------------------------- torch helpers ----
@dataclass
class Quantized:
    """One NVFP4 tensor Q [rows x cols] on the device."""
    codes: torch.Tensor                      # uint8 [rows, cols/2]
    scales: Optional[torch.Tensor]           # uint8 plain layout
    scales_mma: Optional[torch.Tensor]       # uint8 MMA layout
    global_scale: torch.Tensor               # float32 [1]
    rows: int
    cols: int
    codes_col: Optional[torch.Tensor] = None         # 2D only: codes of Q^T
    scales_mma_col: Optional[torch.Tensor] = None    # 2D only: MMA scales of Q^T


_ws_cache = {}


def workspace(device=None) -> torch.Tensor:
    """A per-device scratch buffer for the amax partials (allocated by torch)."""
    dev = torch.device(device if device is not None else "cuda")
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    ws = _ws_cache.get(key)
    n = nvfp4_workspace_size(0, 0)
    if ws is None or ws.numel() < n:
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def _empty_u8(n, device):
    return torch.empty(n, dtype=torch.uint8, device=device)


def quantize_1d(x: torch.Tensor, transpose: bool = False, rounding: int = NVFP4_RNE, sr_seed: int = 0,
                rht: bool = False, rht_seed: int = 0, plain_scales: bool = True, mma_scales: bool = True,
                stream=None, amax: Optional[torch.Tensor] = None, rht_order: int = 16) -> Quantized:
    """Quantize a bf16 [rows x cols] tensor (or its transpose) with 16-element blocks.
    With `amax` (a device float holding max |x|) the amax pass is skipped;
    with `rht` the Q rows are rotated in chunks of `rht_order` points."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    qr, qc = (cols, rows) if transpose else (rows, cols)
    dev = x.device
    codes = torch.empty(qr, qc // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(qr, qc // 16, dtype=torch.uint8, device=dev) if plain_scales else None
    smma = _empty_u8(nvfp4_mma_scale_bytes(qr, qc), dev) if mma_scales else None
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    ws = workspace(dev)
    if amax is not None:
        assert not rht, "the amax of the rotated tensor is not known to a producer"
        nvfp4_quantize_1d_from_amax(x, rows, cols, x.stride(0), int(transpose), rounding, sr_seed, amax, codes,
                                    scales, smma, gs, stream)
    elif rht and rht_order != 16:
        nvfp4_rht_quantize_n(x, rows, cols, x.stride(0), int(transpose), rht_order, rht_seed, rounding, sr_seed,
                             codes, scales, smma, gs, ws, ws.numel(), stream)
    elif rht:
        nvfp4_rht_quantize_sr(x, rows, cols, x.stride(0), int(transpose), rht_seed, rounding, sr_seed, codes,
                              scales, smma, gs, ws, ws.numel(), stream)
    else:
        nvfp4_quantize_1d(x, rows, cols, x.stride(0), int(transpose), rounding, sr_seed, codes, scales, smma,
                          gs, ws, ws.numel(), stream)
    return Quantized(codes, scales, smma, gs, qr, qc)


def quantize_2d(w: torch.Tensor, columnwise: bool = True, plain_scales: bool = True, mma_scales: bool = True,
                stream=None, amax: Optional[torch.Tensor] = None) -> Quantized:
    """Quantize a bf16 weight with 16x16 tiles (rowwise codes, optional columnwise copy)."""
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.stride(1) == 1
    rows, cols = w.shape
    dev = w.device
    cr = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    cc = torch.empty(cols, rows // 2, dtype=torch.uint8, device=dev) if columnwise else None
    sc = torch.empty(rows // 16, cols // 16, dtype=torch.uint8, device=dev) if plain_scales else None
    mr = _empty_u8(nvfp4_mma_scale_bytes(rows, cols), dev) if mma_scales else None
    mc = _empty_u8(nvfp4_mma_scale_bytes(cols, rows), dev) if (mma_scales and columnwise) else None
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    ws = workspace(dev)
    if amax is not None:
        nvfp4_quantize_2d_from_amax(w, rows, cols, w.stride(0), amax, cr, cc, sc, mr, mc, gs, stream)
    else:
        nvfp4_quantize_2d(w, rows, cols, w.stride(0), cr, cc, sc, mr, mc, gs, ws, ws.numel(), stream)
    return Quantized(cr, sc, mr, gs, rows, cols, codes_col=cc, scales_mma_col=mc)


def dequantize(q: Quantized, scale_mode: int = NVFP4_SCALE_1D, out_dtype: int = NVFP4_OUT_F32,
               stream=None) -> torch.Tensor:
    dt = torch.float32 if out_dtype == NVFP4_OUT_F32 else torch.bfloat16
    out = torch.empty(q.rows, q.cols, dtype=dt, device=q.codes.device)
    nvfp4_dequantize(q.codes, q.scales, scale_mode, q.global_scale, q.rows, q.cols, out_dtype, out, stream)
    return out


def gemm(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M: int, N: int, K: int,
         out_dtype: int = NVFP4_OUT_BF16, out: Optional[torch.Tensor] = None, stream=None,
         amax_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """C = alpha * A . B^T with NVFP4 operands (MMA-layout scales).  With
    `amax_out` (a device float) the epilogue also writes max |C| there."""
    if out is None:
        dt = torch.float32 if out_dtype == NVFP4_OUT_F32 else torch.bfloat16
        ldc = (N + 7) // 8 * 8
        out = torch.empty(M, ldc, dtype=dt, device=a_codes.device)[:, :N]
    if amax_out is not None:
        nvfp4_gemm_amax(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M, N, K, out_dtype, out,
                        out.stride(0), amax_out, stream)
    else:
        nvfp4_gemm(a_codes, a_scales_mma, a_gs, b_codes, b_scales_mma, b_gs, M, N, K, out_dtype, out,
                   out.stride(0), stream)
    return out


def mxfp4_quantize(x: torch.Tensor, plain_scales: bool = True, mma_scales: bool = True, stream=None) -> Quantized:
    """MXFP4 quantization of a bf16 [rows x cols] tensor (32-element blocks, E8M0 scales)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    dev = x.device
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device=dev) if plain_scales else None
    smma = _empty_u8(nvfp4_mma_scale_bytes(rows, cols), dev) if mma_scales else None
    nvfp4_mxfp4_quantize(x, rows, cols, x.stride(0), codes, scales, smma, stream)
    return Quantized(codes, scales, smma, torch.ones(1, dtype=torch.float32, device=dev), rows, cols)


def mxfp4_gemm(a: Quantized, b: Quantized, out_dtype: int = NVFP4_OUT_BF16, stream=None) -> torch.Tensor:
    """C = A . B^T of two MXFP4 operands (K-major)."""
    M, K, N = a.rows, a.cols, b.rows
    dt = torch.float32 if out_dtype == NVFP4_OUT_F32 else torch.bfloat16
    ldc = (N + 7) // 8 * 8
    out = torch.empty(M, ldc, dtype=dt, device=a.codes.device)[:, :N]
    nvfp4_mxfp4_gemm(a.codes, a.scales_mma, b.codes, b.scales_mma, M, N, K, out_dtype, out, out.stride(0), stream)
    return out


def quantize_dual(x: torch.Tensor, rounding: int = NVFP4_RNE, sr_seed: int = 0, rht_seed: int = 0,
                  sr_seed_t: int = 0, stream=None):
    """(Q1, Q2): x row-wise and RHT(x^T), from one shared amax read."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    dev = x.device
    q1 = Quantized(torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
                   torch.empty(rows, cols // 16, dtype=torch.uint8, device=dev),
                   _empty_u8(nvfp4_mma_scale_bytes(rows, cols), dev), torch.empty(1, dtype=torch.float32, device=dev),
                   rows, cols)
    q2 = Quantized(torch.empty(cols, rows // 2, dtype=torch.uint8, device=dev),
                   torch.empty(cols, rows // 16, dtype=torch.uint8, device=dev),
                   _empty_u8(nvfp4_mma_scale_bytes(cols, rows), dev), torch.empty(1, dtype=torch.float32, device=dev),
                   cols, rows)
    ws = torch.empty(2 * nvfp4_workspace_size(rows, cols), dtype=torch.uint8, device=dev)
    nvfp4_quantize_dual(x, rows, cols, x.stride(0), rounding, sr_seed, q1.codes, q1.scales, q1.scales_mma,
                        q1.global_scale, rht_seed, sr_seed_t, q2.codes, q2.scales, q2.scales_mma, q2.global_scale,
                        ws, ws.numel(), stream)
    return q1, q2
