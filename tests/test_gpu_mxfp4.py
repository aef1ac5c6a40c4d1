"""MXFP4 variant on the GPU against the oracle: quantized codes and E8M0
scales bit-exact, the GEMM scale layout as its formula states, dequantize
bit-exact, and the GEMM within 2e-3 * sum|a*b| of the float64 product of
the dequantized operands, on both GEMM kernels."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import to_device_bf16

pytestmark = pytest.mark.gpu

TOL = 2e-3


def mx_mma_layout(plain: np.ndarray, rows: int, kb32: int) -> np.ndarray:
    """Plain E8M0 codes [rows x kb32] -> the 4-byte-per-(row, 64-wide K step)
    layout: block b at byte b % 2 of step b // 2, bytes 2 and 3 zero."""
    chunks = (kb32 + 1) // 2
    out = np.zeros(((rows + 127) // 128) * chunks * 512, dtype=np.uint8)
    r = np.arange(rows)[:, None]
    b = np.arange(kb32)[None, :]
    off = ((r // 128) * chunks + b // 2) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 2)
    out[off.ravel()] = plain.reshape(rows, kb32).ravel()
    return out


def _tensor(rows, cols, seed, dist):
    if dist == "outliers":
        return G.make_tensor(rows, cols, seed, outlier_frac=0.001, outlier_mode="set", outlier_value=1e4)
    if dist == "lognormal":
        return G.make_tensor(rows, cols, seed, dist="lognormal_signed", scale=2.0)
    if dist == "zeros":
        x = G.make_tensor(rows, cols, seed)
        x[:, :64] = 0
        x[::3, 64:96] = 0x0001          # subnormal-only blocks
        return x
    return G.make_tensor(rows, cols, seed)


@pytest.mark.parametrize("shape", [(64, 1024), (37, 96), (130, 4096)])
@pytest.mark.parametrize("dist", ["normal", "lognormal", "outliers", "zeros"])
def test_mx_quantize_matches_oracle(shape, dist):
    rows, cols = shape
    x_bits = _tensor(rows, cols, 401, dist)
    q = N.mxfp4_quantize(to_device_bf16(x_bits))
    torch.cuda.synchronize()
    codes, scales = O.mx_quantize(x_bits)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.scales.cpu().numpy(), scales)
    assert np.array_equal(q.scales_mma.cpu().numpy(), mx_mma_layout(scales, rows, cols // 32))
    assert N.nvfp4_get_error() == 0


@pytest.mark.parametrize("out_dtype", [N.NVFP4_OUT_F32, N.NVFP4_OUT_BF16])
def test_mx_dequantize_matches_oracle(out_dtype):
    rows, cols = 96, 512
    x_bits = _tensor(rows, cols, 402, "lognormal")
    codes, scales = O.mx_quantize(x_bits)
    ref = O.mx_dequantize(codes, scales, rows, cols)
    dt = torch.float32 if out_dtype == N.NVFP4_OUT_F32 else torch.bfloat16
    out = torch.empty(rows, cols, dtype=dt, device="cuda")
    N.nvfp4_mxfp4_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), rows, cols,
                             out_dtype, out)
    torch.cuda.synchronize()
    if out_dtype == N.NVFP4_OUT_F32:
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    else:
        want = torch.from_numpy(ref).to(torch.bfloat16)
        assert torch.equal(out.cpu().view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("kernel", ["1", "0"])
@pytest.mark.parametrize("mnk,out_dtype", [((256, 256, 256), N.NVFP4_OUT_F32), ((384, 512, 1024), N.NVFP4_OUT_BF16),
                                           ((200, 300, 320), N.NVFP4_OUT_F32)])
def test_mx_gemm_within_tolerance(monkeypatch, kernel, mnk, out_dtype):
    monkeypatch.setenv("NVFP4_GEMM_PAIR", kernel)
    M, Nn, K = mnk
    a_bits = G.activation(M, K, seed=403)
    b_bits = G.weight(Nn, K, seed=404)
    a = N.mxfp4_quantize(to_device_bf16(a_bits))
    b = N.mxfp4_quantize(to_device_bf16(b_bits))
    c = N.mxfp4_gemm(a, b, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ca, sa = O.mx_quantize(a_bits)
    cb, sb = O.mx_quantize(b_bits)
    assert np.array_equal(a.codes.cpu().numpy(), ca) and np.array_equal(b.codes.cpu().numpy(), cb)
    ref, s = O.mx_gemm_reference(ca, sa, cb, sb, M, Nn, K)
    got = c.float().cpu().numpy().astype(np.float64)
    bound = TOL * s
    if out_dtype == N.NVFP4_OUT_BF16:
        e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126)))
        bound = bound + 2.0 ** (e - 8)
    assert (np.abs(got - ref) <= bound).all(), float(np.max(np.abs(got - ref) / np.maximum(s, 1e-30)))
    assert N.nvfp4_get_error() == 0
