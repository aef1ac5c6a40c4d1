"""Fused amax (the producer of a tensor supplies its amax): nvfp4_gemm_amax
writes max |C| exactly, and quantizing with a given amax skips the amax pass
yet stays bit-identical to the oracle and to the two-pass quantizers."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import to_device_bf16

pytestmark = pytest.mark.gpu


def _dev_amax(x: torch.Tensor) -> torch.Tensor:
    return x.float().abs().max().reshape(1).contiguous()


@pytest.mark.parametrize("kernel", ["1", "0"])
@pytest.mark.parametrize("mnk,out_dtype", [((512, 768, 1024), N.NVFP4_OUT_BF16), ((300, 200, 256), N.NVFP4_OUT_BF16),
                                           ((256, 520, 512), N.NVFP4_OUT_F32)])
def test_gemm_amax_is_max_abs_of_output(monkeypatch, kernel, mnk, out_dtype):
    monkeypatch.setenv("NVFP4_GEMM_PAIR", kernel)
    M, Nn, K = mnk
    a = N.quantize_1d(to_device_bf16(G.activation(M, K, seed=301)))
    b = N.quantize_1d(to_device_bf16(G.weight(Nn, K, seed=302)))
    amax = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")     # overwritten, not accumulated
    c = N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, M, Nn, K,
               out_dtype=out_dtype, amax_out=amax)
    c_plain = N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, M, Nn, K,
                     out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(c, c_plain)
    assert amax.item() == c.float().abs().max().item()
    assert N.nvfp4_get_error() == 0


@pytest.mark.parametrize("transpose,rounding", [(0, N.NVFP4_RNE), (1, N.NVFP4_RNE), (0, N.NVFP4_SR), (1, N.NVFP4_SR)])
def test_quantize_1d_from_amax_matches_oracle(transpose, rounding):
    x_bits = G.activation(384, 512, seed=303)
    x = to_device_bf16(x_bits)
    q = N.quantize_1d(x, transpose=bool(transpose), rounding=rounding, sr_seed=77, amax=_dev_amax(x))
    q2 = N.quantize_1d(x, transpose=bool(transpose), rounding=rounding, sr_seed=77)
    torch.cuda.synchronize()
    codes, scales, gs = O.quantize_1d(x_bits, transpose=bool(transpose), rounding=rounding, sr_seed=77)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.scales.cpu().numpy(), scales)
    assert q.global_scale.item() == np.float32(gs)
    assert torch.equal(q.scales_mma, q2.scales_mma) and torch.equal(q.codes, q2.codes)


def test_quantize_2d_from_amax_matches_two_pass():
    w_bits = G.weight(512, 256, seed=304)
    w = to_device_bf16(w_bits)
    q = N.quantize_2d(w, amax=_dev_amax(w))
    q2 = N.quantize_2d(w)
    torch.cuda.synchronize()
    for a, b in ((q.codes, q2.codes), (q.codes_col, q2.codes_col), (q.scales, q2.scales),
                 (q.scales_mma, q2.scales_mma), (q.scales_mma_col, q2.scales_mma_col),
                 (q.global_scale, q2.global_scale)):
        assert torch.equal(a, b)
    cr, cc, sc, gs = O.quantize_2d(w_bits, columnwise=True)
    assert np.array_equal(q.codes.cpu().numpy(), cr) and np.array_equal(q.codes_col.cpu().numpy(), cc)


def test_gemm_output_quantized_in_one_read():
    """Y = X W^T with the amax from the epilogue, then Y quantized from it:
    identical to quantizing Y with its own amax pass."""
    M, Nn, K = 512, 1024, 512
    a = N.quantize_1d(to_device_bf16(G.activation(M, K, seed=305)))
    b = N.quantize_2d(to_device_bf16(G.weight(Nn, K, seed=306)), columnwise=False)
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    y = N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, M, Nn, K,
               amax_out=amax).contiguous()
    qy = N.quantize_1d(y, amax=amax)
    qy2 = N.quantize_1d(y)
    torch.cuda.synchronize()
    assert torch.equal(qy.codes, qy2.codes) and torch.equal(qy.scales, qy2.scales)
    assert torch.equal(qy.global_scale, qy2.global_scale)
