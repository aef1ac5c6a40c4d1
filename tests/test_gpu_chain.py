"""Two chained layers with the amax handed over by its producer, at the
bench's sizes (X [16384 x 8192], W1 [28672 x 8192], W2 [8192 x 28672]):
Y = X . W1^T from nvfp4_gemm_amax, Yq = nvfp4_quantize_1d_from_amax(Y) in one
read, Z = Yq . W2^T.  The checks: Y on sampled rows against the float64
product of the oracle's dequantized X and W1 (the GEMM tolerance); the handed
amax is max |Y| exactly; Yq is bit-identical to the two-pass quantizer on Y
(the quantizer whose parity with the oracle the other tests establish on
generator inputs -- Y itself comes from the GPU, so the oracle does not
consume it); Z on sampled rows against the float64 product of Yq as the GPU
dequantizes it and the oracle's dequantized W2."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import to_device_bf16
from tests.test_gpu_fullsize import check_quantized_rows, gemm_rows_check, sample_rows

pytestmark = pytest.mark.gpu


def test_chain_amax_from_producer_full_size():
    t, h, f = G.MLP_STEP["tokens"], G.MLP_STEP["hidden"], G.MLP_STEP["ffn"]
    seed = G.seeds("mlp_step")[0]
    x = G.activation(t, h, seed)
    w1 = G.weight(f, h, seed + 1)
    w2 = G.weight(h, f, seed + 3)
    qx = N.quantize_1d(to_device_bf16(x), plain_scales=False)
    qw1 = N.quantize_2d(to_device_bf16(w1), columnwise=False)
    qw2 = N.quantize_2d(to_device_bf16(w2), columnwise=False)
    amax = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    y = N.gemm(qx.codes, qx.scales_mma, qx.global_scale, qw1.codes, qw1.scales_mma, qw1.global_scale, t, f, h,
               amax_out=amax)
    yq = N.quantize_1d(y, amax=amax)
    yq2 = N.quantize_1d(y)
    z = N.gemm(yq.codes, yq.scales_mma, yq.global_scale, qw2.codes, qw2.scales_mma, qw2.global_scale, t, h, f)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    assert amax.item() == y.float().abs().max().item()
    for a, b in ((yq.codes, yq2.codes), (yq.scales, yq2.scales), (yq.scales_mma, yq2.scales_mma),
                 (yq.global_scale, yq2.global_scale)):
        assert torch.equal(a, b)
    rows = sample_rows(t, 4, seed=21)
    sgx = check_quantized_rows(qx, x, rows)
    cw1, _, sw1, gw1 = O.quantize_2d(w1, columnwise=False)
    assert np.float32(qw1.global_scale.item()) == gw1 and np.array_equal(qw1.codes.cpu().numpy(), cw1)
    gx = O.quantize_1d_rows(x, sgx, rows)
    xh = np.concatenate([O.dequantize_f64(gx[r][0][None], gx[r][1][None], 0, sgx, 1, h) for r in rows])
    gemm_rows_check(y[rows].float().cpu().numpy(), xh, O.dequantize_f64(cw1, sw1, 1, gw1, f, h))
    del cw1, sw1
    cw2, _, sw2, gw2 = O.quantize_2d(w2, columnwise=False)
    assert np.float32(qw2.global_scale.item()) == gw2 and np.array_equal(qw2.codes.cpu().numpy(), cw2)
    yh = N.dequantize(yq, N.NVFP4_SCALE_1D, N.NVFP4_OUT_F32)[rows].cpu().numpy().astype(np.float64)
    gemm_rows_check(z[rows].float().cpu().numpy(), yh, O.dequantize_f64(cw2, sw2, 1, gw2, h, f))
