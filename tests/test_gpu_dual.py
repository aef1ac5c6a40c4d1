"""The dual quantizer (x row-wise and RHT(x^T) from one shared amax read):
bit-identical to the two separate calls and to the oracle, RNE and SR,
including shapes that are not multiples of the kernels' tiles."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(256, 512), (272, 400), (1024, 2048)])
@pytest.mark.parametrize("rounding", [N.NVFP4_RNE, N.NVFP4_SR])
def test_dual_matches_separate_calls_and_oracle(shape, rounding):
    rows, cols = shape
    x_bits = G.gradient(rows, cols, seed=501) if rounding == N.NVFP4_SR else G.activation(rows, cols, seed=502)
    x = to_device_bf16(x_bits)
    q1, q2 = N.quantize_dual(x, rounding=rounding, sr_seed=11, rht_seed=12, sr_seed_t=13)
    s1 = N.quantize_1d(x, rounding=rounding, sr_seed=11)
    s2 = N.quantize_1d(x, transpose=True, rounding=rounding, sr_seed=13, rht=True, rht_seed=12)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    for a, b in ((q1.codes, s1.codes), (q1.scales, s1.scales), (q1.scales_mma, s1.scales_mma),
                 (q1.global_scale, s1.global_scale), (q2.codes, s2.codes), (q2.scales, s2.scales),
                 (q2.scales_mma, s2.scales_mma), (q2.global_scale, s2.global_scale)):
        assert torch.equal(a, b)
    c1, sc1, g1 = O.quantize_1d(x_bits, rounding=rounding, sr_seed=11)
    c2, sc2, g2 = O.quantize_1d(x_bits, transpose=True, rht=True, rht_seed=12, rounding=rounding, sr_seed=13)
    assert np.array_equal(q1.codes.cpu().numpy(), c1) and np.array_equal(q1.scales.cpu().numpy(), sc1)
    assert np.array_equal(q2.codes.cpu().numpy(), c2) and np.array_equal(q2.scales.cpu().numpy(), sc2)
    assert np.float32(q1.global_scale.item()) == np.float32(g1) and np.float32(q2.global_scale.item()) == np.float32(g2)


def test_dual_rejects_small_workspace():
    x = to_device_bf16(G.activation(64, 64, seed=503))
    q1, q2 = N.quantize_dual(x)
    ws = torch.empty(N.nvfp4_workspace_size(64, 64), dtype=torch.uint8, device="cuda")    # one set only
    with pytest.raises(N.Nvfp4Error) as e:
        N.nvfp4_quantize_dual(x, 64, 64, 64, N.NVFP4_RNE, 0, q1.codes, q1.scales, q1.scales_mma, q1.global_scale,
                              0, 0, q2.codes, q2.scales, q2.scales_mma, q2.global_scale, ws, ws.numel())
    assert e.value.status == N.NVFP4_ERR_WORKSPACE
