"""The allocation-free quantize entry point (nvfp4_quantize_1d_noalloc).

Callers whose device memory belongs to another allocator, or that may not
allocate at all, cannot pass a workspace; this entry point uses a static
scratch array inside the library instead.  Its outputs must equal those of
nvfp4_quantize_1d (bit for bit, the quantizers' tolerance), on consecutive
calls that share the static scratch.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from tests.helpers import to_device_bf16

pytestmark = pytest.mark.gpu


def outputs(x, transpose, rounding, sr_seed, noalloc):
    rows, cols = x.shape
    qr, qc = (cols, rows) if transpose else (rows, cols)
    dev = x.device
    codes = torch.full((qr, qc // 2), 0xAB, dtype=torch.uint8, device=dev)
    scales = torch.full((qr, qc // 16), 0xCD, dtype=torch.uint8, device=dev)
    smma = torch.full((N.nvfp4_mma_scale_bytes(qr, qc),), 0xEF, dtype=torch.uint8, device=dev)
    gs = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    if noalloc:
        N.nvfp4_quantize_1d_noalloc(x, rows, cols, x.stride(0), int(transpose), rounding, sr_seed, codes, scales,
                                    smma, gs)
    else:
        ws = torch.empty(N.nvfp4_workspace_size(rows, cols), dtype=torch.uint8, device=dev)
        N.nvfp4_quantize_1d(x, rows, cols, x.stride(0), int(transpose), rounding, sr_seed, codes, scales, smma, gs,
                            ws, ws.numel())
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    return codes.cpu().numpy(), scales.cpu().numpy(), smma.cpu().numpy(), gs.cpu().numpy()


def same(a, b):
    return all(np.array_equal(u, v) for u, v in zip(a, b))


@pytest.mark.parametrize("transpose", [False, True])
def test_noalloc_matches_workspace_path_on_two_calls(transpose):
    big = to_device_bf16(G.activation(1024, 4096, seed=71))               # large amax
    small = to_device_bf16(G.gradient(512, 1536, seed=72) )              # tiny values: a stale amax would show
    for x, rounding in ((big, N.NVFP4_RNE), (small, N.NVFP4_SR)):
        ref = outputs(x, transpose, rounding, 9, noalloc=False)
        got = outputs(x, transpose, rounding, 9, noalloc=True)
        assert same(got, ref)
    # two calls in a row on the same input give the reference result both times
    ref = outputs(small, transpose, N.NVFP4_RNE, 0, noalloc=False)
    first = outputs(small, transpose, N.NVFP4_RNE, 0, noalloc=True)
    second = outputs(small, transpose, N.NVFP4_RNE, 0, noalloc=True)
    assert same(first, ref) and same(second, ref)


def test_noalloc_validates_like_the_workspace_path():
    x = to_device_bf16(G.activation(32, 40, seed=73))
    with pytest.raises(N.Nvfp4Error):
        outputs(x, False, N.NVFP4_RNE, 0, noalloc=True)          # 40 columns: not whole 16-blocks
