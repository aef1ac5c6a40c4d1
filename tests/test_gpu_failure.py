"""Failure detection without a GPU fault: a bounded device-side wait that runs
out raises the library's error word, nvfp4_get_error reports
NVFP4_ERR_TIMEOUT once and clears it, and the context keeps working."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import to_device_bf16

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert N.nvfp4_get_error() == N.NVFP4_OK
    assert N.nvfp4_selftest_wait_timeout(20_000_000) == N.NVFP4_OK       # 20 ms, nothing arrives
    assert N.nvfp4_get_error() == N.NVFP4_ERR_TIMEOUT
    assert N.nvfp4_get_error() == N.NVFP4_OK                               # read clears it
    # the same context still quantizes bit-exactly
    x = G.activation(128, 256, seed=91)
    q = N.quantize_1d(to_device_bf16(x))
    torch.cuda.synchronize()
    codes, scales, gs = O.quantize_1d(x)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert N.nvfp4_get_error() == N.NVFP4_OK


def test_selftest_rejects_bad_limits():
    assert N.nvfp4_selftest_wait_timeout(10) == N.NVFP4_ERR_INVALID_ARG
    assert N.nvfp4_selftest_wait_timeout(3_000_000_000) == N.NVFP4_ERR_INVALID_ARG
