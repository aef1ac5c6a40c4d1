"""GPU parity of the larger-order RHT quantizers (32, 64 and 128 points)
against the CPU oracle, bit for bit: codes, block scales (plain and MMA
layouts) and global scales.  Row-wise chunks span 2, 4 or 8 lanes of a warp;
transposed chunks span 2, 4 or 8 warps of a CTA (shared-memory butterflies)."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import first_mismatch, mma_layout, to_device_bf16, unpack_codes

pytestmark = pytest.mark.gpu

ORDERS = (32, 64, 128)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    N.lib()


def check(x_bits, n, transpose, rounding, rht_seed=4100, sr_seed=4101):
    q = N.quantize_1d(to_device_bf16(x_bits), transpose=transpose, rounding=rounding, sr_seed=sr_seed, rht=True,
                      rht_seed=rht_seed, rht_order=n)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    codes, scales, smma = q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.scales_mma.cpu().numpy()
    sg = np.float32(q.global_scale.cpu().item())
    oc, osc, osg = O.quantize_1d(x_bits, transpose=transpose, rht=True, rht_seed=rht_seed, rounding=rounding,
                                 sr_seed=sr_seed, rht_order=n)
    assert sg.view(np.uint32) == np.float32(osg).view(np.uint32), (sg, osg)
    assert first_mismatch(scales, osc) is None, first_mismatch(scales, osc)
    assert first_mismatch(unpack_codes(codes), unpack_codes(oc)) is None, \
        first_mismatch(unpack_codes(codes), unpack_codes(oc))
    exp_mma = mma_layout(osc, osc.shape[0], osc.shape[1])
    assert first_mismatch(smma, exp_mma) is None, first_mismatch(smma, exp_mma)


# (rows, cols) of x; row-wise: cols a multiple of n, some not of 512 (a
# partial unit at the end of each row); transposed: rows (tokens) a multiple
# of n, some not of 128 (a partial token tile), cols (features) not of 256.
ROWWISE = [(3, 128), (33, 640), (130, 1152), (16, 4096)]
TRANSPOSED = [(128, 16), (384, 272), (640, 40), (1152, 520)]


@pytest.mark.parametrize("n", ORDERS)
@pytest.mark.parametrize("shape", ROWWISE)
@pytest.mark.parametrize("rounding", [0, 1])
def test_rht_order_rowwise(n, shape, rounding):
    x = G.make_tensor(*shape, seed=200 + shape[0] + n, dist="normal", scale=1.5, outlier_frac=0.003,
                      outlier_mode="mul", outlier_value=80.0)
    check(x, n, False, rounding)


@pytest.mark.parametrize("n", ORDERS)
@pytest.mark.parametrize("shape", TRANSPOSED)
@pytest.mark.parametrize("rounding", [0, 1])
def test_rht_order_transposed(n, shape, rounding):
    if shape[0] % n:
        pytest.skip("tokens not a multiple of the order")
    x = G.make_tensor(*shape, seed=300 + shape[0] + n, dist="laplace", scale=1e-3, outlier_frac=0.001,
                      outlier_mode="mul", outlier_value=1000.0)
    check(x, n, True, rounding)


def test_rht_order_partial_token_tile():
    """Tokens = 96 with order 32: the last 128-token tile holds one empty warp."""
    x = G.make_tensor(96, 264, seed=7, dist="normal", scale=1.0)
    check(x, 32, True, 1)


@pytest.mark.parametrize("n", ORDERS)
def test_rht_order_zero_tensor(n):
    x = np.zeros((n, 256), dtype=np.uint16)
    x[::3, ::5] = 0x8000   # negative zeros
    check(x, n, True, 1)
    check(x, n, False, 0)


def test_rht_order_16_equals_the_16_point_entry():
    x = G.make_tensor(256, 512, seed=9, dist="normal", scale=1.0)
    xd = to_device_bf16(x)
    a = N.quantize_1d(xd, transpose=True, rht=True, rht_seed=5, rounding=N.NVFP4_SR, sr_seed=6)
    ws = N.workspace(xd.device)
    codes = torch.empty_like(a.codes)
    scales = torch.empty_like(a.scales)
    smma = torch.empty_like(a.scales_mma)
    gs = torch.empty_like(a.global_scale)
    N.nvfp4_rht_quantize_n(xd, 256, 512, 512, 1, 16, 5, N.NVFP4_SR, 6, codes, scales, smma, gs, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(codes, a.codes) and torch.equal(scales, a.scales) and torch.equal(smma, a.scales_mma)
    assert torch.equal(gs, a.global_scale)


def test_rht_order_argument_errors():
    xd = to_device_bf16(np.zeros((192, 256), dtype=np.uint16))
    ws = N.workspace(xd.device)
    codes = torch.empty(256, 96, dtype=torch.uint8, device=xd.device)
    scales = torch.empty(256, 12, dtype=torch.uint8, device=xd.device)
    gs = torch.empty(1, dtype=torch.float32, device=xd.device)
    st = N.lib().nvfp4_rht_quantize_n(xd.data_ptr(), 192, 256, 256, 1, 48, 1, 0, 0, codes.data_ptr(),
                                      scales.data_ptr(), None, gs.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert st == N.NVFP4_ERR_INVALID_ARG
    st = N.lib().nvfp4_rht_quantize_n(xd.data_ptr(), 192, 256, 256, 1, 128, 1, 0, 0, codes.data_ptr(),
                                      scales.data_ptr(), None, gs.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert st == N.NVFP4_ERR_UNSUPPORTED_SHAPE   # 192 tokens, order 128


def test_wgrad_gemm_with_order_128():
    """Both wgrad operands rotated with the same 128-point transform: the GEMM
    of the quantized operands matches the float64 product of the oracle's
    dequantized operands within the GEMM tolerance."""
    T, F, H = 512, 256, 384
    dy = G.make_tensor(T, F, seed=41, dist="laplace", scale=1e-3, outlier_frac=0.001, outlier_mode="mul",
                       outlier_value=1000.0)
    x = G.make_tensor(T, H, seed=42, dist="normal", scale=1.0)
    qa = N.quantize_1d(to_device_bf16(dy), transpose=True, rht=True, rht_seed=77, rounding=N.NVFP4_SR, sr_seed=78,
                       rht_order=128)
    qb = N.quantize_1d(to_device_bf16(x), transpose=True, rht=True, rht_seed=77, rounding=N.NVFP4_RNE,
                       rht_order=128)
    c = N.gemm(qa.codes, qa.scales_mma, qa.global_scale, qb.codes, qb.scales_mma, qb.global_scale, F, H, T,
               out_dtype=N.NVFP4_OUT_F32)
    torch.cuda.synchronize()
    ca, sa, sga = O.quantize_1d(dy, transpose=True, rht=True, rht_seed=77, rounding=1, sr_seed=78, rht_order=128)
    cb, sb, sgb = O.quantize_1d(x, transpose=True, rht=True, rht_seed=77, rounding=0, rht_order=128)
    a_hat = O.dequantize_f64(ca, sa, 0, sga, F, T)
    b_hat = O.dequantize_f64(cb, sb, 0, sgb, H, T)
    ref, s = O.gemm_reference(a_hat, b_hat)
    err = np.abs(c.cpu().numpy().astype(np.float64) - ref)
    assert (err <= 2e-3 * s).all(), (err / np.maximum(s, 1e-300)).max()
    # the rotation cancels along K: the product approximates dY^T X
    exact = G.bf16_bits_to_f32(dy).astype(np.float64).T @ G.bf16_bits_to_f32(x).astype(np.float64)
    rel = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    assert rel < 0.2, rel


def test_rht_order_128_full_size_sampled():
    """The wgrad gradient operand at the MLP step's size (dY 16384 x 28672,
    quantized as dY^T with SR) with the 128-point transform: global scale over
    the whole tensor and sampled rows, bit for bit."""
    from tests.test_gpu_fullsize import sample_rows
    T, F = 16384, 28672
    dy = G.gradient(T, F, seed=G.SEED_BASE["mlp_step"] + 2)
    q = N.quantize_1d(to_device_bf16(dy), transpose=True, rht=True, rht_seed=11, rounding=N.NVFP4_SR, sr_seed=12,
                      rht_order=128)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    sg = O.global_scale(O.amax(dy, transpose=True, rht=True, rht_seed=11, rht_order=128))
    assert np.float32(q.global_scale.item()) == np.float32(sg)
    rows = sample_rows(F, 6, seed=5)
    got = O.quantize_1d_rows(dy, sg, rows, transpose=True, rht=True, rht_seed=11, rounding=1, sr_seed=12,
                             rht_order=128)
    codes = q.codes[rows].cpu().numpy()
    scales = q.scales[rows].cpu().numpy()
    for i, r in enumerate(rows):
        assert np.array_equal(codes[i], got[r][0]), f"codes row {r}"
        assert np.array_equal(scales[i], got[r][1]), f"scales row {r}"
