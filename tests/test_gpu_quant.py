"""GPU parity of the quantizers against the CPU oracle: codes, block scales
(plain and MMA layouts) and global scales must match bit for bit."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import first_mismatch, mma_layout, to_device_bf16, unpack_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    N.lib()


def run_1d(x_bits, transpose=False, rht=False, rht_seed=0, rounding=0, sr_seed=0):
    x = to_device_bf16(x_bits)
    q = N.quantize_1d(x, transpose=transpose, rounding=rounding, sr_seed=sr_seed, rht=rht, rht_seed=rht_seed)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    return (q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.scales_mma.cpu().numpy(),
            np.float32(q.global_scale.cpu().item()))


def check_1d(x_bits, **kw):
    codes, scales, smma, sg = run_1d(x_bits, **kw)
    oc, osc, osg = O.quantize_1d(x_bits, transpose=kw.get("transpose", False), rht=kw.get("rht", False),
                                 rht_seed=kw.get("rht_seed", 0), rounding=kw.get("rounding", 0),
                                 sr_seed=kw.get("sr_seed", 0))
    assert np.float32(sg).view(np.uint32) == np.float32(osg).view(np.uint32), (sg, osg)
    assert first_mismatch(scales, osc) is None, first_mismatch(scales, osc)
    assert first_mismatch(unpack_codes(codes), unpack_codes(oc)) is None, \
        first_mismatch(unpack_codes(codes), unpack_codes(oc))
    exp_mma = mma_layout(osc, osc.shape[0], osc.shape[1])
    assert first_mismatch(smma, exp_mma) is None, first_mismatch(smma, exp_mma)


SHAPES_1D = [(1, 16), (3, 48), (33, 1040), (257, 512), (300, 4096), (16, 8192)]


@pytest.mark.parametrize("shape", SHAPES_1D)
@pytest.mark.parametrize("rounding", [0, 1])
def test_quantize_1d_rowwise(shape, rounding):
    x = G.make_tensor(*shape, seed=100 + shape[0], dist="normal", scale=2.0, outlier_frac=0.003,
                      outlier_mode="mul", outlier_value=80.0)
    check_1d(x, rounding=rounding, sr_seed=77)


def test_quantize_1d_tiny_linear_activation():
    a, _ = G.tiny_linear()
    check_1d(a)


@pytest.mark.parametrize("shape", [(16, 8), (64, 48), (160, 264), (272, 520)])
@pytest.mark.parametrize("rounding", [0, 1])
def test_quantize_1d_transposed(shape, rounding):
    x = G.make_tensor(*shape, seed=200 + shape[1], dist="laplace", scale=1e-3, outlier_frac=0.002,
                      outlier_mode="mul", outlier_value=1000.0)
    check_1d(x, transpose=True, rounding=rounding, sr_seed=5)


@pytest.mark.parametrize("shape", [(16, 8), (64, 48), (160, 264), (400, 1032)])
@pytest.mark.parametrize("rounding", [0, 1])
def test_rht_quantize_transposed(shape, rounding):
    x = G.make_tensor(*shape, seed=300 + shape[0], dist="laplace", scale=1e-3, outlier_frac=0.002,
                      outlier_mode="mul", outlier_value=1000.0)
    check_1d(x, transpose=True, rht=True, rht_seed=3100, rounding=rounding, sr_seed=3101)


@pytest.mark.parametrize("shape", [(1, 16), (5, 64), (33, 1040)])
@pytest.mark.parametrize("rounding", [0, 1])
def test_rht_quantize_rowwise(shape, rounding):
    x = G.make_tensor(*shape, seed=400 + shape[0], dist="normal", scale=1.0, outlier_frac=0.01,
                      outlier_mode="set", outlier_value=1e4)
    check_1d(x, rht=True, rht_seed=9, rounding=rounding, sr_seed=10)


# ------------------------------------------------------------ edge cases ----
def _bits(vals):
    return G._to_bf16_bits(np.asarray(vals, dtype=np.float32))


def test_all_bf16_values_sweep():
    """Every finite bf16 value as an element (blocks hold consecutive bit
    patterns, so block scales also sweep the whole range)."""
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = G.bf16_bits_to_f32(h)
    h = h[np.isfinite(f)]
    n = (h.size + 4095) // 4096 * 4096
    x = np.zeros(n, dtype=np.uint16)
    x[: h.size] = h
    x = x.reshape(-1, 4096)
    for rounding in (0, 1):
        check_1d(x, rounding=rounding, sr_seed=1)
    # the same sweep with a moderate amax, so that mid-range values hit every E2M1 decision
    small = h[np.abs(G.bf16_bits_to_f32(h)) < 64]
    n = (small.size + 16 * 1024 - 1) // (16 * 1024) * (16 * 1024)
    y = np.zeros(n, dtype=np.uint16)
    y[: small.size] = small
    y = y.reshape(-1, 1024)
    for rounding in (0, 1):
        check_1d(y, rounding=rounding, sr_seed=2)
        check_1d(y, transpose=True, rounding=rounding, sr_seed=3)


def test_zero_and_signed_zero_tensor():
    x = np.zeros((4, 64), dtype=np.uint16)
    x[1, 5] = 0x8000
    for rounding in (0, 1):
        check_1d(x, rounding=rounding)
        check_1d(x, rht=True, rounding=rounding)


def test_tiny_and_huge_magnitudes():
    rng = np.random.default_rng(3)
    tiny = (rng.standard_normal((8, 64)) * 2.0 ** -128).astype(np.float32)     # bf16 subnormals
    check_1d(_bits(tiny))
    check_1d(_bits(tiny), rounding=1)
    huge = (rng.standard_normal((8, 64)) * 1e37).astype(np.float32)
    check_1d(_bits(huge))
    check_1d(_bits(huge), rht=True, rounding=1)


def test_rht_subnormal_inputs():
    """RHT of bf16 subnormals: the butterfly sums and their quarter fall in
    binary32's subnormal range, where the amax passes' single 1/4 scaling of
    the maximum must still equal the maximum of the scaled values."""
    rng = np.random.default_rng(5)
    tiny = (rng.standard_normal((32, 64)) * 2.0 ** -130).astype(np.float32)
    tiny[3, 7] = 2.0 ** -133                      # bf16's smallest subnormal
    tiny[20, 40] = -(2.0 ** -126)
    x = _bits(tiny)
    for rounding in (0, 1):
        check_1d(x, rht=True, rounding=rounding, sr_seed=4)
        check_1d(x, transpose=True, rht=True, rounding=rounding, sr_seed=4)


def test_scale_underflow_blocks():
    vals = np.full((2, 64), 2.0 ** -12, dtype=np.float32)
    vals[0, 0] = 3e4
    vals[1, 17] = -2.0 ** -20
    check_1d(_bits(vals))
    check_1d(_bits(vals), rounding=1)


def test_strided_input():
    x = G.make_tensor(40, 96, seed=7)
    xd = to_device_bf16(x)[:, :64]
    q = N.quantize_1d(xd)
    oc, osc, osg = O.quantize_1d(np.ascontiguousarray(x[:, :64]))
    assert np.array_equal(q.codes.cpu().numpy(), oc) and np.array_equal(q.scales.cpu().numpy(), osc)
    assert q.global_scale.item() == osg


def test_sr_is_reproducible_and_seeded():
    x = G.make_tensor(64, 256, seed=8, dist="laplace", scale=1e-3)
    a = run_1d(x, rounding=1, sr_seed=11)
    b = run_1d(x, rounding=1, sr_seed=11)
    c = run_1d(x, rounding=1, sr_seed=12)
    assert np.array_equal(a[0], b[0]) and not np.array_equal(a[0], c[0])


# --------------------------------------------------------------------- 2D ---
@pytest.mark.parametrize("shape", [(16, 16), (32, 48), (128, 256), (272, 528), (400, 784)])
def test_quantize_2d(shape):
    w = G.make_tensor(*shape, seed=500 + shape[0], dist="normal", scale=0.02, outlier_frac=0.002,
                      outlier_mode="mul", outlier_value=30.0)
    q = N.quantize_2d(to_device_bf16(w))
    torch.cuda.synchronize()
    cr, cc, sc, sg = O.quantize_2d(w)
    R, C = shape
    assert q.global_scale.item() == sg
    assert first_mismatch(q.scales.cpu().numpy(), sc) is None
    assert first_mismatch(unpack_codes(q.codes.cpu().numpy()), unpack_codes(cr)) is None
    assert first_mismatch(unpack_codes(q.codes_col.cpu().numpy()), unpack_codes(cc)) is None
    assert first_mismatch(q.scales_mma.cpu().numpy(), mma_layout(sc, R, C // 16, expand_2d=True)) is None
    assert first_mismatch(q.scales_mma_col.cpu().numpy(), mma_layout(np.ascontiguousarray(sc.T), C, R // 16,
                                                                     expand_2d=True)) is None


def test_quantize_2d_ragged_multi_wave():
    """More 128 x 256 tiles (21 x 17 = 357) than CTAs, with a 16-row last
    tile row and a 16-column last tile column: every CTA prefetches a next
    tile, some of them ragged."""
    w = G.make_tensor(2576, 4112, seed=580, dist="normal", scale=0.02, outlier_frac=0.001,
                      outlier_mode="mul", outlier_value=30.0)
    q = N.quantize_2d(to_device_bf16(w))
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    cr, cc, sc, sg = O.quantize_2d(w)
    R, C = w.shape
    assert q.global_scale.item() == sg
    assert first_mismatch(q.scales.cpu().numpy(), sc) is None
    assert first_mismatch(q.codes.cpu().numpy(), cr) is None
    assert first_mismatch(q.codes_col.cpu().numpy(), cc) is None
    assert first_mismatch(q.scales_mma.cpu().numpy(), mma_layout(sc, R, C // 16, expand_2d=True)) is None
    assert first_mismatch(q.scales_mma_col.cpu().numpy(), mma_layout(np.ascontiguousarray(sc.T), C, R // 16,
                                                                     expand_2d=True)) is None


def test_quantize_2d_tiny_linear_weight():
    _, w = G.tiny_linear()
    q = N.quantize_2d(to_device_bf16(w), columnwise=False)
    cr, _, sc, sg = O.quantize_2d(w, columnwise=False)
    assert q.global_scale.item() == sg
    assert np.array_equal(q.codes.cpu().numpy(), cr) and np.array_equal(q.scales.cpu().numpy(), sc)


# ------------------------------------------------------------- dequantize ---
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("out_dtype", [N.NVFP4_OUT_F32, N.NVFP4_OUT_BF16])
def test_dequantize(mode, out_dtype):
    x = G.make_tensor(64, 160, seed=600, dist="normal", scale=3.0, outlier_frac=0.01, outlier_mode="mul",
                      outlier_value=40.0)
    if mode == 0:
        oc, osc, osg = O.quantize_1d(x)
    else:
        oc, _, osc, osg = O.quantize_2d(x, columnwise=False)
    exp = O.dequantize(oc, osc, mode, osg, 64, 160)
    q = N.Quantized(torch.from_numpy(oc).cuda(), torch.from_numpy(osc).cuda(), None,
                    torch.tensor([osg], dtype=torch.float32, device="cuda"), 64, 160)
    out = N.dequantize(q, scale_mode=mode, out_dtype=out_dtype).cpu()
    if out_dtype == N.NVFP4_OUT_F32:
        assert np.array_equal(out.numpy().view(np.uint32), exp.view(np.uint32))
    else:
        ref = torch.from_numpy(exp).to(torch.bfloat16)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_scales_to_mma():
    rng = np.random.default_rng(9)
    for rows, k, mode in [(200, 320, 0), (128, 256, 0), (48, 96, 1)]:
        plain = rng.integers(0, 0x7F, size=((rows // 16) if mode else rows, k // 16)).astype(np.uint8)
        dst = torch.empty(N.nvfp4_mma_scale_bytes(rows, k), dtype=torch.uint8, device="cuda")
        N.nvfp4_scales_to_mma(torch.from_numpy(plain).cuda(), mode, rows, k, dst)
        assert np.array_equal(dst.cpu().numpy(), mma_layout(plain, rows, k // 16, expand_2d=bool(mode)))


@pytest.mark.parametrize("ld", [72, 96])
@pytest.mark.parametrize("rht", [False, True])
def test_strided_input_sr(ld, rht):
    """Stochastic rounding (and the 16-point RHT) on a strided view: rows of
    64 elements every `ld` elements.  ld = 72 leaves every other row 16-byte
    but not 32-byte aligned, so the encode pass takes its two-load path."""
    x = G.make_tensor(40, ld, seed=9 + ld, dist="laplace", scale=1e-3, outlier_frac=0.01, outlier_mode="mul",
                      outlier_value=500.0)
    xd = to_device_bf16(x)[:, :64]
    q = N.quantize_1d(xd, rounding=N.NVFP4_SR, sr_seed=21, rht=rht, rht_seed=22)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    oc, osc, osg = O.quantize_1d(np.ascontiguousarray(x[:, :64]), rht=rht, rht_seed=22, rounding=1, sr_seed=21)
    assert np.array_equal(q.codes.cpu().numpy(), oc) and np.array_equal(q.scales.cpu().numpy(), osc)
    assert np.array_equal(q.scales_mma.cpu().numpy(), mma_layout(osc, 40, 4))
    assert q.global_scale.item() == osg


@pytest.mark.parametrize("ld", [72, 264])
@pytest.mark.parametrize("rounding", [0, 1])
def test_strided_input_transposed_rht(ld, rounding):
    """Q = RHT(x^T) of a strided view (tokens x 64 features every `ld`
    elements): the transposed encode reads through the stride and writes Q's
    rows (one per feature) whole; the SR variant stores its codes straight
    from registers, the RNE one through shared memory."""
    x = G.make_tensor(48, ld, seed=30 + ld, dist="laplace", scale=1e-3, outlier_frac=0.01, outlier_mode="mul",
                      outlier_value=500.0)
    xd = to_device_bf16(x)[:, :64]
    q = N.quantize_1d(xd, transpose=True, rounding=rounding, sr_seed=23, rht=True, rht_seed=24)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    oc, osc, osg = O.quantize_1d(np.ascontiguousarray(x[:, :64]), transpose=True, rht=True, rht_seed=24,
                                 rounding=rounding, sr_seed=23)
    assert np.array_equal(q.codes.cpu().numpy(), oc) and np.array_equal(q.scales.cpu().numpy(), osc)
    assert np.array_equal(q.scales_mma.cpu().numpy(), mma_layout(osc, 64, 3))
    assert q.global_scale.item() == osg
