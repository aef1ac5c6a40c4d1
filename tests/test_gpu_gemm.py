"""GPU block-scaled GEMM against the float64 oracle over the dequantized
operands: |C - C_ref| <= 2e-3 * S elementwise, S = |A_hat| . |B_hat|^T."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import to_device_bf16

pytestmark = pytest.mark.gpu

TOL = 2e-3
WORST = {}


@pytest.fixture(params=["pair", "single_sm"], autouse=True)
def gemm_kernel(request, monkeypatch):
    """Every GEMM test runs on both kernels: the CTA-pair kernel (default)
    and the single-SM kernel (NVFP4_GEMM_PAIR=0)."""
    monkeypatch.setenv("NVFP4_GEMM_PAIR", "1" if request.param == "pair" else "0")
    return request.param


def bf16_half_ulp(x):
    """Half a bf16 unit in the last place at |x| (the store rounding of a bf16 output)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def quantized_pair(a_bits, b_bits, b_2d=False):
    """Quantize A (1D) and B (1D or 2D) on the GPU; the oracle supplies the
    dequantized operands (the quantizers' bit parity is tested separately)."""
    a = N.quantize_1d(to_device_bf16(a_bits))
    if b_2d:
        b = N.quantize_2d(to_device_bf16(b_bits), columnwise=False)
        cb, _, sb, gb = O.quantize_2d(b_bits, columnwise=False)
        b_hat = O.dequantize_f64(cb, sb, 1, gb, *b_bits.shape)
    else:
        b = N.quantize_1d(to_device_bf16(b_bits))
        cb, sb, gb = O.quantize_1d(b_bits)
        b_hat = O.dequantize_f64(cb, sb, 0, gb, *b_bits.shape)
    ca, sa, ga = O.quantize_1d(a_bits)
    a_hat = O.dequantize_f64(ca, sa, 0, ga, *a_bits.shape)
    torch.cuda.synchronize()
    assert np.array_equal(a.codes.cpu().numpy(), ca) and np.array_equal(b.codes.cpu().numpy(), cb)
    return a, b, a_hat, b_hat


def check(c_gpu, a_hat, b_hat, rows=None, bf16_out=False, name=""):
    """|C - C_ref| <= 2e-3 * S; a bf16 output may in addition differ by the
    half-ulp rounding of its own store."""
    if rows is not None:
        a_hat = a_hat[rows]
        c_gpu = c_gpu[rows]
    ref, s = O.gemm_reference(a_hat, b_hat)
    err = np.abs(c_gpu.astype(np.float64) - ref)
    if bf16_out:
        err = np.maximum(err - bf16_half_ulp(ref), 0.0)
    ratio = err / np.maximum(s, 1e-300)
    WORST[name] = float(ratio.max())
    print(f"[gemm tolerance] {name}: worst |C - C_ref| / S = {ratio.max():.3e}")
    bad = err > TOL * s
    assert not bad.any(), f"{bad.sum()} elements out of tolerance; worst ratio {ratio.max()}"
    return ratio.max()


@pytest.mark.parametrize("out_dtype", [N.NVFP4_OUT_F32, N.NVFP4_OUT_BF16])
def test_gemm_tiny_linear(out_dtype):
    a_bits, w_bits = G.tiny_linear()
    a, b, a_hat, b_hat = quantized_pair(a_bits, w_bits, b_2d=True)
    c = N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, 256, 256, 256,
               out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    check(c.float().cpu().numpy(), a_hat, b_hat, bf16_out=out_dtype == N.NVFP4_OUT_BF16,
          name=f"tiny_linear out={out_dtype}")


@pytest.mark.parametrize("mnk", [(128, 256, 256), (384, 512, 1024), (200, 300, 320), (1, 8, 64),
                                 (130, 264, 192), (520, 776, 1536)])
def test_gemm_shapes_fp32(mnk):
    M, Nn, K = mnk
    a_bits = G.make_tensor(M, K, seed=M + 1, dist="normal", scale=1.0, outlier_frac=0.001, outlier_mode="mul",
                           outlier_value=50.0)
    b_bits = G.make_tensor(Nn, K, seed=Nn + 2, dist="normal", scale=0.02)
    a, b, a_hat, b_hat = quantized_pair(a_bits, b_bits)
    c = N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, M, Nn, K,
               out_dtype=N.NVFP4_OUT_F32)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    check(c.cpu().numpy(), a_hat, b_hat, name=f"fp32 {mnk}")


def test_gemm_bf16_output_and_padding_untouched():
    M, Nn, K = 136, 264, 512
    a_bits = G.make_tensor(M, K, seed=11)
    b_bits = G.make_tensor(Nn, K, seed=12, scale=0.05)
    a, b, a_hat, b_hat = quantized_pair(a_bits, b_bits)
    full = torch.full((M, 272), 7.0, dtype=torch.bfloat16, device="cuda")
    N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, M, Nn, K,
           out_dtype=N.NVFP4_OUT_BF16, out=full[:, :Nn])
    torch.cuda.synchronize()
    assert (full[:, Nn:] == 7.0).all()
    check(full[:, :Nn].float().cpu().numpy(), a_hat, b_hat, bf16_out=True, name="bf16 ldc-padded")


def test_gemm_wgrad_rotation_cancels():
    """RHT on both wgrad operands with one sign vector: the quantized product
    matches the oracle's product of the rotated operands, and approximates
    the unrotated bf16 product dY^T X."""
    T, F, H = 256, 272, 160
    dy = G.gradient(T, F, seed=31)
    x = G.activation(T, H, seed=32, outlier_frac=0.0, outlier_mul=1.0)
    qa = N.quantize_1d(to_device_bf16(dy), transpose=True, rht=True, rht_seed=33, rounding=N.NVFP4_SR, sr_seed=34)
    qb = N.quantize_1d(to_device_bf16(x), transpose=True, rht=True, rht_seed=33, rounding=N.NVFP4_RNE)
    c = N.gemm(qa.codes, qa.scales_mma, qa.global_scale, qb.codes, qb.scales_mma, qb.global_scale, F, H, T,
               out_dtype=N.NVFP4_OUT_F32)
    torch.cuda.synchronize()
    ca, sa, ga = O.quantize_1d(dy, transpose=True, rht=True, rht_seed=33, rounding=1, sr_seed=34)
    cb, sb, gb = O.quantize_1d(x, transpose=True, rht=True, rht_seed=33, rounding=0)
    assert np.array_equal(qa.codes.cpu().numpy(), ca) and np.array_equal(qb.codes.cpu().numpy(), cb)
    a_hat = O.dequantize_f64(ca, sa, 0, ga, F, T)
    b_hat = O.dequantize_f64(cb, sb, 0, gb, H, T)
    cg = c.cpu().numpy()
    check(cg, a_hat, b_hat, name="wgrad rht")
    exact = G.bf16_bits_to_f32(dy).astype(np.float64).T @ G.bf16_bits_to_f32(x).astype(np.float64)
    scale = np.abs(G.bf16_bits_to_f32(dy)).astype(np.float64).T @ np.abs(G.bf16_bits_to_f32(x)).astype(np.float64)
    assert np.abs(cg - exact).max() <= 0.25 * scale.max()
    assert np.corrcoef(cg.ravel(), exact.ravel())[0, 1] > 0.9


@pytest.mark.parametrize("mags", [(1e-18, 1e-18), (1e-25, 1e-12), (1e-30, 1e-30)])
@pytest.mark.parametrize("out_dtype", [N.NVFP4_OUT_F32, N.NVFP4_OUT_BF16])
def test_gemm_extreme_global_scales(mags, out_dtype):
    """Operands whose global scales are so small that their product
    alpha = RN(s_gA * s_gB) is not a normal binary32 number: amax 1e-18 on
    both sides gives s_g near 3.7e-22 and alpha near 1.4e-43 (subnormal,
    about 7 significant bits).  C itself is a normal number, and must meet the
    2e-3 * sum|a b| bound against the float64 product of the dequantized
    operands.  At 1e-30 C lies below the binary32 range: there the bound gets
    the format's own floor, half its smallest subnormal (2^-150; bf16 shares
    the exponent range, half its smallest subnormal is 2^-134)."""
    M, Nn, K = 136, 264, 256
    ma, mb = mags
    a_bits = G.make_tensor(M, K, seed=91, dist="normal", scale=ma)
    b_bits = G.make_tensor(Nn, K, seed=92, dist="normal", scale=mb)
    a, b, a_hat, b_hat = quantized_pair(a_bits, b_bits)
    sa, sb = float(a.global_scale.item()), float(b.global_scale.item())
    prod = np.float32(sa) * np.float32(sb)
    assert prod < np.float32(2.0 ** -126)          # alpha would be subnormal or zero
    c = N.gemm(a.codes, a.scales_mma, a.global_scale, b.codes, b.scales_mma, b.global_scale, M, Nn, K,
               out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    cg = c.float().cpu().numpy().astype(np.float64)
    ref, s = O.gemm_reference(a_hat, b_hat)
    err = np.abs(cg - ref)
    bf16 = out_dtype == N.NVFP4_OUT_BF16
    if bf16:
        err = np.maximum(err - bf16_half_ulp(ref), 0.0)
    floor = 2.0 ** -134 if bf16 else 2.0 ** -150
    assert np.isfinite(cg).all()
    bad = err > TOL * s + floor
    assert not bad.any(), f"{bad.sum()} out of tolerance; worst {(err / np.maximum(s, 1e-300)).max()}"
    if ma == mb == 1e-30:
        assert (np.abs(ref) < 2.0 ** -149).all()     # the case really is below the binary32 range
    else:
        assert (np.abs(ref[np.abs(ref) > 0]) >= 2.0 ** -126).mean() > 0.99
