"""Parity at the workloads' full sizes, in the launch configuration the bench
times: the oracle computes the tensor amax over the whole tensor and then
sampled output rows one by one; the GEMMs are checked on sampled rows of C
against float64 products over the oracle's dequantized operands."""
import numpy as np
import pytest
import torch

from nvfp4_bit_block_amax_b200 import inputs as G
from nvfp4_bit_block_amax_b200 import nvfp4 as N
from oracle import oracle as O
from tests.helpers import mma_layout, to_device_bf16, unpack_codes

pytestmark = pytest.mark.gpu

TOL = 2e-3


def sample_rows(n, k=12, seed=0):
    rng = np.random.default_rng(seed)
    rows = set([0, n - 1, n // 2]) | set(rng.integers(0, n, size=k).tolist())
    return sorted(rows)


def check_quantized_rows(q, x_bits, rows, transpose=False, rht=False, rht_seed=0, rounding=0, sr_seed=0):
    amax = O.amax(x_bits, transpose=transpose, rht=rht, rht_seed=rht_seed)
    sg = O.global_scale(amax)
    assert np.float32(q.global_scale.item()) == np.float32(sg)
    got = O.quantize_1d_rows(x_bits, sg, rows, transpose=transpose, rht=rht, rht_seed=rht_seed, rounding=rounding,
                             sr_seed=sr_seed)
    codes = q.codes.cpu().numpy()
    smma = q.scales_mma.cpu().numpy()
    qc = q.cols
    for r in rows:
        oc, osc = got[r]
        assert np.array_equal(codes[r], oc), f"codes row {r}"
        kb = qc // 16
        ck = (kb + 3) // 4
        b = np.arange(kb)
        off = ((r // 128) * ck + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
        assert np.array_equal(smma[off], osc), f"scales row {r}"
    return sg


def dequant_rows(q_codes_rows, q_scales_rows, sg, cols):
    return O.dequantize_f64(q_codes_rows, q_scales_rows, 0, sg, q_codes_rows.shape[0], cols)


def gemm_rows_check(c_rows_gpu, a_hat_rows, b_hat):
    ref, s = O.gemm_reference(a_hat_rows, b_hat)
    err = np.abs(c_rows_gpu.astype(np.float64) - ref)
    # bf16 output: the store itself may round by half a bf16 ulp
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126)))
    err = np.maximum(err - 2.0 ** (e - 8), 0)
    ratio = (err / np.maximum(s, 1e-300)).max()
    print(f"[gemm tolerance] worst |C - C_ref| / S = {ratio:.3e}")
    assert (err <= TOL * s).all(), ratio


def test_mlp_fprop_full_size():
    """X [8192 x 4096] 1D RNE, W1 [14336 x 4096] 2D RNE, Y = X W1^T (bf16)."""
    t, h, f = G.MLP_FPROP["tokens"], G.MLP_FPROP["hidden"], G.MLP_FPROP["ffn"]
    seed, _, _ = G.seeds("mlp_fprop")
    x = G.activation(t, h, seed)
    w = G.weight(f, h, seed + 1)
    qx = N.quantize_1d(to_device_bf16(x), plain_scales=False)
    qw = N.quantize_2d(to_device_bf16(w), columnwise=False)
    y = N.gemm(qx.codes, qx.scales_mma, qx.global_scale, qw.codes, qw.scales_mma, qw.global_scale, t, f, h)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    rows = sample_rows(t, 8, seed=1)
    sgx = check_quantized_rows(qx, x, rows)
    cw, _, sw, sgw = O.quantize_2d(w, columnwise=False)
    assert np.float32(qw.global_scale.item()) == sgw
    assert np.array_equal(qw.codes.cpu().numpy(), cw) and np.array_equal(qw.scales.cpu().numpy(), sw)
    got = O.quantize_1d_rows(x, sgx, rows)
    a_hat = np.concatenate([O.dequantize_f64(got[r][0][None], got[r][1][None], 0, sgx, 1, h) for r in rows])
    w_hat = O.dequantize_f64(cw, sw, 1, sgw, f, h)
    gemm_rows_check(y[rows].float().cpu().numpy(), a_hat, w_hat)


def test_mlp_wgrad_full_size():
    """dY [8192 x 14336], X [8192 x 4096]; both transposed (K = tokens), RHT,
    dY SR, X RNE; dW = dY^T X [14336 x 4096]."""
    t, h, f = G.MLP_WGRAD["tokens"], G.MLP_WGRAD["hidden"], G.MLP_WGRAD["ffn"]
    seed, rs, ss = G.seeds("mlp_wgrad")
    dy = G.gradient(t, f, seed + 2)
    x = G.activation(t, h, seed, outlier_frac=0.0, outlier_mul=1.0)
    qa = N.quantize_1d(to_device_bf16(dy), transpose=True, rht=True, rht_seed=rs, rounding=N.NVFP4_SR, sr_seed=ss,
                       plain_scales=False)
    qb = N.quantize_1d(to_device_bf16(x), transpose=True, rht=True, rht_seed=rs, rounding=N.NVFP4_RNE,
                       plain_scales=False)
    dw = N.gemm(qa.codes, qa.scales_mma, qa.global_scale, qb.codes, qb.scales_mma, qb.global_scale, f, h, t)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    rows = sample_rows(f, 8, seed=2)
    sga = check_quantized_rows(qa, dy, rows, transpose=True, rht=True, rht_seed=rs, rounding=1, sr_seed=ss)
    cb, sb, sgb = O.quantize_1d(x, transpose=True, rht=True, rht_seed=rs, rounding=0)
    assert np.float32(qb.global_scale.item()) == sgb
    assert np.array_equal(qb.codes.cpu().numpy(), cb)
    assert np.array_equal(qb.scales_mma.cpu().numpy(), mma_layout(sb, h, t // 16))
    got = O.quantize_1d_rows(dy, sga, rows, transpose=True, rht=True, rht_seed=rs, rounding=1, sr_seed=ss)
    a_hat = np.concatenate([O.dequantize_f64(got[r][0][None], got[r][1][None], 0, sga, 1, t) for r in rows])
    b_hat = O.dequantize_f64(cb, sb, 0, sgb, h, t)
    gemm_rows_check(dw[rows].float().cpu().numpy(), a_hat, b_hat)


@pytest.mark.parametrize("n", [1 << 20, 1 << 24, 1 << 28])
@pytest.mark.parametrize("dist", G.SWEEP_DISTS)
def test_quantizer_sweep(n, dist):
    seed = G.seeds("sweep")[0] + n.bit_length() * 10 + G.SWEEP_DISTS.index(dist)
    x = G.sweep_tensor(n, dist, seed)
    rows_n, cols = x.shape
    xd = to_device_bf16(x)
    rows = sample_rows(rows_n, 6, seed=n.bit_length())
    q = N.quantize_1d(xd)
    torch.cuda.synchronize()
    check_quantized_rows(q, x, rows)
    del q
    q2 = N.quantize_2d(xd, columnwise=False)
    torch.cuda.synchronize()
    sg = O.global_scale(O.amax(x))
    assert np.float32(q2.global_scale.item()) == np.float32(sg)
    tiles = sorted(set(r // 16 for r in rows))
    got = O.quantize_2d_tiles(x, sg, tiles)
    codes = q2.codes.cpu().numpy()
    scales = q2.scales.cpu().numpy()
    for tr in tiles:
        assert np.array_equal(codes[16 * tr:16 * tr + 16], got[tr][0]) and np.array_equal(scales[tr], got[tr][1])
    del q2
    q3 = N.quantize_1d(xd, rht=True, rht_seed=seed + 100, rounding=N.NVFP4_SR, sr_seed=seed + 101)
    torch.cuda.synchronize()
    check_quantized_rows(q3, x, rows, rht=True, rht_seed=seed + 100, rounding=1, sr_seed=seed + 101)
    del q3
    if n <= (1 << 28):
        q4 = N.quantize_1d(xd, transpose=True, rht=True, rht_seed=seed + 100, rounding=N.NVFP4_SR, sr_seed=seed + 102)
        torch.cuda.synchronize()
        check_quantized_rows(q4, x, sample_rows(cols, 6, seed=3), transpose=True, rht=True, rht_seed=seed + 100,
                             rounding=1, sr_seed=seed + 102)


def check_2d_tiles(q2, x, tiles):
    """2D outputs on sampled 16-row tile rows against the oracle: row codes,
    plain tile scales, the W^T codes of those tiles' columns (the same codes
    transposed, the pages' "row- and column-wise quantization agree"), and
    both MMA scale layouts at the positions those tiles fill."""
    R, C = x.shape
    sg = O.global_scale(O.amax(x))
    assert np.float32(q2.global_scale.item()) == np.float32(sg)
    got = O.quantize_2d_tiles(x, sg, tiles)
    codes = q2.codes.cpu().numpy()
    scales = q2.scales.cpu().numpy() if q2.scales is not None else None
    ccol = q2.codes_col.cpu().numpy() if q2.codes_col is not None else None
    mrow = q2.scales_mma.cpu().numpy() if q2.scales_mma is not None else None
    mcol = q2.scales_mma_col.cpu().numpy() if q2.scales_mma_col is not None else None
    kb_row, kb_col = C // 16, R // 16
    for tr in tiles:
        oc, osc = got[tr]
        assert np.array_equal(codes[16 * tr:16 * tr + 16], oc), f"row codes, tile row {tr}"
        if scales is not None:
            assert np.array_equal(scales[tr], osc), f"tile scales, tile row {tr}"
        if ccol is not None:
            nib = unpack_codes(oc)                          # [16 x C] codes of rows 16tr .. 16tr+15
            exp = nib.T                                     # [C x 16]: W^T rows, K positions 16tr ..
            exp_bytes = (exp[:, 0::2] | (exp[:, 1::2] << 4)).astype(np.uint8)
            assert np.array_equal(ccol[:, 8 * tr:8 * tr + 8], exp_bytes), f"W^T codes, tile row {tr}"
        if mrow is not None:
            ck = (kb_row + 3) // 4
            r = np.arange(16 * tr, 16 * tr + 16)[:, None]
            b = np.arange(kb_row)[None, :]
            off = ((r // 128) * ck + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
            assert np.array_equal(mrow[off], np.broadcast_to(osc, (16, kb_row))), f"MMA scales, tile row {tr}"
        if mcol is not None:
            ck = (kb_col + 3) // 4
            c = np.arange(C)
            off = ((c // 128) * ck + tr // 4) * 512 + (c % 32) * 16 + ((c // 32) % 4) * 4 + (tr % 4)
            assert np.array_equal(mcol[off], osc[c // 16]), f"MMA scales of W^T, tile row {tr}"
    return sg


def test_quantizer_max_size_rowwise():
    """The sweep's largest tensor (2^30 elements), 1D RNE."""
    n = 1 << 30
    x = G.sweep_tensor(n, "normal", G.seeds("sweep")[0] + 999)
    q = N.quantize_1d(to_device_bf16(x), plain_scales=False)
    torch.cuda.synchronize()
    check_quantized_rows(q, x, sample_rows(x.shape[0], 6, seed=9))


@pytest.mark.parametrize("dist", ["outliers"])
def test_quantizer_max_size_all_modes(dist):
    """2^30 elements (262144 x 4096 bf16, a 2 GiB input: byte offsets past
    2^31) through the 2D quantizer (row codes, W^T codes, plain and both MMA
    scale layouts), the row-wise RHT + SR quantizer and the transposed RHT +
    SR quantizer, each on sampled rows / tile rows against the oracle, which
    computes the tensor amax over the whole (rotated) tensor."""
    n = 1 << 30
    seed = G.seeds("sweep")[0] + 998
    x = G.sweep_tensor(n, dist, seed)
    R, C = x.shape
    xd = to_device_bf16(x)
    rows = sample_rows(R, 5, seed=10)
    q2 = N.quantize_2d(xd, columnwise=True)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    check_2d_tiles(q2, x, sorted(set(r // 16 for r in rows)))
    del q2
    torch.cuda.empty_cache()
    q3 = N.quantize_1d(xd, rht=True, rht_seed=seed + 100, rounding=N.NVFP4_SR, sr_seed=seed + 101,
                       plain_scales=False)
    torch.cuda.synchronize()
    check_quantized_rows(q3, x, rows, rht=True, rht_seed=seed + 100, rounding=1, sr_seed=seed + 101)
    del q3
    torch.cuda.empty_cache()
    q4 = N.quantize_1d(xd, transpose=True, rht=True, rht_seed=seed + 100, rounding=N.NVFP4_SR, sr_seed=seed + 102,
                       plain_scales=False)
    torch.cuda.synchronize()
    check_quantized_rows(q4, x, sample_rows(C, 5, seed=11), transpose=True, rht=True, rht_seed=seed + 100,
                         rounding=1, sr_seed=seed + 102)


@pytest.mark.parametrize("mode", [N.NVFP4_SCALE_1D, N.NVFP4_SCALE_2D])
@pytest.mark.parametrize("out_dtype", [N.NVFP4_OUT_F32, N.NVFP4_OUT_BF16])
def test_dequantize_full_size(mode, out_dtype):
    """Dequantize at the step's activation size (16384 x 8192): the GPU's
    codes are first checked against the oracle on sampled rows, then the GPU
    dequantization of those rows against the oracle's dequantization of its
    own codes (bf16 output: the binary32 value rounded to nearest even)."""
    t, h = G.MLP_STEP["tokens"], G.MLP_STEP["hidden"]
    seed = G.seeds("mlp_step")[0] + 30 + mode
    x = G.activation(t, h, seed) if mode == N.NVFP4_SCALE_1D else G.weight(t, h, seed)
    xd = to_device_bf16(x)
    rows = sample_rows(t, 6, seed=12)
    if mode == N.NVFP4_SCALE_1D:
        q = N.quantize_1d(xd, mma_scales=False)
        torch.cuda.synchronize()
        sg = O.global_scale(O.amax(x))
        got = O.quantize_1d_rows(x, sg, rows)
        codes, scales = q.codes.cpu().numpy(), q.scales.cpu().numpy()
        exp = {}
        for r in rows:
            assert np.array_equal(codes[r], got[r][0]) and np.array_equal(scales[r], got[r][1])
            exp[r] = O.dequantize(got[r][0][None], got[r][1][None], 0, sg, 1, h)[0]
    else:
        q = N.quantize_2d(xd, columnwise=False, mma_scales=False)
        torch.cuda.synchronize()
        tiles = sorted(set(r // 16 for r in rows))
        sg = check_2d_tiles(q, x, tiles)
        got = O.quantize_2d_tiles(x, sg, tiles)
        exp = {}
        for r in rows:
            oc, osc = got[r // 16]
            exp[r] = O.dequantize(oc, osc[None], 1, sg, 16, h)[r % 16]
    out = N.dequantize(q, scale_mode=mode, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    for r in rows:
        g = out[r].cpu()
        if out_dtype == N.NVFP4_OUT_F32:
            assert np.array_equal(g.numpy().view(np.uint32), exp[r].view(np.uint32)), f"row {r}"
        else:
            ref = torch.from_numpy(exp[r]).to(torch.bfloat16)
            assert torch.equal(g.view(torch.int16), ref.view(torch.int16)), f"row {r}"


def test_mlp_step_full_size():
    """The bench's step (tokens 16384, hidden 8192, ffn 28672): fprop, dgrad,
    wgrad GEMMs with their quantizers, sampled rows against the oracle."""
    t, h, f = G.MLP_STEP["tokens"], G.MLP_STEP["hidden"], G.MLP_STEP["ffn"]
    seed, rs, ss = G.seeds("mlp_step")
    x = G.activation(t, h, seed)
    w = G.weight(f, h, seed + 1)
    dy = G.gradient(t, f, seed + 2)
    xd, wd, dyd = to_device_bf16(x), to_device_bf16(w), to_device_bf16(dy)
    qx = N.quantize_1d(xd, plain_scales=False)
    qw = N.quantize_2d(wd)
    qdy = N.quantize_1d(dyd, rounding=N.NVFP4_SR, sr_seed=ss, plain_scales=False)
    y = N.gemm(qx.codes, qx.scales_mma, qx.global_scale, qw.codes, qw.scales_mma, qw.global_scale, t, f, h)
    dx = N.gemm(qdy.codes, qdy.scales_mma, qdy.global_scale, qw.codes_col, qw.scales_mma_col, qw.global_scale,
                t, h, f)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    rows = sample_rows(t, 4, seed=5)
    sgx = check_quantized_rows(qx, x, rows)
    sgd = check_quantized_rows(qdy, dy, rows, rounding=1, sr_seed=ss)
    cw, ccw, sw, sgw = O.quantize_2d(w)
    assert np.float32(qw.global_scale.item()) == sgw
    assert np.array_equal(qw.codes.cpu().numpy(), cw) and np.array_equal(qw.codes_col.cpu().numpy(), ccw)
    gx = O.quantize_1d_rows(x, sgx, rows)
    gd = O.quantize_1d_rows(dy, sgd, rows, rounding=1, sr_seed=ss)
    xh = np.concatenate([O.dequantize_f64(gx[r][0][None], gx[r][1][None], 0, sgx, 1, h) for r in rows])
    dyh = np.concatenate([O.dequantize_f64(gd[r][0][None], gd[r][1][None], 0, sgd, 1, f) for r in rows])
    wh = O.dequantize_f64(cw, sw, 1, sgw, f, h)
    gemm_rows_check(y[rows].float().cpu().numpy(), xh, wh)
    gemm_rows_check(dx[rows].float().cpu().numpy(), dyh, np.ascontiguousarray(wh.T))
    del y, dx, qx, qdy, wh
    torch.cuda.empty_cache()
    qa = N.quantize_1d(dyd, transpose=True, rht=True, rht_seed=rs, rounding=N.NVFP4_SR, sr_seed=ss + 1,
                       plain_scales=False)
    qb = N.quantize_1d(xd, transpose=True, rht=True, rht_seed=rs, rounding=N.NVFP4_RNE, plain_scales=False)
    dw = N.gemm(qa.codes, qa.scales_mma, qa.global_scale, qb.codes, qb.scales_mma, qb.global_scale, f, h, t)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    rows_f = sample_rows(f, 4, seed=6)
    sga = check_quantized_rows(qa, dy, rows_f, transpose=True, rht=True, rht_seed=rs, rounding=1, sr_seed=ss + 1)
    cb, sb, sgb = O.quantize_1d(x, transpose=True, rht=True, rht_seed=rs, rounding=0)
    assert np.float32(qb.global_scale.item()) == sgb and np.array_equal(qb.codes.cpu().numpy(), cb)
    ga = O.quantize_1d_rows(dy, sga, rows_f, transpose=True, rht=True, rht_seed=rs, rounding=1, sr_seed=ss + 1)
    ah = np.concatenate([O.dequantize_f64(ga[r][0][None], ga[r][1][None], 0, sga, 1, t) for r in rows_f])
    bh = O.dequantize_f64(cb, sb, 0, sgb, h, t)
    gemm_rows_check(dw[rows_f].float().cpu().numpy(), ah, bh)


def test_mxfp4_full_size_sampled_rows():
    """MXFP4 of the MLP step's activation (16384 x 8192) and an MXFP4 GEMM at
    the fprop shape: sampled rows against the oracle (MXFP4 has no tensor
    scale, so a row's codes depend on that row alone)."""
    T, H = G.MLP_STEP["tokens"], G.MLP_STEP["hidden"]
    sb = G.SEED_BASE["mlp_step"]
    x_bits = G.activation(T, H, seed=sb + 20)
    qx = N.mxfp4_quantize(to_device_bf16(x_bits))
    w_bits = G.weight(4096, H, seed=sb + 21)
    qw = N.mxfp4_quantize(to_device_bf16(w_bits))
    c = N.mxfp4_gemm(qx, qw, out_dtype=N.NVFP4_OUT_F32)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error() == 0
    rows = sample_rows(T, seed=7)
    codes_x, scales_x = O.mx_quantize(x_bits[rows])
    assert np.array_equal(qx.codes.cpu().numpy()[rows], codes_x)
    assert np.array_equal(qx.scales.cpu().numpy()[rows], scales_x)
    cw, sw = O.mx_quantize(w_bits)
    assert np.array_equal(qw.codes.cpu().numpy(), cw)
    ref, s = O.mx_gemm_reference(codes_x, scales_x, cw, sw, len(rows), 4096, H)
    err = np.abs(c.cpu().numpy()[rows].astype(np.float64) - ref)
    assert (err <= TOL * s).all(), float((err / np.maximum(s, 1e-300)).max())


def test_mlp_step_dual_quantizer_full_size():
    """The step's dual quantizer calls at full size (X RNE, dY SR) are
    bit-identical to the separate calls that the step test checks against the
    oracle."""
    t, h, f = G.MLP_STEP["tokens"], G.MLP_STEP["hidden"], G.MLP_STEP["ffn"]
    seed, rs, ss = G.seeds("mlp_step")
    for bits, rnd, s1, s2 in ((G.activation(t, h, seed), N.NVFP4_RNE, 0, 0),
                              (G.gradient(t, f, seed + 2), N.NVFP4_SR, ss, ss + 1)):
        xd = to_device_bf16(bits)
        q1, q2 = N.quantize_dual(xd, rounding=rnd, sr_seed=s1, rht_seed=rs, sr_seed_t=s2)
        a = N.quantize_1d(xd, rounding=rnd, sr_seed=s1)
        b = N.quantize_1d(xd, transpose=True, rht=True, rht_seed=rs, rounding=rnd, sr_seed=s2)
        torch.cuda.synchronize()
        assert N.nvfp4_get_error() == 0
        for u, v in ((q1.codes, a.codes), (q1.scales_mma, a.scales_mma), (q1.global_scale, a.global_scale),
                     (q2.codes, b.codes), (q2.scales_mma, b.scales_mma), (q2.global_scale, b.global_scale)):
            assert torch.equal(u, v)
        del xd, q1, q2, a, b
        torch.cuda.empty_cache()
