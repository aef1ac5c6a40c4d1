"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Every test here runs on the CPU and compares the oracle with something other
than itself: values the pages print (fixtures under tests/golden, each with its
citation), an independent library (ml_dtypes' E2M1 / E4M3 conversions), closed
forms, invariants, exact rational arithmetic, or an independent re-statement
of the pipeline on tiny inputs.
"""
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from oracle import oracle as O
from nvfp4_bit_block_amax_b200 import inputs as G

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


CODEBOOK = [Fraction(r[0]) for r in _golden_rows("e2m1_codebook.txt")]  # magnitudes, code order


def bf16(vals):
    """Exact bf16 bit patterns of values that are bf16-representable."""
    f = np.asarray(vals, dtype=np.float32)
    bits = G._to_bf16_bits(f)
    assert (G.bf16_bits_to_f32(bits) == f).all(), "value not representable in bf16"
    return bits


def all_bf16_finite():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = G.bf16_bits_to_f32(h)
    return f[np.isfinite(f)]


# ------------------------------------------------------------------ format --
def test_e2m1_codebook_matches_pages():
    vals = [O.e2m1_value(c) for c in range(16)]
    assert [Fraction(v) for v in vals[:8]] == CODEBOOK
    assert vals[8:] == [-v for v in vals[:8]]
    assert np.signbit(vals[8])  # code 8 is negative zero
    # an independent decoder agrees on all 16 codes
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(lib, np.array(vals)) and np.array_equal(np.signbit(lib), np.signbit(vals))


def test_format_constants_from_pages():
    c = {r[0]: float(r[1]) for r in _golden_rows("format_constants.txt")}
    assert O.e2m1_value(7) == c["e2m1_max"]
    assert O.e4m3_value(0x7E) == c["e4m3_max"]
    assert max(O.e4m3_value(i) for i in range(0x7F)) == c["e4m3_max"]
    # s_global = amax / (448 * 6): an amax of 2688 gives exactly 1
    assert O.global_scale(2688.0) == 1.0
    assert O.global_scale(c["e4m3_max"] * c["e2m1_max"] * 0.25) == 0.25


def test_e4m3_decoder_matches_library():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ours = np.array([O.e4m3_value(i) for i in range(256)])
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2  # 0x7F, 0xFF
    assert np.array_equal(lib[~nan], ours[~nan])


def test_worked_example_reconstruction():
    """payload 4 x s_block {1.0, 1.5} x s_global 0.25 = {1.0, 1.5}."""
    for payload, s_block, s_global, expected in _golden_rows("worked_example.txt"):
        code = [c for c in range(8) if O.e2m1_value(c) == float(payload)][0]
        s_code = O.e4m3_rne_satfinite(float(s_block))
        assert O.e4m3_value(s_code) == float(s_block)
        # a one-row tensor of two blocks; the element of interest is at column 0
        codes = np.zeros((1, 16), dtype=np.uint8)
        codes[0, 0] = code
        scales = np.array([[s_code, s_code]], dtype=np.uint8)
        out = O.dequantize(codes, scales, 0, float(s_global), 1, 32)
        assert out[0, 0] == float(expected)
        assert (out[0, 1:] == 0).all()


def test_storage_bits_per_element():
    g = {r[0]: float(r[1]) for r in _golden_rows("storage_bits.txt")}
    assert 16 * 4 + 8 == g["block_bits_1d"]
    for rows, cols in [(16, 64), (64, 256), (256, 1024)]:
        n = rows * cols
        x = G.make_tensor(rows, cols, 7)
        codes, scales, _ = O.quantize_1d(x)
        bits = 8 * (codes.nbytes + scales.nbytes + 4) / n
        assert bits == pytest.approx(g["bits_per_elem_1d"] + 32 / n, abs=0)
        cr, _, sc, _ = O.quantize_2d(x, columnwise=False)
        bits2 = 8 * (cr.nbytes + sc.nbytes + 4) / n
        assert bits2 == 4 + 8 / 256 + 32 / n
        assert abs(bits2 - 32 / n - g["bits_per_elem_2d_approx"]) < 0.005
    # MXFP4 for comparison: 32 payloads of 4 bits share one 8-bit scale
    assert (32 * 4 + 8) / 32 == g["bits_per_elem_mxfp4"]


# ------------------------------------------------------------ E2M1 rounding --
def _argmin_rne(a: Fraction) -> int:
    """Nearest codebook magnitude, ties to the code with mantissa bit 0."""
    if a >= CODEBOOK[-1]:
        return 7
    d = [abs(a - m) for m in CODEBOOK]
    best = min(d)
    cands = [c for c in range(8) if d[c] == best]
    return [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]


def test_e2m1_rne_every_bf16_value():
    f = all_bf16_finite()
    ours = O.e2m1_rne_array(f)
    lib = f.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    assert np.array_equal(ours, lib)
    # exact-rational argmin on every distinct magnitude below 8
    mags = np.unique(np.abs(f[np.abs(f) < 8]))
    exp = np.array([_argmin_rne(Fraction(float(m))) for m in mags], dtype=np.uint8)
    assert np.array_equal(O.e2m1_rne_array(mags), exp)


def test_e2m1_rne_ties_and_neighbours():
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for t, code in ties.items():
        assert O.e2m1_rne(t) == code
        assert O.e2m1_rne(-t) == code | 8
        up = np.nextafter(F32(t), F32(10))
        dn = np.nextafter(F32(t), F32(0))
        assert O.e2m1_rne(up) == _argmin_rne(Fraction(float(up)))
        assert O.e2m1_rne(dn) == _argmin_rne(Fraction(float(dn)))
        assert O.e2m1_rne(up) == O.e2m1_rne(dn) + 1 or (t in (0.25,) and O.e2m1_rne(up) == 1)
    assert O.e2m1_rne(6.0) == 7 and O.e2m1_rne(1e30) == 7 and O.e2m1_rne(np.inf) == 7
    assert O.e2m1_rne(-0.0) == 8 and O.e2m1_rne(-1e-30) == 8 and O.e2m1_rne(0.0) == 0


def test_e2m1_sr_never_moves_representable_values():
    for c in range(16):
        v = O.e2m1_value(c)
        for u in (0, 1, 12345, 65535):
            assert O.e2m1_sr(v, u) == c or (v == 0 and O.e2m1_sr(v, u) in (0, 8) and
                                            O.e2m1_sr(v, u) == c)
    assert O.e2m1_sr(7.0, 0) == 7 and O.e2m1_sr(-100.0, 65535) == 15


@pytest.mark.parametrize("v", [0.1, 0.3, 0.7, 1.2, 2.6, 3.3, 4.9])
def test_e2m1_sr_unbiased(v):
    """E[SR(v)] = v within 3 standard errors over 10^6 draws ("随机舍入": the
    expectation of the quantized value equals the original value)."""
    n = 1_000_000
    for sign in (1, -1):
        vv = F32(sign * v)
        codes = O.e2m1_sr_array(np.full(n, vv, dtype=F32), seed=20260 + int(v * 10), first_index=0)
        vals = np.array([O.e2m1_value(c) for c in range(16)])[codes]
        a = Fraction(float(abs(vv)))
        lo = max(m for m in CODEBOOK if m <= a)
        hi = min(m for m in CODEBOOK if m > a)
        gap = float(hi - lo)
        p = float((a - lo) / (hi - lo))
        se = gap * np.sqrt(p * (1 - p) / n)
        assert abs(vals.mean() - float(vv)) <= 3 * se
        # exact up-rate of the 16-bit carry rule: floor(p * 2^16) / 2^16
        rate = np.mean(np.abs(vals) == float(hi))
        exact = np.floor(p * 65536) / 65536
        assert abs(rate - exact) <= 3 * np.sqrt(exact * (1 - exact) / n)
        assert set(np.unique(np.abs(vals))) <= {float(lo), float(hi)}


def test_sr_up_rule_is_carry_of_16_bits():
    # v = 0.3 as binary32 (0.30000001...) lies in [0, 0.5): p = 2v, p * 65536 =
    # 39321.60..., f = 39321; up iff f + u >= 65536, i.e. u >= 26215
    f = int(np.floor(float(Fraction(float(F32(0.3))) / Fraction(1, 2)) * 65536))
    assert f == 39321
    assert O.e2m1_sr(0.3, 65536 - f - 1) == 0 and O.e2m1_sr(0.3, 65536 - f) == 1
    assert O.e2m1_sr(-0.3, 65535) == 9 and O.e2m1_sr(-0.3, 0) == 8
    # p just above 0: f = 0 and no u rounds up; p = 1/2^16 exactly: only u = 65535
    tiny = F32(2.0) + F32(2.0 ** -16)          # in [2, 3): p = 2^-16
    assert O.e2m1_sr(tiny, 65535) == 5 and O.e2m1_sr(tiny, 65534) == 4
    below = F32(np.nextafter(F32(2.0 ** -16) * F32(0.5), F32(0)))   # p just under 2^-16 in [0, 0.5)
    assert O.e2m1_sr(below, 65535) == 0


# ------------------------------------------------------------ E4M3 rounding --
def test_e4m3_every_bf16_value_in_range():
    f = all_bf16_finite()
    f = f[(f >= 0) & (f <= 464) & ~np.signbit(f)]    # block amaxes are never -0
    ours = O.e4m3_array(f)
    lib = f.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, lib)


def test_e4m3_dense_sweep_and_saturation():
    rng = np.random.default_rng(3)
    # dense float32 sweep around every code midpoint, plus random values
    vals = np.array([O.e4m3_value(i) for i in range(0x7F)], dtype=np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(F32)
    sweep = np.concatenate([mids, np.nextafter(mids, F32(0)), np.nextafter(mids, F32(1e9)),
                            rng.uniform(0, 448, 100000).astype(F32),
                            (2.0 ** rng.uniform(-12, -6, 20000)).astype(F32)])
    ours = O.e4m3_array(sweep)
    lib = sweep.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, lib)
    # exact tie behaviour below the subnormal range: 2^-10 ties to 0, above it rounds up
    assert O.e4m3_rne_satfinite(2.0 ** -10) == 0
    assert O.e4m3_rne_satfinite(float(np.nextafter(F32(2.0 ** -10), F32(1)))) == 1
    # saturation (FN variant, max 448): everything above 448 maps to 448
    for s in (448.0, 449.0, 464.0, 465.0, 1e6, 3e38, float("inf")):
        assert O.e4m3_rne_satfinite(s) == 0x7E


# -------------------------------------------------------------------- Philox --
def test_philox_known_answers():
    for r in _golden_rows("philox4x32_10_kat.txt"):
        h = [int(t, 16) for t in r]
        assert O.philox4x32_10(h[0:4], h[4:6]).tolist() == h[6:10]


def test_sr_bits_layout():
    seed = 0x1234_5678_9ABC_DEF0
    out = O.philox4x32_10([5, 0, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
    for j in range(8):
        w = int(out[j // 2])
        exp = (w & 0xFFFF) if j % 2 == 0 else (w >> 16)
        assert O.sr_bits(seed, 40 + j) == exp
    big = (1 << 35) * 8 + 3
    out = O.philox4x32_10([0, 1 << 3, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
    assert O.sr_bits(seed, big) == int(out[1]) >> 16


def test_philox_uniformity():
    u = np.array([O.sr_bits(99, i) for i in range(80000)])
    hist = np.bincount(u >> 12, minlength=16)
    chi2 = (((hist - 5000.0) ** 2) / 5000.0).sum()
    assert chi2 < 45  # 15 dof, p ~ 1e-4


# ----------------------------------------------------------------------- RHT --
def sylvester(n):
    """Sylvester recursion ("构造 Hadamard 矩阵的方法": four H_n blocks, the
    lower-right one negated)."""
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def test_rht_butterflies_are_sylvester_hadamard():
    ones = np.ones(16, dtype=F32)
    cols = np.stack([O.rht16(np.eye(16, dtype=F32)[j], ones) for j in range(16)], axis=1)
    h = (cols * 4).astype(np.int64)
    assert np.array_equal(h, sylvester(16))
    assert np.array_equal(h @ h.T, 16 * np.eye(16, dtype=np.int64))   # H H^T = 16 I


def test_rht_sign_vector_and_orthogonality():
    d = O.rht_signs(77)
    assert set(np.unique(d)) <= {-1.0, 1.0}
    w = int(O.philox4x32_10([0, 0, 1, 0], [77, 0])[0])
    assert all((d[j] < 0) == bool((w >> j) & 1) for j in range(16))
    q = sylvester(16) * d[None, :] / 4.0        # (1/4) H D
    assert np.allclose(q.T @ q, np.eye(16), atol=0, rtol=0)
    rng = np.random.default_rng(5)
    for _ in range(50):
        x = rng.standard_normal(16).astype(F32)
        y = O.rht16(x, d).astype(np.float64)
        ref = q @ x.astype(np.float64)
        # four rounded additions of magnitudes <= sum|x|: error bound 4 * 2^-24 * sum|x| / 4 * 4
        assert np.all(np.abs(y - ref) <= 4 * 2.0 ** -24 * np.abs(x).sum())
        # the inverse recovers x (orthogonal transform)
        assert np.allclose(q.T @ y, x, rtol=0, atol=1e-6 * np.abs(x).sum())


def test_rht_exact_on_small_integers():
    d = O.rht_signs(3)
    rng = np.random.default_rng(6)
    for _ in range(100):
        x = rng.integers(-64, 65, 16).astype(F32)
        y = O.rht16(x, d)
        exact = (sylvester(16) @ (d.astype(np.int64) * x.astype(np.int64))) / 4.0
        assert np.array_equal(y.astype(np.float64), exact)


# ---------------------------------------------------- independent re-statement --
def _mirror_e4m3(sf):
    sf = F32(min(sf, F32(448.0)))
    return int(np.array([sf], dtype=F32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0])


def _mirror_e2m1_rne(v):
    return int(np.array([v], dtype=F32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)[0])


def _mirror_e2m1_sr(v, u):
    sign = 8 if np.signbit(v) else 0
    a = Fraction(float(abs(v))) if np.isfinite(v) else Fraction(10)
    if a >= CODEBOOK[-1]:
        return sign | 7
    lo = max(i for i in range(8) if CODEBOOK[i] <= a)
    if CODEBOOK[lo] == a:
        return sign | lo
    p = (a - CODEBOOK[lo]) / (CODEBOOK[lo + 1] - CODEBOOK[lo])
    f = (p * 65536).numerator // (p * 65536).denominator  # floor
    return sign | (lo + 1 if f + u >= 65536 else lo)


def mirror_quantize_1d(x_bits, transpose=False, rht_seed=None, rounding=0, sr_seed=0):
    """Independent statement of the 1D path: Q = x or x^T; optional exact RHT
    (small-integer inputs only); amax -> s_global -> per-block E4M3 scale ->
    per-element E2M1 code; low nibble = even element."""
    xf = G.bf16_bits_to_f32(x_bits)
    q = (xf.T if transpose else xf).astype(F32)
    qr, qc = q.shape
    if rht_seed is not None:
        d = O.rht_signs(rht_seed).astype(np.int64)
        h = sylvester(16)
        y = np.empty_like(q)
        for r in range(qr):
            for c0 in range(0, qc, 16):
                chunk = q[r, c0:c0 + 16].astype(np.int64)
                y[r, c0:c0 + 16] = (h @ (d * chunk)) / 4.0
        q = y
    amax = F32(np.abs(q).max()) if q.size else F32(0)
    sg = F32(amax / F32(2688.0))
    t = F32(F32(6.0) * sg)
    codes = np.zeros((qr, qc), dtype=np.uint8)
    scales = np.zeros((qr, qc // 16), dtype=np.uint8)
    for r in range(qr):
        for b in range(qc // 16):
            blk = q[r, 16 * b:16 * b + 16]
            bmax = F32(np.abs(blk).max())
            sf = F32(0.0) if t == 0 else F32(bmax / t)
            sc = _mirror_e4m3(sf)
            scales[r, b] = sc
            s_dec = F32(np.array([sc], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(F32)[0])
            for j in range(16):
                yv = blk[j]
                if s_dec == 0 or yv == 0:
                    codes[r, 16 * b + j] = 8 if np.signbit(yv) else 0
                    continue
                prod = F32(s_dec * sg)
                rr = F32(np.inf) if prod == 0 else F32(F32(1.0) / prod)
                v = F32(yv * rr)
                if rounding:
                    u = O.sr_bits(sr_seed, r * qc + 16 * b + j)
                    codes[r, 16 * b + j] = _mirror_e2m1_sr(v, u)
                else:
                    codes[r, 16 * b + j] = _mirror_e2m1_rne(v)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, scales, sg


@pytest.mark.parametrize("shape", [(1, 16), (16, 16), (2, 32), (3, 48)])
@pytest.mark.parametrize("rounding", [0, 1])
def test_quantize_1d_matches_restatement(shape, rounding):
    x = G.make_tensor(*shape, seed=11 + shape[0], dist="normal", scale=3.0, outlier_frac=0.05,
                      outlier_mode="set", outlier_value=40.0)
    got = O.quantize_1d(x, rounding=rounding, sr_seed=9)
    exp = mirror_quantize_1d(x, rounding=rounding, sr_seed=9)
    assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1]) and got[2] == exp[2]


@pytest.mark.parametrize("rounding", [0, 1])
def test_quantize_transposed_rht_matches_restatement(rounding):
    rng = np.random.default_rng(12)
    x = bf16(rng.integers(-64, 65, size=(32, 24)).astype(F32))   # Q = x^T is 24 x 32
    got = O.quantize_1d(x, transpose=True, rht=True, rht_seed=5, rounding=rounding, sr_seed=6)
    exp = mirror_quantize_1d(x, transpose=True, rht_seed=5, rounding=rounding, sr_seed=6)
    assert got[0].shape == (24, 16) and got[1].shape == (24, 2)
    assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1]) and got[2] == exp[2]


def test_quantize_2d_matches_restatement():
    w = G.make_tensor(32, 48, seed=21, dist="normal", scale=0.02)
    cr, cc, sc, sg = O.quantize_2d(w)
    wf = G.bf16_bits_to_f32(w)
    assert sg == F32(F32(np.abs(wf).max()) / F32(2688.0))
    t = F32(F32(6.0) * sg)
    for tr in range(2):
        for tc in range(3):
            tile = wf[16 * tr:16 * tr + 16, 16 * tc:16 * tc + 16]
            exp_sc = _mirror_e4m3(F32(F32(np.abs(tile).max()) / t))
            assert sc[tr, tc] == exp_sc
            s_dec = F32(np.array([exp_sc], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(F32)[0])
            rr = F32(F32(1.0) / F32(s_dec * sg))
            for i in range(16):
                for j in range(16):
                    r, c = 16 * tr + i, 16 * tc + j
                    code = _mirror_e2m1_rne(F32(tile[i, j] * rr))
                    assert ((cr[r, c // 2] >> (4 * (c % 2))) & 0xF) == code
                    assert ((cc[c, r // 2] >> (4 * (r % 2))) & 0xF) == code


# ---------------------------------------------------------------- invariants --
def _random_codes_scales(rng, rows, cols, pow2_scales=False):
    n_blocks = rows * cols // 16
    codes = rng.integers(0, 16, size=(rows, cols)).astype(np.uint8)
    codes[:, ::16] = rng.choice([7, 15], size=(rows, cols // 16))      # every block holds +-6
    if pow2_scales:
        sc_vals = 2.0 ** rng.integers(-6, 8, size=n_blocks)
    else:
        normal_codes = np.arange(0x18, 0x7F)                           # normal E4M3 values >= 2^-6
        sc_vals = np.array([O.e4m3_value(c) for c in rng.choice(normal_codes, n_blocks)])
    sc_vals[rng.integers(0, n_blocks)] = 448.0
    return codes, sc_vals.reshape(rows, cols // 16)


@pytest.mark.parametrize("g_exp", [-10, 0, 5])
def test_exact_round_trip_of_representable_inputs(g_exp):
    rng = np.random.default_rng(40 + g_exp)
    rows, cols = 8, 64
    codes, scv = _random_codes_scales(rng, rows, cols)
    g = 2.0 ** g_exp
    vals = np.array([O.e2m1_value(c) for c in range(16)])[codes] * np.repeat(scv, 16, axis=1) * g
    x = bf16(vals)
    c_got, s_got, sg = O.quantize_1d(x)
    assert sg == g
    assert np.array_equal(s_got, np.array([[O.e4m3_rne_satfinite(v) for v in row] for row in scv]))
    unpacked = np.stack([c_got & 0xF, c_got >> 4], axis=-1).reshape(rows, cols)
    # zero codes keep the sign of the input zero; compare magnitudes and signs of nonzeros
    assert np.array_equal(unpacked & 7, codes & 7)
    nz = (codes & 7) != 0
    assert np.array_equal(unpacked[nz], codes[nz])
    deq = O.dequantize(c_got, s_got, 0, sg, rows, cols)
    assert np.array_equal(deq, vals.astype(F32))


def test_sr_round_trip_with_power_of_two_scales():
    rng = np.random.default_rng(50)
    rows, cols = 8, 64
    codes, scv = _random_codes_scales(rng, rows, cols, pow2_scales=True)
    vals = np.array([O.e2m1_value(c) for c in range(16)])[codes] * np.repeat(scv, 16, axis=1) * 2.0 ** -3
    x = bf16(vals)
    c_got, _, _ = O.quantize_1d(x, rounding=1, sr_seed=1234)
    unpacked = np.stack([c_got & 0xF, c_got >> 4], axis=-1).reshape(rows, cols)
    pow2_blocks = np.repeat(np.log2(scv) == np.round(np.log2(scv)), 16, axis=1)
    assert np.array_equal((unpacked & 7)[pow2_blocks], (codes & 7)[pow2_blocks])


def test_amax_block_gets_max_scale_and_six():
    for seed in range(5):
        x = G.make_tensor(16, 64, seed=60 + seed, dist="normal", scale=0.5)
        xf = G.bf16_bits_to_f32(x)
        codes, scales, sg = O.quantize_1d(x)
        r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
        assert scales[r, c // 16] == 0x7E
        code = (codes[r, c // 2] >> (4 * (c % 2))) & 0xF
        assert code == (15 if xf[r, c] < 0 else 7)
        assert scales.max() == 0x7E


@pytest.mark.parametrize("k", [-3, -1, 2, 4])
def test_power_of_two_scaling_invariance(k):
    x = G.make_tensor(16, 64, seed=70, dist="normal", scale=1.0, outlier_frac=0.02, outlier_mode="mul",
                      outlier_value=50.0)
    xs = bf16(G.bf16_bits_to_f32(x) * F32(2.0 ** k))
    for rounding in (0, 1):
        c0, s0, g0 = O.quantize_1d(x, rounding=rounding, sr_seed=3)
        c1, s1, g1 = O.quantize_1d(xs, rounding=rounding, sr_seed=3)
        assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and g1 == g0 * F32(2.0 ** k)


def test_2d_rowwise_equals_columnwise_transpose():
    """16x16 scaling makes rowwise and columnwise quantization numerically
    identical ("Empat pengaman": second safeguard)."""
    w = G.make_tensor(64, 48, seed=80, dist="normal", scale=0.015)
    cr, cc, sc, sg = O.quantize_2d(w)
    ur = np.stack([cr & 0xF, cr >> 4], axis=-1).reshape(64, 48)
    uc = np.stack([cc & 0xF, cc >> 4], axis=-1).reshape(48, 64)
    assert np.array_equal(ur, uc.T)
    # quantizing W^T in 2D gives the same codes as the columnwise copy, and transposed scales
    wt = np.ascontiguousarray(w.T)
    crt, cct, sct, sgt = O.quantize_2d(wt)
    assert np.array_equal(crt, cc) and np.array_equal(cct, cr) and np.array_equal(sct, sc.T) and sgt == sg


def test_zero_tensor_and_signed_zeros():
    x = bf16(np.zeros((2, 32), dtype=F32))
    x[0, 3] = 0x8000                     # -0.0
    codes, scales, sg = O.quantize_1d(x)
    assert sg == 0 and (scales == 0).all()
    assert (codes[0, 1] >> 4) == 8 and (codes & 0x77 == 0).all()


def test_tiny_negative_keeps_sign():
    vals = np.zeros((1, 16), dtype=F32)
    vals[0, 0] = 6.0
    vals[0, 1] = -2.0 ** -7
    codes, _, _ = O.quantize_1d(bf16(vals))
    assert (codes[0, 0] >> 4) == 8


def test_zero_block_scale_gives_signed_zeros():
    vals = np.zeros((1, 32), dtype=F32)
    vals[0, 0] = 448.0 * 6 * 2 ** 10      # huge amax: the second block's scale underflows to 0
    vals[0, 16] = 2.0 ** -10
    vals[0, 17] = -2.0 ** -10
    codes, scales, _ = O.quantize_1d(bf16(vals))
    assert scales[0, 1] == 0
    assert codes[0, 8] == 0x80            # +0 then -0


# ---------------------------------------------------------------- dequantize --
def test_dequantize_matches_exact_product():
    x = G.make_tensor(32, 64, seed=90, dist="normal", scale=2.0)
    codes, scales, sg = O.quantize_1d(x)
    deq = O.dequantize(codes, scales, 0, sg, 32, 64)
    exact = O.dequantize_f64(codes, scales, 0, sg, 32, 64)
    assert np.array_equal(deq, exact.astype(F32))
    w = G.make_tensor(32, 64, seed=91, dist="normal", scale=0.02)
    cr, _, sc, sgw = O.quantize_2d(w, columnwise=False)
    assert np.array_equal(O.dequantize(cr, sc, 1, sgw, 32, 64), O.dequantize_f64(cr, sc, 1, sgw, 32, 64).astype(F32))


def test_quantization_error_is_bounded():
    """Each reconstructed element is within half a grid step of the input
    (RNE) -- the grid step at |v| is at most 2 (between 4 and 6) in units of
    s_dec * s_global, below 6 * s_dec * s_global overall."""
    x = G.make_tensor(16, 256, seed=92, dist="normal", scale=1.0)
    codes, scales, sg = O.quantize_1d(x)
    deq = O.dequantize_f64(codes, scales, 0, sg, 16, 256)
    xf = G.bf16_bits_to_f32(x).astype(np.float64)
    unit = np.repeat(np.array([[O.e4m3_value(s) for s in row] for row in scales]), 16, axis=1) * float(sg)
    assert np.all(np.abs(deq - xf) <= 1.0 * unit * (1 + 1e-6))


# ---------------------------------------------------------------- GEMM reference --
def test_gemm_reference_exact_small():
    rng = np.random.default_rng(100)
    a = rng.integers(-3, 4, size=(3, 5)).astype(np.float64) * 0.5
    b = rng.integers(-3, 4, size=(4, 5)).astype(np.float64) * 0.25
    c, s = O.gemm_reference(a, b)
    for i in range(3):
        for j in range(4):
            exact = sum(Fraction(a[i, k]) * Fraction(b[j, k]) for k in range(5))
            bound = sum(abs(Fraction(a[i, k]) * Fraction(b[j, k])) for k in range(5))
            assert Fraction(c[i, j]) == exact and Fraction(s[i, j]) == bound
    assert c.shape == (3, 4)   # C = A B^T: rows of A by rows of B


def test_gemm_reference_over_quantized_operands():
    a, w = G.tiny_linear(32, 48, 64)
    ca, sa, ga = O.quantize_1d(a)
    cw, _, sw, gw = O.quantize_2d(w, columnwise=False)
    ah = O.dequantize_f64(ca, sa, 0, ga, 32, 64)
    wh = O.dequantize_f64(cw, sw, 1, gw, 48, 64)
    c, s = O.gemm_reference(ah, wh)
    # the quantized product approximates the bf16 product within the quantization error
    af, wf = G.bf16_bits_to_f32(a).astype(np.float64), G.bf16_bits_to_f32(w).astype(np.float64)
    assert np.abs(c - af @ wf.T).max() <= 0.5 * (np.abs(af) @ np.abs(wf).T).max()
    assert (s >= np.abs(c)).all()
