"""Pins for the oracle's larger-order random Hadamard transforms (32, 64 and
128 points), each against something other than the oracle itself: the
Sylvester matrix written from its closed form, exact rational arithmetic for
the normalisation, the Philox known-answer-pinned generator for the signs,
integer arithmetic for exact cases, and an independent restatement of the
quantize path.

Sources: "MXFP4 和 NVFP4 的区别", "构造 Hadamard 矩阵的方法" (Sylvester
recursion for any power-of-two order) and "为什么不用 Conference 矩阵,而用
Hadamard" (fast transform by butterflies); "随机 Hadamard 变换" (random sign
diagonal, orthogonal rotation before quantization).
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from nvfp4_bit_block_amax_b200 import inputs as G
from oracle import oracle as O
from tests.test_oracle_pins import _mirror_e2m1_rne, _mirror_e2m1_sr, _mirror_e4m3, bf16, mirror_quantize_1d

F32 = np.float32
ORDERS = (16, 32, 64, 128)


def sylvester_closed_form(n):
    """H[i][j] = (-1)^popcount(i & j) (natural-order Sylvester matrix)."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


@pytest.mark.parametrize("n", ORDERS)
def test_norm_is_rn_of_inverse_sqrt(n):
    c = O.rht_norm(n)
    k = n.bit_length() - 1
    if k % 2 == 0:
        assert c == F32(2.0 ** (-k // 2))          # exact power of two
    else:
        # |c - 1/sqrt(n)| < half an ulp of c  <=>  (c - u/2)^2 < 1/n < (c + u/2)^2
        cf = Fraction(float(c))
        half = Fraction(float(np.spacing(c))) / 2
        assert (cf - half) ** 2 < Fraction(1, n) < (cf + half) ** 2


@pytest.mark.parametrize("n", ORDERS)
def test_butterflies_are_sylvester_matrix(n):
    ones = np.ones(n, dtype=F32)
    c = O.rht_norm(n)
    cols = np.stack([O.rht_n(np.eye(n, dtype=F32)[j], ones) for j in range(n)], axis=1)
    # each column of the transform of a unit vector is exactly +-c
    assert np.array_equal(cols, (sylvester_closed_form(n) * np.float64(c)).astype(F32))
    h = sylvester_closed_form(n)
    assert np.array_equal(h @ h.T, n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("n", ORDERS)
def test_sign_vector_bits(n):
    seed = 0x1234_5678_9ABC
    d = O.rht_signs_n(seed, n)
    words = O.philox4x32_10([0, 0, 1, 0], [seed & 0xFFFFFFFF, seed >> 32])
    for j in range(n):
        assert (d[j] < 0) == bool((int(words[j // 32]) >> (j % 32)) & 1)
    # the 16-point transform's signs are the first 16 of every order
    assert np.array_equal(d[:16], O.rht_signs(seed))


@pytest.mark.parametrize("n", ORDERS)
def test_orthogonal_and_within_rounding_of_exact(n):
    d = O.rht_signs_n(91, n)
    q = sylvester_closed_form(n) * d[None, :].astype(np.float64) / np.sqrt(n)   # exact-rotation reference
    assert np.allclose(q.T @ q, np.eye(n), rtol=0, atol=1e-13)
    k = n.bit_length() - 1
    c = float(O.rht_norm(n))
    rng = np.random.default_rng(n)
    for _ in range(40):
        x = rng.standard_normal(n).astype(F32)
        y = O.rht_n(x, d).astype(np.float64)
        ref = q @ x.astype(np.float64)
        # k rounded butterfly levels, the rounded factor and the final multiply
        bound = (k + 3) * 2.0 ** -24 * c * np.abs(x).sum()
        assert np.all(np.abs(y - ref) <= bound)
        assert np.allclose(q.T @ y, x, rtol=0, atol=(k + 4) * 2.0 ** -24 * np.abs(x).sum())


@pytest.mark.parametrize("n", ORDERS)
def test_exact_on_small_integers(n):
    d = O.rht_signs_n(7, n)
    h = sylvester_closed_form(n)
    c = O.rht_norm(n)
    rng = np.random.default_rng(100 + n)
    for _ in range(50):
        x = rng.integers(-64, 65, n).astype(F32)
        y = O.rht_n(x, d)
        s = h @ (d.astype(np.int64) * x.astype(np.int64))      # exact integer butterflies
        assert np.array_equal(y, s.astype(F32) * c)             # then one binary32 multiply


def test_order_16_is_the_16_point_transform():
    d = O.rht_signs(5)
    rng = np.random.default_rng(1)
    for _ in range(20):
        x = rng.standard_normal(16).astype(F32)
        assert np.array_equal(O.rht_n(x, d), O.rht16(x, d))


def rotated_q_exact(x_bits, n, rht_seed, transpose):
    """Q (x or x^T) rotated, for small-integer inputs: the butterfly sums are
    exact integers, so each rotated value is one binary32 multiply RN(c * s)."""
    xf = G.bf16_bits_to_f32(x_bits)
    q = (xf.T if transpose else xf).astype(F32)
    qr, qc = q.shape
    d = O.rht_signs_n(rht_seed, n).astype(np.int64)
    h = sylvester_closed_form(n)
    c = O.rht_norm(n)
    y = np.empty_like(q)
    for r in range(qr):
        for c0 in range(0, qc, n):
            y[r, c0:c0 + n] = (h @ (d * q[r, c0:c0 + n].astype(np.int64))).astype(F32) * c
    return y


@pytest.mark.parametrize("n", (32, 64, 128))
@pytest.mark.parametrize("transpose", (False, True))
@pytest.mark.parametrize("rounding", (0, 1))
def test_quantize_with_larger_order_matches_restatement(n, transpose, rounding):
    rng = np.random.default_rng(n + 7 * transpose + 3 * rounding)
    rows, cols = (2 * n, 48) if transpose else (5, 2 * n)
    x = bf16(rng.integers(-64, 65, size=(rows, cols)).astype(F32))
    got = O.quantize_1d(x, transpose=transpose, rht=True, rht_seed=21, rounding=rounding, sr_seed=22, rht_order=n)
    exp = _mirror_from_rotated(rotated_q_exact(x, n, 21, transpose), rounding, 22)
    assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1]) and got[2] == exp[2]


def _mirror_from_rotated(q, rounding, sr_seed):
    """mirror_quantize_1d's steps after the rotation, on a float32 Q."""
    qr, qc = q.shape
    amax = F32(np.abs(q).max())
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
                    codes[r, 16 * b + j] = _mirror_e2m1_sr(v, O.sr_bits(sr_seed, r * qc + 16 * b + j))
                else:
                    codes[r, 16 * b + j] = _mirror_e2m1_rne(v)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, scales, sg


def test_restatement_helper_agrees_with_16_point_mirror():
    """The float32-input restatement reproduces the pinned 16-point mirror."""
    rng = np.random.default_rng(3)
    x = bf16(rng.integers(-64, 65, size=(32, 24)).astype(F32))
    a = _mirror_from_rotated(rotated_q_exact(x, 16, 5, True), 1, 6)
    b = mirror_quantize_1d(x, transpose=True, rht_seed=5, rounding=1, sr_seed=6)
    assert all(np.array_equal(u, v) for u, v in zip(a[:2], b[:2])) and a[2] == b[2]


@pytest.mark.parametrize("n", (32, 64, 128))
def test_amax_of_rotated_tensor(n):
    x = G.make_tensor(3 * n, 32, seed=n, dist="normal", scale=1.0, outlier_frac=0.01, outlier_mode="mul",
                      outlier_value=50.0)
    y = rotated_q_float(x, n, 44)
    assert O.amax(x, transpose=True, rht=True, rht_seed=44, rht_order=n) == F32(np.abs(y).max())


def rotated_q_float(x_bits, n, rht_seed):
    """Q = x^T rotated by sequential butterflies written out in numpy float32
    (the same rounded operations, in the order h = 1, 2, ..., n/2)."""
    q = G.bf16_bits_to_f32(x_bits).T.astype(F32)
    d = O.rht_signs_n(rht_seed, n)
    c = O.rht_norm(n)
    out = np.empty_like(q)
    for r in range(q.shape[0]):
        for c0 in range(0, q.shape[1], n):
            t = (q[r, c0:c0 + n] * d).astype(F32)
            h = 1
            while h < n:
                idx = np.array([i for i in range(n) if not i & h])
                a, b = t[idx].copy(), t[idx + h].copy()
                t[idx] = a + b
                t[idx + h] = a - b
                h <<= 1
            out[r, c0:c0 + n] = t * c
    return out


def test_bad_order_rejected():
    x = np.zeros((4, 64), dtype=np.uint16)
    with pytest.raises(ValueError):
        O.quantize_1d(x, rht=True, rht_order=48)
    with pytest.raises(ValueError):
        O.quantize_1d(np.zeros((4, 96), dtype=np.uint16), rht=True, rht_order=64)   # 96 % 64 != 0


@pytest.mark.parametrize("n", ORDERS)
def test_rounding_order_is_h_ascending(n):
    """On non-integer inputs the rounded sums depend on the butterfly order:
    the oracle equals numpy float32 butterflies h = 1, 2, ..., n/2 bit for bit
    (and differs from the reversed order somewhere)."""
    rng = np.random.default_rng(500 + n)
    d = O.rht_signs_n(8, n)
    c = O.rht_norm(n)
    differs = False
    for _ in range(30):
        x = rng.standard_normal(n).astype(F32)
        fwd = _butterflies(x * d, n, reverse=False) * c
        rev = _butterflies(x * d, n, reverse=True) * c
        assert np.array_equal(O.rht_n(x, d), fwd)
        differs |= not np.array_equal(fwd, rev)
    assert differs


def _butterflies(t, n, reverse):
    t = t.astype(F32).copy()
    hs = [1 << s for s in range(n.bit_length() - 1)]
    for h in (hs[::-1] if reverse else hs):
        idx = np.array([i for i in range(n) if not i & h])
        a, b = t[idx].copy(), t[idx + h].copy()
        t[idx] = a + b
        t[idx + h] = a - b
    return t
