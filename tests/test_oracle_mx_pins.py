"""Pins of the oracle's MXFP4 functions against what the pages and plain
mathematics fix, independently of the oracle's own code:
  - storage: 4.25 bits per element ("Melatih model dalam 4 bit", "Anatomi
    NVFP4": MXFP4 with 32-element blocks and an E8M0 power-of-two scale);
  - the scale is a power of two (E8M0: eight exponent bits, no mantissa --
    "NVFP4 Is a Scaling System", "Generic FP4, MXFP4, and NVFP4"), chosen so
    that the block maximum lands in [4, 8) (reading: OCP rule, floor(log2) - 2);
  - brute force: an exact-rational restatement on small tensors;
  - exact round trip of representable blocks; power-of-two invariance."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O
from nvfp4_bit_block_amax_b200 import inputs as G

F32 = np.float32
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


CODEBOOK = [Fraction(r[0]) for r in _golden_rows("e2m1_codebook.txt")]


def _bf16_f(bits):
    return np.asarray(bits, dtype=np.uint32).__lshift__(16).view(np.float32)


def _floor_log2(a: Fraction) -> int:
    k = 0
    while a >= 2:
        a /= 2
        k += 1
    while a < 1:
        a *= 2
        k -= 1
    return k


def _mirror_code(x: Fraction, e: int, negative: bool) -> int:
    """E2M1 nearest-even of x / 2^e with saturation, by exhaustive distance."""
    v = abs(x) / (Fraction(2) ** e)
    if v >= CODEBOOK[-1]:
        c = 7
    else:
        d = [abs(v - m) for m in CODEBOOK]
        best = min(d)
        cands = [i for i in range(8) if d[i] == best]
        c = [i for i in cands if i % 2 == 0][0] if len(cands) > 1 else cands[0]
    return c | (8 if negative else 0)


def _mirror_mx(bits: np.ndarray):
    rows, cols = bits.shape
    f = _bf16_f(bits)
    codes = np.zeros((rows, cols), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    for r in range(rows):
        for b in range(cols // 32):
            blk = [Fraction(float(v)) for v in f[r, 32 * b:32 * b + 32]]
            amax = max(abs(v) for v in blk)
            e = -127 if amax == 0 else max(-127, min(127, _floor_log2(amax) - 2))
            scales[r, b] = e + 127
            for j in range(32):
                codes[r, 32 * b + j] = _mirror_code(blk[j], e, bool(np.signbit(f[r, 32 * b + j])))
    return codes, scales


def _unpack(codes):
    lo, hi = codes & 0xF, codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def test_storage_is_4_25_bits_per_element():
    g = {r[0]: float(r[1]) for r in _golden_rows("storage_bits.txt")}
    for rows, cols in [(8, 64), (64, 1024)]:
        codes, scales = O.mx_quantize(G.make_tensor(rows, cols, 11))
        assert 8 * (codes.nbytes + scales.nbytes) / (rows * cols) == g["bits_per_elem_mxfp4"]


def test_scale_exponent_is_floor_log2_minus_2():
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.lognormal(0, 8, 2000).astype(F32), F32([1.0, 2.0, 4.0, 6.0, 7.999, 8.0, 0.5]),
                           F32([2.0 ** -126, 2.0 ** -149, 3e38])])
    for a in vals:
        k = _floor_log2(Fraction(float(a)))
        assert O.mx_scale_exp(float(a)) == max(-127, min(127, k - 2))
        assert math.frexp(float(a))[1] - 1 == k        # a second, independent floor(log2)
    assert O.mx_scale_exp(0.0) == -127
    for c in (0, 1, 127, 200, 254):
        assert O.e8m0_value(c) == 2.0 ** (c - 127)


@pytest.mark.parametrize("dist", ["normal", "lognormal_signed", "outliers"])
def test_brute_force_small_tensors(dist):
    kw = {"outlier_frac": 0.01, "outlier_mode": "set", "outlier_value": 1e4} if dist == "outliers" else {}
    x = G.make_tensor(4, 128, 21, dist="normal" if dist == "outliers" else dist, **kw)
    codes, scales = O.mx_quantize(x)
    mc, ms = _mirror_mx(x)
    assert np.array_equal(scales, ms)
    assert np.array_equal(_unpack(codes), mc)


def test_edge_blocks_zero_subnormal_huge():
    x = np.zeros((3, 64), dtype=np.uint16)
    x[1, :32] = 0x0001                 # smallest bf16 subnormal
    x[1, 32:] = 0x8001
    x[2, :32] = 0x7F7F                 # largest finite bf16
    x[2, 32] = 0x3F80                  # 1.0 next to a block of zeros
    codes, scales = O.mx_quantize(x)
    mc, ms = _mirror_mx(x)
    assert np.array_equal(scales, ms) and np.array_equal(_unpack(codes), mc)
    assert scales[0, 0] == 0 and (_unpack(codes)[0] == 0).all()      # zero block: code 0, scale 2^-127
    assert (_unpack(codes)[1, 32:] == 8).all()                       # tiny negatives keep the sign


def test_block_max_lands_in_4_to_6():
    x = G.make_tensor(16, 256, 31, dist="lognormal_signed", scale=2.0)
    codes, scales = O.mx_quantize(x)
    c = _unpack(codes)
    f = np.abs(_bf16_f(x))
    for r in range(16):
        for b in range(8):
            j = int(np.argmax(f[r, 32 * b:32 * b + 32]))
            assert c[r, 32 * b + j] & 7 in (6, 7)          # 4 or 6 (saturated from [7, 8))
            assert (c[r, 32 * b:32 * b + 32] & 7).max() == c[r, 32 * b + j] & 7


def test_representable_blocks_round_trip():
    rng = np.random.default_rng(9)
    for e in (-20, -2, 0, 5, 60):
        book = np.array([float(m) for m in CODEBOOK])
        vals = book[rng.integers(0, 8, (2, 64))]
        vals[:, 0] = 6.0
        vals[:, 32] = 4.0                               # each block's max in [4, 8)
        vals *= rng.choice([-1.0, 1.0], vals.shape) * 2.0 ** e
        bits = (vals.astype(F32).view(np.uint32) >> 16).astype(np.uint16)
        codes, scales = O.mx_quantize(bits)
        assert (scales == e + 127).all()
        assert np.array_equal(O.mx_dequantize(codes, scales, 2, 64), vals.astype(F32))


def test_power_of_two_invariance():
    x = G.make_tensor(8, 128, 41)
    f = _bf16_f(x)
    codes, scales = O.mx_quantize(x)
    for k in (-7, 3, 20):
        y = (f * F32(2.0 ** k)).view(np.uint32) >> 16
        c2, s2 = O.mx_quantize(y.astype(np.uint16))
        assert np.array_equal(c2, codes) and np.array_equal(s2.astype(int), scales.astype(int) + k)
