"""Seeded synthetic inputs for the NVFP4 path (shared by tests, bench and smoke).

This module holds no quantization arithmetic: it only draws numbers with
numpy's PCG64 generator and rounds them to bf16 (round to nearest even), so
that the CUDA path and the CPU oracle see bit-identical inputs.  Tensors are
returned as uint16 bf16 bit patterns, row-major.

Workload shapes follow the MLP linear layer of "Melatih model dalam 4 bit:
pengaman numerik di balik NVFP4" ("Empat pengaman": the three MLP GEMMs --
fprop, dgrad, wgrad -- are the ones quantized).  Value distributions are the
stated synthetic recipes (normal activations with sparse outliers, small
normal weights, Laplace gradients with sparse large outliers).
"""
from __future__ import annotations

import numpy as np

_CHUNK = 1 << 24  # elements drawn per chunk (bounds host memory on large tensors)


def _to_bf16_bits(f32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _draw(rng: np.random.Generator, n: int, dist: str, scale: float) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(n, dtype=np.float32) * np.float32(scale)
    if dist == "laplace":
        # inverse-CDF draw in float32: u uniform on [0,1), x = -b sign(u-1/2) log(1 - 2|u-1/2|)
        # (the argument of the log is kept >= 2^-24 so that u = 0 stays finite)
        h = rng.random(n, dtype=np.float32) - np.float32(0.5)
        mag = -np.log(np.maximum(np.float32(1.0) - np.float32(2.0) * np.abs(h), np.float32(2.0 ** -24)))
        return np.copysign(mag, h) * np.float32(scale)
    if dist == "lognormal_signed":
        mag = rng.lognormal(0.0, scale, n).astype(np.float32)
        sign = np.where(rng.integers(0, 2, n, dtype=np.uint8) == 1, np.float32(-1.0), np.float32(1.0))
        return mag * sign
    raise ValueError(f"unknown distribution {dist!r}")


def make_tensor(rows: int, cols: int, seed: int, dist: str = "normal", scale: float = 1.0,
                outlier_frac: float = 0.0, outlier_mode: str = "none", outlier_value: float = 0.0) -> np.ndarray:
    """Draw a [rows x cols] bf16 tensor.

    dist: "normal" (N(0, scale^2)), "laplace" (Laplace(0, scale)),
          "lognormal_signed" (exp(N(0, scale^2)) with a random sign).
    outliers: round(outlier_frac * n) distinct positions, chosen without
    replacement; mode "set" replaces them by +-outlier_value (random sign),
    mode "mul" multiplies them by outlier_value.
    """
    n = rows * cols
    rng = np.random.Generator(np.random.PCG64(seed))
    out = np.empty(n, dtype=np.uint16)
    vals = None
    if outlier_mode != "none" and outlier_frac > 0:
        k = int(round(outlier_frac * n))
    else:
        k = 0
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        f = _draw(rng, e - s, dist, scale)
        out[s:e] = _to_bf16_bits(f)
        del f
    if k:
        idx = rng.choice(n, size=k, replace=False)
        base = bf16_bits_to_f32(out[idx])
        if outlier_mode == "set":
            sign = np.where(rng.integers(0, 2, k, dtype=np.uint8) == 1, -1.0, 1.0).astype(np.float32)
            vals = sign * np.float32(outlier_value)
        elif outlier_mode == "mul":
            vals = base * np.float32(outlier_value)
        else:
            raise ValueError(f"unknown outlier mode {outlier_mode!r}")
        out[idx] = _to_bf16_bits(vals)
    return out.reshape(rows, cols)


# ------------------------------------------------------------------ recipes --
# Each recipe returns bf16 bit arrays.  Seeds: the tiny linear uses seed 0
# (activation) and 1 (weight); elsewhere tensor t of a workload uses its
# SEED_BASE + t.

def tiny_linear(m: int = 256, n: int = 256, k: int = 256, seed: int = 0):
    """A [m x k] N(0,1) with 0.1% of entries set to +-50; W [n x k] N(0, 0.02^2)."""
    a = make_tensor(m, k, seed, "normal", 1.0, 0.001, "set", 50.0)
    w = make_tensor(n, k, seed + 1, "normal", 0.02)
    return a, w


def activation(rows: int, cols: int, seed: int, outlier_frac: float = 0.0005, outlier_mul: float = 100.0):
    """Activations X: N(0,1) with a fraction of entries scaled by outlier_mul."""
    return make_tensor(rows, cols, seed, "normal", 1.0, outlier_frac, "mul", outlier_mul)


def weight(rows: int, cols: int, seed: int, std: float = 0.015):
    """Weights W: N(0, std^2)."""
    return make_tensor(rows, cols, seed, "normal", std)


def gradient(rows: int, cols: int, seed: int, b: float = 1e-3, outlier_frac: float = 0.001,
             outlier_mul: float = 1000.0):
    """Gradients dY: Laplace(0, b) with a fraction of entries scaled by outlier_mul."""
    return make_tensor(rows, cols, seed, "laplace", b, outlier_frac, "mul", outlier_mul)


def sweep_tensor(n_elems: int, dist: str, seed: int, cols: int = 4096):
    """Quantizer sweep tensor of n_elems elements in rows of `cols`.

    dist: "normal" (N(0,1)), "lognormal" (lognormal(0, 2) with random signs),
    "outliers" (N(0,1) with 0.1% of entries set to +-1e4)."""
    rows = n_elems // cols
    if dist == "normal":
        return make_tensor(rows, cols, seed, "normal", 1.0)
    if dist == "lognormal":
        return make_tensor(rows, cols, seed, "lognormal_signed", 2.0)
    if dist == "outliers":
        return make_tensor(rows, cols, seed, "normal", 1.0, 0.001, "set", 1e4)
    raise ValueError(dist)


# Workload shapes (tokens x hidden, ffn), from the MLP-layer recipes.
MLP_FPROP = dict(tokens=8192, hidden=4096, ffn=14336)         # Y = X W1^T
MLP_WGRAD = dict(tokens=8192, hidden=4096, ffn=14336)         # dW = dY^T X
MLP_STEP = dict(tokens=16384, hidden=8192, ffn=28672)         # fprop + dgrad + wgrad
SWEEP_SIZES = (1 << 20, 1 << 24, 1 << 28, 1 << 30)
SWEEP_DISTS = ("normal", "lognormal", "outliers")
SEED_BASE = {"tiny_linear": 0, "mlp_fprop": 2000, "mlp_wgrad": 3000, "sweep": 4000, "mlp_step": 5000}


def seeds(workload: str):
    """(tensor seed base, rht_seed, sr_seed) of a named workload."""
    b = SEED_BASE[workload]
    return b, b + 100, b + 101
