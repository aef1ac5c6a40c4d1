"""Shared test helpers: moving bf16 bit arrays to the device and the MMA
scale-layout permutation (the layout nvfp4.h defines, restated here from its
formula so that the tests do not depend on the library's own indexing)."""
import numpy as np
import torch


def to_device_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def mma_layout(plain: np.ndarray, rows: int, kb: int, expand_2d: bool = False) -> np.ndarray:
    """Plain scales -> MMA layout bytes.  plain is [rows x kb] (1D) or
    [rows/16 x kb] (2D, expanded per row when expand_2d)."""
    chunks_k = (kb + 3) // 4
    rchunks = (rows + 127) // 128
    out = np.zeros(rchunks * chunks_k * 512, dtype=np.uint8)
    r = np.arange(rows)[:, None]
    b = np.arange(kb)[None, :]
    off = ((r // 128) * chunks_k + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
    vals = plain[np.arange(rows) // 16] if expand_2d else plain
    out[off.ravel()] = np.asarray(vals, dtype=np.uint8).reshape(rows, kb).ravel()
    return out


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    lo = packed & 0xF
    hi = packed >> 4
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def first_mismatch(a: np.ndarray, b: np.ndarray):
    idx = np.argwhere(a != b)
    if idx.size == 0:
        return None
    i = tuple(idx[0])
    return f"{len(idx)} mismatches; first at {i}: got {a[i]} expected {b[i]}"
