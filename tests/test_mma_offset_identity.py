"""The row-wise encode kernels compute the GEMM scale-layout offset of block b
of row r as (r >> 7) * (chunks_k << 9) + ((16 b) >> 6 << 9) + ((r & 31) << 4 |
((r >> 5) & 3) << 2 | (b & 3)), with r taken as a 32-bit unsigned value.  This
checks that form against the layout's definition (nvfp4.h: chunk (r/128, b/4)
at ((r/128) * chunks_k + b/4) * 512, inside it (r%32)*16 + ((r/32)%4)*4 + b%4)
over the whole admissible row range (r < 2^31)."""
import numpy as np


def layout_offset(r, b, chunks_k):
    return ((r // 128) * chunks_k + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + b % 4


def kernel_offset(r, b, chunks_k):
    r32 = r & 0xFFFFFFFF
    col0 = 16 * b
    return (r32 >> 7) * (chunks_k << 9) + ((col0 >> 6) << 9) + (((r32 & 31) << 4) | (((r32 >> 5) & 3) << 2) | (b & 3))


def test_offset_identity_random_and_extremes():
    rng = np.random.default_rng(11)
    rows = [0, 1, 31, 32, 127, 128, 129, 2**24 + 5, 2**31 - 1] + [int(v) for v in rng.integers(0, 2**31, 2000)]
    for r in rows:
        chunks_k = int(rng.integers(1, 2**25))
        for b in [0, 1, 2, 3, 4, 63, 64, 4 * chunks_k - 1] + [int(v) for v in rng.integers(0, 4 * chunks_k, 8)]:
            assert kernel_offset(r, b, chunks_k) == layout_offset(r, b, chunks_k), (r, b, chunks_k)
