"""CPU check of the rounding argument behind the kernels' hardware-convert
E2M1 path (block-128 staged and streaming row-wise kernels).

The convert rounds to nearest with ties to even; the codebook rule of the
QAT page (_round_to_e2m1: bucketize(|y|, midpoints, right=True)) sends ties
to the larger magnitude. The kernels give the convert
y' = fl32(x * (2^-k (1 + 2^-20)) + 0) instead of y = x * 2^-k. Emulated here
in float64 (the product of a bf16 value and the 24-bit multiplier is exact in
float64; one rounding to float32 is the fma's), then rounded to the E2M1
grid with ties to even: for every finite bf16 x and every k the kernels use
the convert for ([-125, 16]), with |y| below the block bound 8.5, the
magnitude index equals the codebook rule's and the sign of a zero code
follows the +0 addend (x = -0 gives +0)."""
from __future__ import annotations

import numpy as np

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def rne_index(a: np.ndarray) -> np.ndarray:
    """Index of the nearest grid value, ties to the even index (the even
    mantissa bit of E2M1 codes 0..7 is bit 0), saturating at 6."""
    d = np.abs(a[:, None] - GRID[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    even = cand & ((np.arange(8) & 1) == 0)[None, :]
    return np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))


def test_nudged_convert_equals_ties_up_rule():
    b = np.arange(65536, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    x = f[np.isfinite(f)].astype(np.float64)
    mult = 1.0 + 2.0 ** -20  # 2^-k (1 + 2^-20): mantissa bit 3 of the fp32 multiplier set
    for k in range(-125, 17):
        y = x * 2.0 ** -k
        keep = np.abs(y) < 8.5  # |y| <= amax / 2^k < 8.49 inside a fast-path block
        yk, xk = y[keep], x[keep]
        yn = (yk * mult).astype(np.float32).astype(np.float64) + 0.0
        got = rne_index(np.abs(yn))
        ref = np.searchsorted(MIDS, np.abs(yk), side="right")  # bucketize(right=True)
        assert np.array_equal(got, ref), f"k={k}: {np.count_nonzero(got != ref)} differ"
        # sign: the +0 addend turns -0 into +0; every nonzero product keeps its sign
        zero_in = xk == 0
        assert not np.any(np.signbit(yn[zero_in]))
        assert np.array_equal(np.signbit(yn[~zero_in]), np.signbit(xk[~zero_in]))
