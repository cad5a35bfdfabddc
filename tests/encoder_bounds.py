"""Step tables of the E4M3 and E2M1 encoders, derived from the oracle.

bounds[i] is the smallest fp32 magnitude bit pattern whose code is i + 1
(codes of non-negative values, saturating encoders), found by bisection over
the bit patterns with the oracle's encoder. Test infrastructure only.
"""
from __future__ import annotations

import numpy as np

import oracle

MAX_FINITE_BITS = 0x7F7FFFFF


def _f32(bits: int) -> float:
    return float(np.array([bits], dtype=np.uint32).view(np.float32)[0])


def encoder_bounds(encode, n_codes: int) -> np.ndarray:
    """Bounds for codes 1 .. n_codes - 1 of a monotone encoder of magnitudes."""
    out = []
    for c in range(1, n_codes):
        lo, hi = 0, MAX_FINITE_BITS           # encode(f(lo)) < c <= encode(f(hi))
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if encode(_f32(mid)) >= c:
                hi = mid
            else:
                lo = mid
        out.append(hi)
    return np.array(out, dtype=np.uint32)


def e4m3_bounds() -> np.ndarray:
    return encoder_bounds(oracle.e4m3_encode, 127)   # codes 0 .. 126 (0x7E = 448)


def e2m1_bounds() -> np.ndarray:
    return encoder_bounds(oracle.e2m1_encode, 8)     # codes 0 .. 7 (6.0)
