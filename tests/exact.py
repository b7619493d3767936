"""Independent exact-arithmetic helpers for pinning the oracle.

These do not share code with ``oracle``: rounding is done by comparing the
candidate neighbours of a value with Python's exact ``Fraction`` arithmetic,
not by constructing the significand.
"""

from fractions import Fraction

import numpy as np


def f32_exact(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def nearest_f32(fr: Fraction) -> np.float32:
    """The float32 nearest to the rational ``fr`` (ties to an even last bit)."""
    f = np.float32(float(fr))
    cands = {f, np.nextafter(f, np.float32(-np.inf)), np.nextafter(f, np.float32(np.inf))}
    cands = [c for c in cands if np.isfinite(c)]

    def key(c):
        return (abs(Fraction(float(c)) - fr), int(np.float32(c).view(np.uint32)) & 1)

    return np.float32(min(cands, key=key))


def bf16_bits_of(v: float) -> int:
    return int(np.float32(v).view(np.uint32)) >> 16


def nearest_bf16_bits(v32: np.float32) -> int:
    """bfloat16 bit pattern nearest to float32 ``v32`` (ties to even)."""
    u = int(np.float32(v32).view(np.uint32))
    lo = u >> 16
    hi = lo + 1
    val = Fraction(float(np.float32(v32)))

    def as_frac(b):
        return Fraction(float(np.uint32(b << 16).view(np.float32)))

    dlo = abs(as_frac(lo) - val)
    dhi = abs(as_frac(hi) - val)
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    return lo if lo % 2 == 0 else hi
