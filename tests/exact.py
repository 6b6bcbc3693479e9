"""Exact-arithmetic helpers for the oracle's pins (test infrastructure).

Rounding to binary32 is characterised here by brute force: among the three
fp32 neighbours of an approximation, take the one nearest to the exact
rational value, ties to the even significand.  This is independent of the
oracle's C arithmetic."""
from __future__ import annotations

from fractions import Fraction

import numpy as np

F32 = np.float32


def frac(x) -> Fraction:
    return Fraction(float(x))


def nearest_f32(fr: Fraction) -> np.float32:
    c = F32(float(fr))
    cands = [np.nextafter(c, F32(-np.inf)), c, np.nextafter(c, F32(np.inf))]
    best = None
    for cand in cands:
        if not np.isfinite(cand):
            continue
        err = abs(frac(cand) - fr)
        even = (int(np.array(cand, dtype=np.float32).view(np.uint32)) & 1) == 0
        key = (err, 0 if even else 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return F32(best[1])


def rne_fraction(fr: Fraction) -> int:
    """Nearest integer, ties to even, of an exact rational."""
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def seq_sum_f32(vals) -> np.float32:
    """fp32 sum in the given order, each addition rounded to nearest even."""
    acc = F32(vals[0])
    for v in vals[1:]:
        acc = nearest_f32(frac(acc) + frac(v))
    return acc


def unpack_codes(codes: np.ndarray, n: int, bits: int) -> np.ndarray:
    """Codes as integers; INT4 bytes hold the even element in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    if bits == 8:
        return codes[:n].astype(np.int64)
    out = np.empty(n, dtype=np.int64)
    out[0::2] = codes & 0x0F
    out[1::2] = codes >> 4
    return out
