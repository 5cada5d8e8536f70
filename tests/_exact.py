"""Exact rational re-derivations used to pin the oracle (no code shared with it).

Everything here works on ``fractions.Fraction`` values, so each rounding is carried
out exactly from its definition: binary32 round-to-nearest-even for the two
divisions of the quantizer, and nearest-finite-E4M3 with ties to the even code.
The E4M3 candidate values come from ml_dtypes' float8_e4m3fn type, an
implementation independent of the oracle's decoder.
"""
from __future__ import annotations

from fractions import Fraction

import ml_dtypes
import numpy as np

_HALF = Fraction(1, 2)


def e4m3_values_lib() -> np.ndarray:
    """Value of each of the 256 codes, decoded by ml_dtypes (float64)."""
    return np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


_CANDS = None


def _cands():
    global _CANDS
    if _CANDS is None:
        vals = e4m3_values_lib()
        _CANDS = [(Fraction(float(vals[c])), c) for c in range(0x7F)]  # +0 .. 448
    return _CANDS


def round_binary32(q: Fraction) -> Fraction:
    """Round a rational to the nearest binary32 value, ties to even (no overflow)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)  # below 2^-126 the spacing is that of the subnormals
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > _HALF or (rem == _HALF and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def nearest_e4m3(v: Fraction, negative: bool) -> int:
    """Code of the finite E4M3 value nearest to v, ties to the even code; values
    beyond 448 go to 448.  `negative` gives the sign (needed for -0)."""
    a = abs(v)
    best = None
    for val, code in _cands():
        d = abs(a - val)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return best[1] | (0x80 if negative else 0)


def bf16_to_fraction(bits: int) -> tuple[Fraction, bool]:
    f = np.array([bits], dtype=np.uint16).astype(np.uint32) << 16
    x = float(f.view(np.float32)[0])
    return Fraction(x), bool(bits & 0x8000)


def quantize_group_exact(bits) -> tuple[list[int], Fraction]:
    """Brute-force quantization of one group of BF16 bit patterns."""
    vals = [bf16_to_fraction(int(b)) for b in bits]
    amax = max(abs(v) for v, _ in vals)
    if amax == 0:
        return [0] * len(vals), Fraction(0)
    s = round_binary32(amax / 448)
    codes = [nearest_e4m3(round_binary32(v / s), neg) for v, neg in vals]
    return codes, s
