"""The quantizers compute each group scale amax / 448 with three operations (a
multiply by RN(1/448) and one FMA correction step, Markstein's method) instead of a
full IEEE division.  amax is always a non-negative BF16 value, so the claim that this
equals the correctly rounded quotient can be checked for every possible input: here,
with exact rational arithmetic and binary32 rounding from its definition.  (The GPU
side is checked against the oracle for every BF16 amax in test_quant_gpu.py.)"""
from fractions import Fraction

import numpy as np

from tests._exact import round_binary32


def test_scale_sequence_is_the_ieee_quotient_for_every_bf16_amax():
    inv = round_binary32(Fraction(1, 448))
    bits = np.arange(1, 0x7F80, dtype=np.uint32) << 16      # every positive finite BF16
    vals = bits.view(np.float32)
    bad = []
    for v in vals:
        a = Fraction(float(v))
        q0 = round_binary32(a * inv)               # q0 = RN(amax * RN(1/448))
        d = round_binary32(a - q0 * 448)           # d = fma(-q0, 448, amax)
        s = round_binary32(q0 + d * inv)           # s = fma(d, RN(1/448), q0)
        if s != round_binary32(a / 448):
            bad.append(float(v))
    assert not bad, f"{len(bad)} amax values differ, e.g. {bad[:3]}"
    # zero: q0 = d = s = 0
    assert round_binary32(Fraction(0) * inv) == 0
