"""Pins for the oracle's power-of-two (E8M0) scale quantizers.

Puro-2B part 3/7, section 3.2: on the RTX 5090 the 128-blocks run through Transformer
Engine's MXFP8 path, where every block scale is a power of two (an 8-bit exponent).
Reading: the scale is the smallest 2^e with amax <= 448 * 2^e, e in [-127, 127], code
e + 127; dividing by 2^e is exact, so each code is one RNE of x * 2^-e onto E4M3.

Checks: the exponent of every positive finite BF16 amax against exact rational
arithmetic, brute-force groups, exact cases, invariants, the three layouts, and the
FP32-scale path against the power-of-two one on a GEMM.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockwise_fp8_linear_b200 import synth
from tests._exact import bf16_to_fraction, e4m3_values_lib, nearest_e4m3


def _exact_exponent(amax: Fraction) -> int:
    """Smallest integer e with amax <= 448 * 2^e, found on exact rationals."""
    if amax == 0:
        return -127
    t = amax / 448
    e = t.numerator.bit_length() - t.denominator.bit_length()
    while Fraction(2) ** e < t:
        e += 1
    while Fraction(2) ** (e - 1) >= t:
        e -= 1
    return max(-127, min(127, e))


def _bf16_value(bits: int) -> Fraction:
    return bf16_to_fraction(bits)[0]


def test_exponent_every_bf16_amax():
    for bits in range(0, 0x7F80):
        a = _bf16_value(bits)
        got = oracle.e8m0_exponent(float(a))
        assert got == _exact_exponent(a), (hex(bits), got)


def _group_exact(bits):
    vals = [bf16_to_fraction(int(b)) for b in bits]
    amax = max(abs(v) for v, _ in vals)
    if amax == 0:
        return [0] * len(vals), 0
    e = _exact_exponent(amax)
    scale = Fraction(2) ** e
    return [nearest_e4m3(v / scale, neg) for v, neg in vals], e + 127


@pytest.mark.parametrize("seed", range(8))
def test_group_brute_force_exact(seed):
    rng = np.random.default_rng(100 + seed)
    kind = seed % 4
    if kind == 0:
        x = rng.standard_normal(128)
    elif kind == 1:
        x = rng.standard_normal(128) * np.exp2(rng.integers(-20, 20, 128))
    elif kind == 2:
        x = rng.standard_normal(128) * 2.0 ** -128       # scale clamped at 2^-127
    else:
        x = rng.standard_normal(128); x[rng.integers(0, 128)] *= 1e4
    bits = synth.f64_to_bf16_bits(x)
    q, c = oracle.quantize_group_e8m0(bits)
    q_ref, c_ref = _group_exact(bits)
    assert int(c) == c_ref
    assert [int(v) for v in q] == q_ref


def test_exact_powers_of_two():
    """A group of E4M3 values times 2^k with an element at +-448 * 2^k has scale
    exactly 2^k and returns its own codes."""
    vals = e4m3_values_lib()
    finite = np.array([c for c in range(256) if np.isfinite(vals[c]) and c not in (0x00, 0x80)])
    rng = np.random.default_rng(7)
    for k in (-120, -9, -1, 0, 3, 40, 119):
        codes = rng.choice(finite, 128)
        codes[5] = 0xFE
        x = vals[codes] * 2.0 ** k
        bits = synth.f64_to_bf16_bits(x)
        if not np.all(np.isfinite(x)):
            continue
        back = np.array([float(_bf16_value(int(b))) for b in bits])
        if not np.array_equal(back, x):
            continue  # BF16 cannot hold these values at this exponent
        q, c = oracle.quantize_group_e8m0(bits)
        assert int(c) == k + 127
        assert np.array_equal(q, codes.astype(np.uint8))


def test_invariants_and_zero_group():
    rng = np.random.default_rng(3)
    for _ in range(200):
        x = rng.standard_normal(128) * np.exp2(rng.uniform(-60, 60))
        bits = synth.f64_to_bf16_bits(x)
        q, c = oracle.quantize_group_e8m0(bits)
        e = int(c) - 127
        amax = max(abs(_bf16_value(int(b))) for b in bits)
        assert amax <= 448 * Fraction(2) ** e
        assert e == -127 or amax > 224 * Fraction(2) ** e
        dec = oracle.e4m3_decode_table()[q]
        assert np.all(np.abs(dec) <= 448)
        i = int(np.argmax(np.abs(x)))
        assert 224 <= abs(dec[i]) <= 448
    z = np.zeros(128, dtype=np.uint16)
    z[::3] = 0x8000
    q, c = oracle.quantize_group_e8m0(z)
    assert int(c) == 0 and not q.any()


def test_layouts():
    x = synth.normal_bf16(256, 384, 1.0, seed=11, outliers=True)
    q, s = oracle.quant_act_e8m0(x)
    qt, st = oracle.quant_act_t_e8m0(np.ascontiguousarray(x.T))
    assert np.array_equal(qt, q) and np.array_equal(st, s)  # qt[k][m] is the code of X[k][m]
    for m in (0, 77, 255):
        for kb in range(3):
            qq, cc = oracle.quantize_group_e8m0(x[m, kb * 128:(kb + 1) * 128])
            assert np.array_equal(q[m, kb * 128:(kb + 1) * 128], qq) and s[kb, m] == cc
    w = synth.normal_bf16(256, 384, 0.02, seed=12)
    qw, sw, qwt = oracle.quant_weight_e8m0(w, want_t=True)
    assert np.array_equal(qwt, qw.T)
    for nb in range(2):
        for kb in range(3):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            amax = max(abs(_bf16_value(int(b))) for b in blk.ravel()[::1])
            assert int(sw[nb, kb]) == _exact_exponent(amax) + 127


def test_fp32_and_power_of_two_scales_on_a_gemm():
    """Both forms of the recipe against the exact product of the BF16 inputs: the
    power-of-two scale never saturates but leaves up to one bit of the E4M3 range
    unused, so its error is at least comparable to the FP32-scale error; both stay
    at the few-percent level of E4M3's 3-bit mantissa."""
    T, Din, Dout = 256, 1024, 384
    X = synth.normal_bf16(T, Din, 1.0, seed=21, outliers=True)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=22)
    xf = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wf = (W.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y_true = xf @ wf.T
    qx, sx = oracle.quant_act(X)
    qw, sw, _ = oracle.quant_weight(W)
    y32, _ = oracle.gemm(oracle.FPROP, qx, sx, qw, sw, T, Dout, Din)
    ex, cx = oracle.quant_act_e8m0(X)
    ew, cw, _ = oracle.quant_weight_e8m0(W)
    y8, _ = oracle.gemm(oracle.FPROP, ex, oracle.e8m0_to_float(cx), ew,
                        oracle.e8m0_to_float(cw), T, Dout, Din)
    rel = lambda y: np.linalg.norm(y - y_true) / np.linalg.norm(y_true)
    r32, r8 = rel(y32), rel(y8)
    assert r32 < 0.05 and r8 < 0.05
    assert r8 >= 0.9 * r32


@pytest.mark.parametrize("pos", [(0, 0), (0, 127), (77, 3), (127, 127)])
def test_weight_scale_is_the_whole_blocks_amax(pos):
    """Puro-2B part 3/7, section 3.2: a weight's scale covers its 128x128 tile, so the
    exponent follows the tile's largest magnitude wherever it sits; the planted
    element lands exactly on +-448 and every other code is the exact nearest value
    of x / 2^e."""
    rng = np.random.default_rng(5)
    w = rng.uniform(-1.0, 1.0, size=(128, 256))
    i, j = pos
    w[i, 128 + j] = -3584.0                     # 448 * 2^3, exactly representable in BF16
    bits = synth.f64_to_bf16_bits(w)
    q, s, _ = oracle.quant_weight_e8m0(bits)
    assert int(s[0, 1]) == 3 + 127
    assert q[i, 128 + j] == 0xFE                 # -448
    amax0 = max(abs(_bf16_value(int(b))) for b in bits[:, :128].ravel())
    assert int(s[0, 0]) == _exact_exponent(amax0) + 127
    for r in (0, i, 127):
        for c in (0, j, 127):
            v = bf16_to_fraction(int(bits[r, 128 + c]))
            assert int(q[r, 128 + c]) == nearest_e4m3(v[0] / 8, v[1])
