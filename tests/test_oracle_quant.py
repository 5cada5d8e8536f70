"""Pins for the oracle's quantizers (1x128 groups, token-dim groups, 128x128 blocks).

Checks: brute force with exact rational arithmetic, exact cases built from E4M3
values times powers of two, invariants, and relations between the three layouts.
"""
import numpy as np
import pytest

import oracle
from blockwise_fp8_linear_b200 import synth
from tests._exact import e4m3_values_lib, quantize_group_exact


def _bits_from_f32(x):
    """float32 values that are exactly BF16 -> BF16 bit patterns."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "values must be BF16-representable"
    return (b >> 16).astype(np.uint16)


def _scale_f32(s) -> int:
    return int(np.float32(s).view(np.uint32))


@pytest.mark.parametrize("seed", range(6))
def test_group_brute_force_exact(seed):
    rng = np.random.default_rng(seed)
    kind = seed % 3
    if kind == 0:
        x = rng.standard_normal(128)
    elif kind == 1:
        x = rng.standard_normal(128) * 1e-3
        x[rng.integers(0, 128)] *= 20
    else:  # wide dynamic range within the group, including tiny values
        x = rng.standard_normal(128) * 2.0 ** rng.integers(-40, 10, 128)
    bits = synth.f64_to_bf16_bits(x)
    bits[5] = 0x8000  # a negative zero inside a nonzero group
    codes, s = oracle.quantize_group(bits)
    want_codes, want_s = quantize_group_exact(bits)
    assert _scale_f32(s) == _scale_f32(np.float32(float(want_s)))
    assert list(codes) == want_codes
    assert codes[5] == 0x80


def test_weight_slab_brute_force_exact():
    """A 128x256 weight slab (two 128x128 blocks) against exact arithmetic."""
    rng = np.random.default_rng(99)
    w = rng.standard_normal((128, 256)) * 0.02
    w[:, 128:] *= 37.0  # the second block has a different scale
    w[3, 200] = 1.5
    bits = synth.f64_to_bf16_bits(w)
    q, s, _ = oracle.quant_weight(bits)
    assert s.shape == (1, 2)
    for kb in range(2):
        blk = bits[:, kb * 128:(kb + 1) * 128].ravel()
        want_codes, want_s = quantize_group_exact(blk)
        assert _scale_f32(s[0, kb]) == _scale_f32(np.float32(float(want_s)))
        assert list(q[:, kb * 128:(kb + 1) * 128].ravel()) == want_codes


@pytest.mark.parametrize("e", [-30, -12, -7, -1, 0, 3, 9])
def test_exact_power_of_two_groups(e):
    """Groups of E4M3 values times 2^e with one element at +-448*2^e: the scale is
    exactly 2^e, each quotient is exactly the chosen E4M3 value, so the codes are
    the chosen codes and dequantization gives back x bit for bit."""
    vals = e4m3_values_lib()
    rng = np.random.default_rng(1000 + e)
    finite_codes = np.array([c for c in range(256) if not np.isnan(vals[c])])
    codes = rng.choice(finite_codes, 128)
    codes[17] = 0x7E if e % 2 else 0xFE
    codes[0] = 0x80  # -0 stays -0 in a nonzero group
    x = vals[codes] * 2.0 ** e
    bits = _bits_from_f32(x.astype(np.float32))
    q, s = oracle.quantize_group(bits)
    assert float(s) == 2.0 ** e
    assert list(q) == list(codes)
    assert np.array_equal(vals[q] * float(s), x)


def test_all_zero_group_and_signed_zero():
    z = np.zeros(128, dtype=np.uint16)
    z[::2] = 0x8000
    q, s = oracle.quantize_group(z)
    assert float(s) == 0.0 and np.all(q == 0)
    # a single nonzero value: every other entry is +-0, the value maps to 448
    z[7] = _bits_from_f32(np.float32(-3.0))[()]
    q, s = oracle.quantize_group(z)
    assert float(s) == np.float32(3.0) / np.float32(448.0)
    assert q[7] == 0xFE and q[0] == 0x80 and q[1] == 0x00


def test_group_invariants_random():
    x = synth.normal_bf16(512, 1024, 1.0, seed=5, outliers=True)
    q, s = oracle.quant_act(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    vals = e4m3_values_lib()
    for m in range(0, 512, 37):
        for kb in range(8):
            g = xf[m, kb * 128:(kb + 1) * 128]
            amax = np.float32(np.max(np.abs(g)))
            sc = s[kb, m]
            assert sc == amax / np.float32(448.0)          # s == amax/448 bitwise
            codes = q[m, kb * 128:(kb + 1) * 128]
            dq = vals[codes]
            assert np.all(np.abs(dq) <= 448)
            i = np.argmax(np.abs(g))
            assert codes[i] == (0xFE if g[i] < 0 else 0x7E)  # the amax element -> 448
            normal = np.abs(dq) >= 2.0 ** -6
            err = np.abs(dq * sc - g)[normal]
            assert np.all(err <= np.abs(g[normal]) * (2.0 ** -4 + 2.0 ** -20))


def test_act_t_is_act_of_transpose():
    x = synth.normal_bf16(384, 256, 1.0, seed=11, outliers=True)
    qt, st = oracle.quant_act_t(x)
    q2, s2 = oracle.quant_act(np.ascontiguousarray(x.T))
    assert qt.shape == (256, 384) and st.shape == (3, 256)
    assert np.array_equal(qt, q2)
    assert np.array_equal(st.view(np.uint32), s2.view(np.uint32))


def test_act_layouts_against_groupwise():
    """quant_act places group (m, kb) at q[m, kb*128:] and s[kb, m]."""
    x = synth.normal_bf16(256, 384, 1.0, seed=12)
    q, s = oracle.quant_act(x)
    for m in (0, 1, 129, 255):
        for kb in range(3):
            gq, gs = oracle.quantize_group(x[m, kb * 128:(kb + 1) * 128])
            assert np.array_equal(q[m, kb * 128:(kb + 1) * 128], gq)
            assert s[kb, m] == gs


def test_weight_layout_and_transpose():
    w = synth.normal_bf16(384, 256, 0.02, seed=13)
    q, s, qt = oracle.quant_weight(w, want_t=True)
    assert s.shape == (3, 2)
    assert np.array_equal(qt, q.T)
    for nb in range(3):
        for kb in range(2):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            gq, gs = oracle.quantize_group(np.ascontiguousarray(blk).ravel())
            assert s[nb, kb] == gs
            assert np.array_equal(q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128].ravel(), gq)
    # the scale of each block is set by that block's own amax: scaling one block
    # by a power of two changes only its scale
    w2 = synth.bf16_bits_to_f32(w).copy()
    w2[128:256, 0:128] *= 4.0
    q2, s2, _ = oracle.quant_weight(_bits_from_f32(w2))
    assert s2[1, 0] == s[1, 0] * 4 and np.array_equal(q2, q)
    s_other = s2.copy(); s_other[1, 0] = s[1, 0]
    assert np.array_equal(s_other, s)


def test_bad_sizes_rejected():
    with pytest.raises(ValueError):
        oracle.quant_act(np.zeros((128, 200), dtype=np.uint16))   # features not a multiple of 128
    with pytest.raises(ValueError):
        oracle.quant_act_t(np.zeros((100, 64), dtype=np.uint16))
    with pytest.raises(ValueError):
        oracle.quant_weight(np.zeros((128, 200), dtype=np.uint16))
    with pytest.raises(ValueError):
        oracle.quant_weight(np.zeros((100, 128), dtype=np.uint16))  # weights stay whole blocks


# ---- token counts that are not a multiple of 128 (the last token group is partial) ----

def test_act_t_partial_group_exact():
    """M = 147 tokens: per column, one full group of 128 and a last group of the 19
    tokens present; every group's codes and scale against the exact rational
    checker run on exactly those values (the scale is amax/448 over the 19 present
    tokens, not over a padded 128)."""
    M, K = 147, 128
    x = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(147, 0), outliers=True)
    qt, st = oracle.quant_act_t(x)
    assert qt.shape == (K, M) and st.shape == (2, K)
    for k in range(0, K, 7):
        for mb, (r0, r1) in enumerate(((0, 128), (128, M))):
            codes, sc = quantize_group_exact(x[r0:r1, k])
            assert list(qt[k, r0:r1]) == codes, (k, mb)
            assert np.float32(st[mb, k]) == np.float32(float(sc)), (k, mb)


def test_act_t_ragged_equals_zero_padded():
    """Zero tokens change no amax, so the ragged result equals the quantization of the
    input zero-padded to a multiple of 128 tokens, restricted to the tokens present."""
    for M in (16, 200, 272):
        K = 256
        x = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(M, 1), outliers=True)
        pad = np.zeros(((M + 127) // 128 * 128, K), dtype=np.uint16)
        pad[:M] = x
        qt, st = oracle.quant_act_t(x)
        qtp, stp = oracle.quant_act_t(pad)
        assert np.array_equal(qt, qtp[:, :M])
        assert np.array_equal(st.view(np.uint32), stp.view(np.uint32))


def test_act_ragged_rows_independent():
    """Groups along K: each token row is quantized on its own, so M = 37 rows equal
    the first 37 rows of a 128-row call on the same values."""
    K = 384
    big = synth.normal_bf16(128, K, 1.0, seed=synth.seed_for(37, 2), outliers=True)
    q, s = oracle.quant_act(big[:37])
    qb, sb = oracle.quant_act(big)
    assert q.shape == (37, K) and s.shape == (K // 128, 37)
    assert np.array_equal(q, qb[:37])
    assert np.array_equal(s.view(np.uint32), sb[:, :37].view(np.uint32))
