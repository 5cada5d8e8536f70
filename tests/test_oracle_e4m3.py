"""Pins for the oracle's E4M3 decoder and RNE-saturating encoder.

The oracle is checked against things other than itself: two independent
float8_e4m3fn implementations (torch, ml_dtypes), the spot values of the format
definition (tests/golden), and a brute-force nearest-value search.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from tests._exact import e4m3_values_lib

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spot_values.txt")


def _torch_table():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_all_codes_match_two_libraries():
    ours = oracle.e4m3_decode_table()
    for ref in (_torch_table(), e4m3_values_lib()):
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(ours), nan)
        assert np.array_equal(ours[~nan], ref[~nan])
        # signed zeros too
        assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_decode_spot_values_from_format_definition():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for code, val in rows:
        got = oracle.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            want = float(val)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), code


def test_decode_structure():
    t = oracle.e4m3_decode_table()
    finite = t[~np.isnan(t)]
    assert finite.size == 254
    assert np.max(finite) == 448.0 and np.min(finite) == -448.0
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)  # codes 0x00..0x7E are increasing
    assert np.array_equal(t[0x80:0xFF], -t[0x00:0x7F])


def test_encode_roundtrip_every_finite_code():
    t = oracle.e4m3_decode_table()
    codes = [c for c in range(256) if not math.isnan(t[c])]
    got = oracle.e4m3_encode_array(np.array([t[c] for c in codes], dtype=np.float32))
    assert list(got) == codes


def _brute_force(v: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 value by exhaustive search, ties to the even code.

    Distances to the two bracketing candidates are exact in float64 (Sterbenz /
    both operands on a grid much finer than 2^-53 relative), which is all that
    decides the result.  Magnitudes beyond 1024 are clamped to 1024: every
    candidate is <= 448, so that keeps their order of distance and keeps the
    float64 differences exact."""
    cand = e4m3_values_lib()[:0x7F]  # +0 .. 448, increasing
    a = np.minimum(np.abs(v.astype(np.float64)), 1024.0)
    out = np.empty(v.shape, dtype=np.uint8)
    step = 1 << 16
    for s in range(0, a.size, step):
        blk = a[s:s + step, None]
        d = np.abs(blk - cand[None, :])
        dmin = d.min(axis=1, keepdims=True)
        tie = d == dmin
        # among tied candidates prefer the even code
        even = (np.arange(0x7F) % 2 == 0)[None, :]
        pick = np.where((tie & even).any(axis=1), np.argmax(tie & even, axis=1), np.argmax(tie, axis=1))
        out[s:s + step] = pick
    out |= np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    return out


def _edge_floats():
    """Every float32 in [2^-12, 512] with structured mantissas, plus all E4M3
    midpoints and their float32 neighbours."""
    vals = []
    low20 = [0, 1, 2, 0x3FFFF, 0x40000, 0x7FFFF, 0x80000, 0x80001, 0xBFFFF, 0xC0000,
             0xC0001, 0xFFFFE, 0xFFFFF]
    for e in range(127 - 12, 127 + 10):
        for top in range(8):  # the 3 mantissa bits E4M3 keeps in a normal binade
            for lo in low20:
                vals.append((e << 23) | (top << 20) | lo)
    f = np.array(vals, dtype=np.uint32).view(np.float32)
    cand = e4m3_values_lib()[:0x7F]
    mids = ((cand[:-1] + cand[1:]) / 2).astype(np.float32)  # exact in float32
    ext = [mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0))]
    extra = np.array([448, 449, 463.99997, 464, 464.00003, 480, 1e6, 3.4e38, 0.0,
                      2 ** -10, 2 ** -11, 2 ** -10 * 3, 2 ** -149, 1e-45], dtype=np.float32)
    allv = np.concatenate([f, *ext, extra])
    return np.concatenate([allv, -allv])


def test_encode_brute_force_edges():
    v = _edge_floats()
    assert np.array_equal(oracle.e4m3_encode_array(v), _brute_force(v))


def test_encode_brute_force_random():
    rng = np.random.default_rng(12345)
    parts = [
        # log-uniform magnitudes spanning subnormal E4M3 .. beyond saturation
        (2.0 ** rng.uniform(-14, 10, 2_000_000)).astype(np.float32),
        # random bit patterns restricted to finite values
        rng.integers(0, 0x7F800000, 2_000_000, dtype=np.uint32).view(np.float32),
        rng.standard_normal(2_000_000).astype(np.float32) * 50,
    ]
    v = np.concatenate(parts)
    v[::2] *= -1
    assert np.array_equal(oracle.e4m3_encode_array(v), _brute_force(v))


def test_encode_matches_libraries_in_range():
    """torch and ml_dtypes round to nearest-even; they turn magnitudes above 464
    into NaN rather than saturating, so compare where |v| <= 464."""
    rng = np.random.default_rng(7)
    v = np.concatenate([(2.0 ** rng.uniform(-14, 8.85, 1_000_000)).astype(np.float32),
                        _edge_floats()])
    v = v[np.abs(v) <= 464]
    ours = oracle.e4m3_encode_array(v)
    t = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    m = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, t)
    assert np.array_equal(ours, m)


def test_encode_saturates_and_keeps_sign_of_zero():
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(464.0) == 0x7E          # tie between 448 and (absent) 480
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-30) == 0x80
    assert oracle.e4m3_encode(2 ** -10) == 0x00       # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(3 * 2 ** -10) == 0x02   # tie between 2^-9 and 2*2^-9 -> even
