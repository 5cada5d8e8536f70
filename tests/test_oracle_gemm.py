"""Pins for the oracle's blockwise GEMM (fprop / dgrad / wgrad).

Checks: exact integer cases against numpy integer matmul, numpy float64 matmul of
independently dequantized operands (ml_dtypes decode table, scales expanded with
np.repeat) on non-square shapes, exact rational sums on a few outputs, and the
three GEMMs of the linear layer expressed through X, W and dY.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockwise_fp8_linear_b200 import synth
from tests._exact import e4m3_values_lib

VALS = e4m3_values_lib()


def _rand_codes(rng, shape):
    finite = np.array([c for c in range(256) if not np.isnan(VALS[c])], dtype=np.uint8)
    return rng.choice(finite, size=shape).astype(np.uint8)


def _rand_scales(rng, shape):
    return (rng.uniform(0.5, 2.0, size=shape) * 2.0 ** rng.integers(-8, 8, size=shape)).astype(np.float32)


def _dequant_a(a, sa):
    """ahat[m][k] = code * sa[k/128][m]."""
    return VALS[a] * np.repeat(sa.astype(np.float64), 128, axis=0).T


def _dequant_b(mode, b, sb, N, K):
    """bhat as an [N][K] float64 matrix for each mode."""
    if mode == oracle.FPROP:      # b[N][K], sb[N/128][K/128]
        return VALS[b] * np.repeat(np.repeat(sb.astype(np.float64), 128, 0), 128, 1)
    if mode == oracle.DGRAD:      # b[K][N], sb[K/128][N/128]
        return (VALS[b] * np.repeat(np.repeat(sb.astype(np.float64), 128, 0), 128, 1)).T
    return VALS[b] * np.repeat(sb.astype(np.float64), 128, axis=0).T  # WGRAD: sb[K/128][N]


def _case(mode, M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = _rand_codes(rng, (M, K))
    sa = _rand_scales(rng, (K // 128, M))
    if mode == oracle.FPROP:
        b = _rand_codes(rng, (N, K)); sb = _rand_scales(rng, (N // 128, K // 128))
    elif mode == oracle.DGRAD:
        b = _rand_codes(rng, (K, N)); sb = _rand_scales(rng, (K // 128, N // 128))
    else:
        b = _rand_codes(rng, (N, K)); sb = _rand_scales(rng, (K // 128, N))
    return a, sa, b, sb


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("M,N,K", [(128, 256, 384), (256, 128, 256), (384, 384, 128)])
def test_gemm_matches_numpy_matmul(mode, M, N, K):
    a, sa, b, sb = _case(mode, M, N, K, seed=M * 7 + N * 3 + K + mode)
    y, asum = oracle.gemm(mode, a, sa, b, sb, M, N, K)
    A = _dequant_a(a, sa)
    B = _dequant_b(mode, b, sb, N, K)
    y_np = A @ B.T
    asum_np = np.abs(A) @ np.abs(B).T
    assert np.all(np.abs(y - y_np) <= 1e-12 * asum_np + 1e-300)
    assert np.allclose(asum, asum_np, rtol=1e-12, atol=0)
    assert np.all(asum >= np.abs(y))


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_gemm_exact_integer_case(mode):
    """Small-integer E4M3 codes and power-of-two scales: every product and partial
    sum is an exact dyadic number, so the FP64 result equals the integer matmul."""
    M, N, K = 128, 256, 256
    rng = np.random.default_rng(40 + mode)
    ints = {int(v): c for c, v in enumerate(VALS) if not np.isnan(v) and v == int(v) and abs(v) <= 8}
    keys = np.array(sorted(ints))
    ia = rng.choice(keys, (M, K)); a = np.vectorize(ints.get)(ia).astype(np.uint8)
    ea = rng.integers(-3, 4, (K // 128, M))
    sa = (2.0 ** ea).astype(np.float32)
    if mode == oracle.FPROP:
        ib = rng.choice(keys, (N, K)); eb = rng.integers(-3, 4, (N // 128, K // 128))
        b = np.vectorize(ints.get)(ib).astype(np.uint8)
        bfull = ib * 2.0 ** np.repeat(np.repeat(eb, 128, 0), 128, 1)
    elif mode == oracle.DGRAD:
        ib = rng.choice(keys, (K, N)); eb = rng.integers(-3, 4, (K // 128, N // 128))
        b = np.vectorize(ints.get)(ib).astype(np.uint8)
        bfull = (ib * 2.0 ** np.repeat(np.repeat(eb, 128, 0), 128, 1)).T
    else:
        ib = rng.choice(keys, (N, K)); eb = rng.integers(-3, 4, (K // 128, N))
        b = np.vectorize(ints.get)(ib).astype(np.uint8)
        bfull = ib * 2.0 ** np.repeat(eb, 128, 0).T
    sb = (2.0 ** eb).astype(np.float32)
    afull = ia * 2.0 ** np.repeat(ea, 128, 0).T
    # scale every term to an integer with a common power of two, multiply in int64
    shift = 6
    ai = np.rint(afull * 2 ** shift).astype(np.int64)
    bi = np.rint(bfull * 2 ** shift).astype(np.int64)
    exact = (ai @ bi.T).astype(np.float64) / 2.0 ** (2 * shift)
    y, _ = oracle.gemm(mode, a, sa, b, sb, M, N, K)
    assert np.array_equal(y, exact)


def test_gemm_rational_spot_check():
    mode, M, N, K = 0, 128, 128, 256
    a, sa, b, sb = _case(mode, M, N, K, seed=3)
    y, asum = oracle.gemm(mode, a, sa, b, sb, M, N, K)
    for (m, n) in [(0, 0), (5, 127), (127, 64), (77, 3)]:
        acc = Fraction(0)
        for k in range(K):
            ah = Fraction(float(VALS[a[m, k]])) * Fraction(float(sa[k // 128, m]))
            bh = Fraction(float(VALS[b[n, k]])) * Fraction(float(sb[n // 128, k // 128]))
            acc += ah * bh
        assert abs(Fraction(y[m, n]) - acc) <= Fraction(asum[m, n]) * Fraction(1, 2 ** 45)


def test_rows_subset_and_thread_independence():
    mode, M, N, K = 2, 256, 128, 384
    a, sa, b, sb = _case(mode, M, N, K, seed=8)
    y1, s1 = oracle.gemm(mode, a, sa, b, sb, M, N, K, nthreads=1)
    y4, s4 = oracle.gemm(mode, a, sa, b, sb, M, N, K, nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(s1, s4)
    rows = np.array([255, 0, 130])
    yr, _ = oracle.gemm(mode, a, sa, b, sb, M, N, K, rows=rows)
    assert np.array_equal(yr, y1[rows])


def test_linear_layer_three_gemms():
    """Fprop Y = X W^T, dgrad dX = dY W, wgrad dW = dY^T X, each computed from the
    oracle's own quantized operands, against numpy matmul of the dequantized
    tensors in the layer's natural shapes."""
    T, Din, Dout = 256, 384, 128
    X = synth.normal_bf16(T, Din, 1.0, seed=21, outliers=True)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=22)
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=23)

    qx, sx = oracle.quant_act(X)              # [T][Din], [Din/128][T]
    qw, sw, _ = oracle.quant_weight(W)        # [Dout][Din], [Dout/128][Din/128]
    qdy, sdy = oracle.quant_act(dY)           # [T][Dout], [Dout/128][T]
    qdyt, sdyt = oracle.quant_act_t(dY)       # [Dout][T], [T/128][Dout]
    qxt, sxt = oracle.quant_act_t(X)          # [Din][T], [T/128][Din]

    Xh = VALS[qx] * np.repeat(sx.astype(np.float64), 128, 0).T
    Wh = VALS[qw] * np.repeat(np.repeat(sw.astype(np.float64), 128, 0), 128, 1)
    dYh = VALS[qdy] * np.repeat(sdy.astype(np.float64), 128, 0).T
    dYth = VALS[qdyt].T * np.repeat(sdyt.astype(np.float64), 128, 0)   # [T][Dout]
    Xth = VALS[qxt].T * np.repeat(sxt.astype(np.float64), 128, 0)      # [T][Din]

    y, sy = oracle.gemm(oracle.FPROP, qx, sx, qw, sw, T, Dout, Din)
    assert np.all(np.abs(y - Xh @ Wh.T) <= 1e-12 * sy)
    dx, sdx = oracle.gemm(oracle.DGRAD, qdy, sdy, qw, sw, T, Din, Dout)
    assert np.all(np.abs(dx - dYh @ Wh) <= 1e-12 * sdx)
    dw, sdw = oracle.gemm(oracle.WGRAD, qdyt, sdyt, qxt, sxt, Dout, Din, T)
    assert np.all(np.abs(dw - dYth.T @ Xth) <= 1e-12 * sdw)
    # and the quantized layer is close to the BF16 layer it stands for
    Xf = synth.bf16_bits_to_f32(X).astype(np.float64)
    Wf = synth.bf16_bits_to_f32(W).astype(np.float64)
    ref = Xf @ Wf.T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.05


def test_bad_arguments_rejected():
    z = np.zeros((128, 128), dtype=np.uint8)
    s = np.zeros((1, 128), dtype=np.float32)
    with pytest.raises(ValueError):
        oracle.gemm(3, z, s, z, s, 128, 128, 128)
    with pytest.raises(ValueError):
        oracle.gemm(0, z, s, z, s, 128, 128, 100)


# ---- token counts that are not a multiple of 128 ----

def _dequant_a_ragged(a, sa, K):
    """ahat[m][k] = code * sa[k/128][m] for a reduction K that may end in a partial block."""
    return VALS[a] * np.repeat(sa.astype(np.float64), 128, axis=0)[:K].T


@pytest.mark.parametrize("mode,M", [(0, 200), (1, 16), (0, 144)])
def test_gemm_ragged_tokens_fprop_dgrad(mode, M):
    """FPROP / DGRAD with M tokens not a multiple of 128 (rows are independent):
    numpy float64 matmul of the dequantized operands."""
    N, K = 256, 384
    a, sa, b, sb = _case(mode, M, N, K, seed=900 + M + mode)
    y, asum = oracle.gemm(mode, a, sa, b, sb, M, N, K)
    A = _dequant_a(a, sa)
    B = _dequant_b(mode, b, sb, N, K)
    assert y.shape == (M, N)
    assert np.all(np.abs(y - A @ B.T) <= 1e-12 * (np.abs(A) @ np.abs(B).T) + 1e-300)


@pytest.mark.parametrize("K", [16, 200, 400])
def test_gemm_ragged_reduction_wgrad(K):
    """WGRAD over K tokens not a multiple of 128: the last reduction block holds
    K mod 128 tokens and carries its own (partial-group) scales."""
    M, N = 128, 256
    rng = np.random.default_rng(K)
    KB = (K + 127) // 128
    a = _rand_codes(rng, (M, K)); sa = _rand_scales(rng, (KB, M))
    b = _rand_codes(rng, (N, K)); sb = _rand_scales(rng, (KB, N))
    y, asum = oracle.gemm(oracle.WGRAD, a, sa, b, sb, M, N, K)
    A = _dequant_a_ragged(a, sa, K)
    B = VALS[b] * np.repeat(sb.astype(np.float64), 128, axis=0)[:K].T
    assert np.all(np.abs(y - A @ B.T) <= 1e-12 * (np.abs(A) @ np.abs(B).T) + 1e-300)
    assert np.allclose(asum, np.abs(A) @ np.abs(B).T, rtol=1e-12, atol=0)


def test_gemm_ragged_wgrad_through_the_layer():
    """The layer's wgrad over 200 tokens, from the oracle's own token-wise quantizer,
    equals the same computation on the inputs zero-padded to 256 tokens."""
    T, Din, Dout = 200, 256, 128
    X = synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(200, 0), outliers=True)
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(200, 2))
    a, sa = oracle.quant_act_t(dY)
    b, sb = oracle.quant_act_t(X)
    y, _ = oracle.gemm(oracle.WGRAD, a, sa, b, sb, Dout, Din, T)
    pad = lambda v: np.concatenate([v, np.zeros((256 - T, v.shape[1]), dtype=np.uint16)])
    ap, sap = oracle.quant_act_t(pad(dY))
    bp, sbp = oracle.quant_act_t(pad(X))
    yp, _ = oracle.gemm(oracle.WGRAD, ap, sap, bp, sbp, Dout, Din, 256)
    assert np.array_equal(y, yp)


def test_gemm_ragged_bad_sizes():
    rng = np.random.default_rng(1)
    a = _rand_codes(rng, (128, 200)); sa = _rand_scales(rng, (2, 128))
    b = _rand_codes(rng, (128, 200)); sb = _rand_scales(rng, (2, 128))
    with pytest.raises(ValueError):   # FPROP reduction = features: whole blocks only
        oracle.gemm(oracle.FPROP, a, sa, b, sb, 128, 128, 200)
