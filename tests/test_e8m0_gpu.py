"""GPU parity of the power-of-two (E8M0) scale path against the CPU oracle.

Quantizers: FP8 codes and E8M0 scale codes bit-exact.  GEMM: the block-scaled MMA
result against the oracle's FP64 GEMM over the same dequantized operands (the scales
2^e are exact in FP32), with the tolerance of the FP32-scale GEMM."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_fp8_linear_b200 import (DGRAD, FPROP, WGRAD, fp8_gemm_blockwise_e8m0,
                                       fp8_quant_act_dual_e8m0, fp8_quant_act_e8m0,
                                       fp8_quant_act_t_e8m0, fp8_quant_weight_e8m0, synth)
from tests._gpu import bf16_dev_to_f64, check_gemm, to_dev_bf16

pytestmark = pytest.mark.gpu


def _blocks(codes_rk: np.ndarray) -> np.ndarray:
    """Compact E8M0 codes [rows][K/128] -> the tensor-core scale blocks
    [rows/128][(K/128)*512]: row r's code at bytes 16 (r % 32) + 4 (r / 32) .. +3."""
    R, KB = codes_rk.shape
    out = np.zeros((R // 128, KB, 512), dtype=np.uint8)
    r = np.arange(128)
    off = (r % 32) * 16 + (r // 32) * 4
    for rb in range(R // 128):
        c = codes_rk[rb * 128:(rb + 1) * 128, :]          # [128][KB]
        for j in range(4):
            out[rb][:, off + j] = c.T
    return out.reshape(R // 128, KB * 512)


def _wblocks(codes_nk: np.ndarray) -> np.ndarray:
    """Weight codes [N/128][K/128] -> blocks with every byte the block's code."""
    NB, KB = codes_nk.shape
    return np.repeat(codes_nk[:, :, None], 512, axis=2).reshape(NB, KB * 512)


def _eq(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = gpu.cpu().numpy()
    if not np.array_equal(g, ref):
        bad = np.argwhere(g != ref)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: gpu={g[i]:#x} ref={ref[i]:#x}")


SHAPES = [(128, 1024), (384, 640), (256, 128), (8192, 2048), (8192, 6144)]


@pytest.mark.parametrize("M,K", SHAPES)
def test_quant_e8m0_all_layouts(M, K):
    x = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(40, M + K), outliers=True)
    xd = to_dev_bf16(x)
    q, s = fp8_quant_act_e8m0(xd)
    qr, sr = oracle.quant_act_e8m0(x)
    _eq(q, qr, "row codes"); _eq(s, _blocks(sr.T), "row scales")
    qt, st = fp8_quant_act_t_e8m0(xd)
    qtr, str_ = oracle.quant_act_t_e8m0(x)
    _eq(qt, qtr, "token codes"); _eq(st, _blocks(str_.T), "token scales")
    q2, s2, qt2, st2 = fp8_quant_act_dual_e8m0(xd)
    _eq(q2, qr, "dual row codes"); _eq(s2, _blocks(sr.T), "dual row scales")
    _eq(qt2, qtr, "dual token codes"); _eq(st2, _blocks(str_.T), "dual token scales")


@pytest.mark.parametrize("N,K,want_t", [(1024, 1024, True), (4096, 2048, False), (2048, 6144, True)])
def test_quant_weight_e8m0(N, K, want_t):
    w = synth.normal_bf16(N, K, 0.02, seed=synth.seed_for(41, N + K))
    q, s, qt = fp8_quant_weight_e8m0(to_dev_bf16(w), want_t=want_t)
    qr, sr, qtr = oracle.quant_weight_e8m0(w, want_t=want_t)
    _eq(q, qr, "codes"); _eq(s, _wblocks(sr), "scales")
    if want_t:
        _eq(qt, qtr, "transposed codes")


def test_quant_e8m0_edge_cases():
    """Zero groups, signed zeros, BF16 subnormals (scale clamped at 2^-127), values near
    the BF16 maximum, and every positive finite BF16 amax with values below it."""
    rng = np.random.default_rng(5)
    x = synth.f64_to_bf16_bits(rng.standard_normal((256, 384)))
    x[0, :] = 0
    x[1, :] = 0x8000
    x[2, :] = rng.integers(1, 0x0080, 384)
    x[3, :] = rng.integers(0x8001, 0x8080, 384)
    x[4, :] = rng.integers(0x7E00, 0x7F7F, 384)
    x[5, ::2] = 0x8000
    x[6, :] = synth.f64_to_bf16_bits(rng.standard_normal(384) * 2.0 ** -126)
    x = x.astype(np.uint16)
    for arr in (x, np.ascontiguousarray(x.T)):
        q, s, qt, st = fp8_quant_act_dual_e8m0(to_dev_bf16(arr))
        qr, sr = oracle.quant_act_e8m0(arr)
        qtr, str_ = oracle.quant_act_t_e8m0(arr)
        _eq(q, qr, "codes"); _eq(s, _blocks(sr.T), "scales")
        _eq(qt, qtr, "t codes"); _eq(st, _blocks(str_.T), "t scales")
        qw, sw, qwt = fp8_quant_weight_e8m0(to_dev_bf16(arr), want_t=True)
        qwr, swr, qwtr = oracle.quant_weight_e8m0(arr, want_t=True)
        _eq(qw, qwr, "w codes"); _eq(sw, _wblocks(swr), "w scales"); _eq(qwt, qwtr, "w t codes")
    amax = np.arange(1, 0x7F80, dtype=np.int64)
    j = np.arange(1, 128, dtype=np.int64)
    grp = np.concatenate([amax[:, None], np.maximum(amax[:, None] - 3 * j[None, :], 0) |
                          ((j % 2) << 15)[None, :]], axis=1).astype(np.uint16)
    pad = (-grp.shape[0]) % 128
    grp = np.concatenate([grp, np.zeros((pad, 128), dtype=np.uint16)])
    q, s = fp8_quant_act_e8m0(to_dev_bf16(grp))
    qr, sr = oracle.quant_act_e8m0(grp)
    _eq(q, qr, "sweep codes"); _eq(s, _blocks(sr.T), "sweep scales")


def _layer(T, Din, Dout, seed):
    X = synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(seed, 0), outliers=True)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(seed, 1))
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(seed, 2))
    return X, W, dY


def _rows(M, n):
    if M <= n:
        return None
    base = np.concatenate([np.arange(0, M, 128), np.arange(127, M, 128)])
    extra = np.random.default_rng(M).choice(M, n, replace=False)
    return np.unique(np.concatenate([base, extra]))


def _run(mode, X, W, dY, sample=None):
    T, Din = X.shape
    Dout = W.shape[0]
    if mode == FPROP:
        a_d, sa_d = fp8_quant_act_e8m0(to_dev_bf16(X)); b_d, sb_d, _ = fp8_quant_weight_e8m0(to_dev_bf16(W))
        a, sa = oracle.quant_act_e8m0(X); b, sb, _ = oracle.quant_weight_e8m0(W)
        M, N, K = T, Dout, Din
    elif mode == DGRAD:
        a_d, sa_d = fp8_quant_act_e8m0(to_dev_bf16(dY)); b_d, sb_d, _ = fp8_quant_weight_e8m0(to_dev_bf16(W))
        a, sa = oracle.quant_act_e8m0(dY); b, sb, _ = oracle.quant_weight_e8m0(W)
        M, N, K = T, Din, Dout
    else:
        a_d, sa_d = fp8_quant_act_t_e8m0(to_dev_bf16(dY)); b_d, sb_d = fp8_quant_act_t_e8m0(to_dev_bf16(X))
        a, sa = oracle.quant_act_t_e8m0(dY); b, sb = oracle.quant_act_t_e8m0(X)
        M, N, K = Dout, Din, T
    sa_blk = _blocks(sa.T)
    sb_blk = _wblocks(sb) if mode != WGRAD else _blocks(sb.T)
    for g, r, w in ((a_d, a, "a"), (sa_d, sa_blk, "sa"), (b_d, b, "b"), (sb_d, sb_blk, "sb")):
        _eq(g, r, w)
    y = bf16_dev_to_f64(fp8_gemm_blockwise_e8m0(mode, a_d, sa_d, b_d, sb_d, M, N, K))
    rows = _rows(M, sample) if sample else None
    y_ref, asum = oracle.gemm(mode, a, oracle.e8m0_to_float(sa), b, oracle.e8m0_to_float(sb),
                              M, N, K, rows=rows)
    if rows is not None:
        y = y[rows]
    return y, y_ref, asum


@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
@pytest.mark.parametrize("T,Din,Dout", [
    (128, 1024, 1024),    # one row-tile: single-CTA path
    (384, 640, 896),      # N not a multiple of 256: single-CTA path, ragged grid
    (1024, 1024, 2048),   # CTA pairs (16+ tiles of 256 x 256)
    (2048, 1536, 1024),   # CTA pairs, 12-block reductions in fprop
    (256, 512, 17152),    # dgrad reduction of 134 blocks: weight codes read in chunks of 128
])
def test_gemm_e8m0_small_full(mode, T, Din, Dout):
    X, W, dY = _layer(T, Din, Dout, seed=T + Din + Dout + 7 * mode)
    y, y_ref, asum = _run(mode, X, W, dY)
    check_gemm(y, y_ref, asum, f"e8m0 mode {mode} {T}x{Din}x{Dout}")


# gate: the MLP backward workload taken literally (one 6144-wide gate weight: dgrad
# reduces over 6144, wgrad gives dW[6144][2048] over 8192 tokens)
FULL = {"qkv": (8192, 2048, 4096), "gate_up": (8192, 2048, 12288), "down": (8192, 6144, 2048),
        "gate": (8192, 2048, 6144)}


@pytest.mark.parametrize("name", list(FULL))
@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_e8m0_full_size_sampled(name, mode):
    T, Din, Dout = FULL[name]
    X, W, dY = _layer(T, Din, Dout, seed=len(name) * 31 + mode)
    y, y_ref, asum = _run(mode, X, W, dY, sample=16)
    check_gemm(y, y_ref, asum, f"e8m0 {name} mode {mode}")


@pytest.mark.parametrize("mode", [FPROP, WGRAD])
def test_gemm_e8m0_zero_and_deterministic(mode):
    T, Din, Dout = 1024, 1024, 1024
    X, W, dY = _layer(T, Din, Dout, seed=3)
    Xz = np.zeros_like(X); dYz = np.zeros_like(dY)
    y, y_ref, _ = _run(mode, Xz, W, dYz)
    assert np.all(y == 0) and np.all(y_ref == 0)
    a, sa = fp8_quant_act_t_e8m0(to_dev_bf16(dY)) if mode == WGRAD else fp8_quant_act_e8m0(to_dev_bf16(X))
    if mode == WGRAD:
        b, sb = fp8_quant_act_t_e8m0(to_dev_bf16(X)); M, N, K = Dout, Din, T
    else:
        b, sb, _ = fp8_quant_weight_e8m0(to_dev_bf16(W)); M, N, K = T, Dout, Din
    y1 = fp8_gemm_blockwise_e8m0(mode, a, sa, b, sb, M, N, K)
    y2 = fp8_gemm_blockwise_e8m0(mode, a, sa, b, sb, M, N, K)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_e8m0_sweep_size_sampled(mode):
    """The largest micro-batch of the sweep (M = 32768 tokens): the wgrad reduction runs
    over 256 blocks of 128 tokens in one accumulator."""
    T, Din, Dout = 32768, 6144, 2048
    X, W, dY = _layer(T, Din, Dout, seed=90 + mode)
    y, y_ref, asum = _run(mode, X, W, dY, sample=8)
    check_gemm(y, y_ref, asum, f"e8m0 down M=32768 mode {mode}")
