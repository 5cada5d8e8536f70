"""GPU parity of the three quantizers against the CPU oracle: bit-exact FP8 codes and
FP32 scales, at small ragged sizes, at the full Qwen3-1.7B layer sizes, on edge
cases, and exhaustively over every (BF16 amax, BF16 value) pair that can change a
code."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_fp8_linear_b200 import (fp8_quant_act, fp8_quant_act_dual, fp8_quant_act_t,
                                       fp8_quant_weight, synth)
from tests._gpu import to_dev_bf16

pytestmark = pytest.mark.gpu


def _eq_bits(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = gpu.cpu().numpy()
    if ref.dtype == np.float32:
        g, ref = g.view(np.uint32), ref.view(np.uint32)
    if not np.array_equal(g, ref):
        bad = np.argwhere(g != ref)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: gpu={g[i]:#x} ref={ref[i]:#x}")


# (16384, 2048): the activation shape of a 16k-token batch at model width 2048
ACT_SHAPES = [(128, 1024), (384, 640), (256, 128), (8192, 2048), (16384, 2048), (8192, 6144),
              (32768, 2048)]


@pytest.mark.parametrize("M,K", ACT_SHAPES)
def test_quant_act_parity(M, K):
    x = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(1, M + K), outliers=True)
    q, s = fp8_quant_act(to_dev_bf16(x))
    qr, sr = oracle.quant_act(x)
    _eq_bits(q, qr, "codes")
    _eq_bits(s, sr, "scales")


@pytest.mark.parametrize("M,K", ACT_SHAPES)
def test_quant_act_t_parity(M, K):
    x = synth.normal_bf16(M, K, 1e-3, seed=synth.seed_for(3, M + K))
    qt, st = fp8_quant_act_t(to_dev_bf16(x))
    qr, sr = oracle.quant_act_t(x)
    _eq_bits(qt, qr, "codes")
    _eq_bits(st, sr, "scales")


@pytest.mark.parametrize("M,K", ACT_SHAPES)
def test_quant_act_dual_parity(M, K):
    """One read, both layouts: each bit-identical to the oracle's own quantizer."""
    x = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(4, M + K), outliers=True)
    q, s, qt, st = fp8_quant_act_dual(to_dev_bf16(x))
    qr, sr = oracle.quant_act(x)
    qtr, str_ = oracle.quant_act_t(x)
    _eq_bits(q, qr, "row codes")
    _eq_bits(s, sr, "row scales")
    _eq_bits(qt, qtr, "token codes")
    _eq_bits(st, str_, "token scales")


@pytest.mark.parametrize("N,K,want_t", [(1024, 1024, False), (384, 640, True), (4096, 2048, True),
                                        (12288, 2048, False), (2048, 6144, True)])
def test_quant_weight_parity(N, K, want_t):
    w = synth.normal_bf16(N, K, 0.02, seed=synth.seed_for(2, N + K))
    q, s, qt = fp8_quant_weight(to_dev_bf16(w), want_t=want_t)
    qr, sr, qtr = oracle.quant_weight(w, want_t=want_t)
    _eq_bits(q, qr, "codes")
    _eq_bits(s, sr, "scales")
    if want_t:
        _eq_bits(qt, qtr, "transposed codes")


def _edge_tensor(M, K, seed):
    """Rows / blocks exercising the degenerate cases: all-zero groups, signed zeros,
    a single nonzero value, BF16 subnormals (subnormal FP32 scales), values near
    the BF16 maximum, and groups with a huge dynamic range."""
    rng = np.random.default_rng(seed)
    x = synth.f64_to_bf16_bits(rng.standard_normal((M, K)))
    x[0, :] = 0                                       # all zero
    x[1, :] = 0x8000                                  # all -0
    x[2, :] = 0; x[2, 5] = synth.f64_to_bf16_bits(np.array([-3.0]))[0]
    x[3, :] = rng.integers(1, 0x0080, K)              # positive BF16 subnormals
    x[4, :] = rng.integers(0x8001, 0x8080, K)         # negative BF16 subnormals
    x[5, :] = rng.integers(0x7E00, 0x7F7F, K)         # near the BF16 maximum
    x[6, :] = (rng.integers(0, 0x7F7F, K) | (rng.integers(0, 2, K) << 15)).astype(np.uint16)
    x[7, ::2] = 0x8000                                # -0 inside nonzero groups
    x[8, :] = synth.f64_to_bf16_bits(rng.standard_normal(K) * 2.0 ** -120)
    x[9, :] = synth.f64_to_bf16_bits(rng.standard_normal(K) * 2.0 ** 100)
    return x.astype(np.uint16)


def test_quant_edge_cases_all_layouts():
    x = _edge_tensor(256, 384, seed=17)
    q, s = fp8_quant_act(to_dev_bf16(x))
    qr, sr = oracle.quant_act(x)
    _eq_bits(q, qr, "act codes"); _eq_bits(s, sr, "act scales")
    xt = np.ascontiguousarray(x.T)  # puts the special rows into token-dim groups
    qt, st = fp8_quant_act_t(to_dev_bf16(xt))
    qtr, str_ = oracle.quant_act_t(xt)
    _eq_bits(qt, qtr, "act_t codes"); _eq_bits(st, str_, "act_t scales")
    for arr in (x, xt):
        a = np.ascontiguousarray(arr)
        q, s, qt, st = fp8_quant_act_dual(to_dev_bf16(a))
        qr, sr = oracle.quant_act(a)
        qtr, str_ = oracle.quant_act_t(a)
        _eq_bits(q, qr, "dual row codes"); _eq_bits(s, sr, "dual row scales")
        _eq_bits(qt, qtr, "dual token codes"); _eq_bits(st, str_, "dual token scales")
    for blk in (x, xt):
        w = np.ascontiguousarray(blk)
        q, s, qt = fp8_quant_weight(to_dev_bf16(w), want_t=True)
        qr, sr, qtr = oracle.quant_weight(w, want_t=True)
        _eq_bits(q, qr, "weight codes"); _eq_bits(s, sr, "weight scales")
        _eq_bits(qt, qtr, "weight transposed codes")
    # a weight made of single special blocks
    w = np.zeros((256, 256), dtype=np.uint16)
    w[128:, :128] = 0x8000
    w[:128, 128:] = 1
    w[128:, 128:] = 0x7F7F
    q, s, _ = fp8_quant_weight(to_dev_bf16(w))
    qr, sr, _ = oracle.quant_weight(w)
    _eq_bits(q, qr, "special-block codes"); _eq_bits(s, sr, "special-block scales")


def test_quant_division_exhaustive():
    """For every positive finite BF16 amax and the 2540 BF16 magnitudes just below it
    (the twenty binades where the quotient can still round to a nonzero E4M3 code),
    with both signs, the GPU codes equal the oracle's."""
    amax = np.arange(1, 0x7F80, dtype=np.int64)             # positive finite BF16
    G, J = 20, 127
    j = np.arange(1, J + 1, dtype=np.int64)
    rows = []
    for g in range(G):
        xb = amax[:, None] - (g * J + j)[None, :]
        xb = np.maximum(xb, 0)
        sign = ((j % 2) << 15)[None, :]
        grp = np.concatenate([amax[:, None], xb | sign], axis=1)
        rows.append(grp.astype(np.uint16))
    x = np.concatenate(rows, axis=0)
    pad = (-x.shape[0]) % 128
    x = np.concatenate([x, np.zeros((pad, 128), dtype=np.uint16)], axis=0)
    step = 1 << 17
    for r0 in range(0, x.shape[0], step):
        blk = np.ascontiguousarray(x[r0:r0 + step])
        q, s = fp8_quant_act(to_dev_bf16(blk))
        qr, sr = oracle.quant_act(blk)
        _eq_bits(q, qr, f"codes rows {r0}+")
        _eq_bits(s, sr, f"scales rows {r0}+")


def test_quant_repeatable_and_stream_ordered():
    x = synth.normal_bf16(1024, 2048, 1.0, seed=99, outliers=True)
    xd = to_dev_bf16(x)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        q1, s1 = fp8_quant_act(xd)
    side.synchronize()
    q2, s2 = fp8_quant_act(xd)
    assert torch.equal(q1, q2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))
