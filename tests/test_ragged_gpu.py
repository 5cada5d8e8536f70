"""GPU parity for token counts that are not a multiple of 128 (the last token group
partial, reading R17 of the oracle): the activation quantizers at ragged M, FPROP
and DGRAD with ragged M (single-CTA path), WGRAD and the FP32 main-grad wgrad with
a ragged reduction (single-CTA and CTA-pair paths).  Codes and scales bit-exact,
GEMMs within the usual tolerance, and every output written through a view of a
larger buffer whose tail must come back untouched (no store past the end)."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_fp8_linear_b200 import (DGRAD, FPROP, WGRAD, fp8_gemm_blockwise,
                                       fp8_gemm_wgrad_acc32, fp8_quant_act, fp8_quant_act_dual,
                                       fp8_quant_act_t, fp8_quant_weight, fp8bw_last_device_error,
                                       synth)
from tests._gpu import bf16_dev_to_f64, check_gemm, to_dev_bf16

pytestmark = pytest.mark.gpu

SENTINEL = 0x5A


def _guarded(shape, dtype):
    """A contiguous tensor of `shape` at the start of a larger buffer, plus the tail to
    check afterwards (filled with a sentinel byte pattern)."""
    n = int(np.prod(shape))
    itemsize = torch.empty(0, dtype=dtype).element_size()
    raw = torch.full(((n + 4096) * itemsize,), SENTINEL, dtype=torch.uint8, device="cuda")
    view = raw[: n * itemsize].view(dtype).view(*shape)
    return view, raw[n * itemsize:]


def _untouched(tail, what):
    assert bool((tail == SENTINEL).all()), f"{what}: bytes written past the end of the buffer"


def _same(gpu, ref, what):
    g = gpu.cpu().numpy()
    r = np.ascontiguousarray(ref)
    if r.dtype == np.float32:
        assert np.array_equal(g.view(np.uint32), r.view(np.uint32)), what
    else:
        assert np.array_equal(g, r), what


@pytest.mark.parametrize("M,K", [(16, 128), (144, 384), (1040, 256), (8208, 2048)])
def test_quantizers_ragged_tokens(M, K):
    X = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(M, K), outliers=True)
    xd = to_dev_bf16(X)
    q_ref, s_ref = oracle.quant_act(X)
    qt_ref, st_ref = oracle.quant_act_t(X)
    G = (M + 127) // 128
    q, q_tail = _guarded((M, K), torch.uint8)
    s, s_tail = _guarded((K // 128, M), torch.float32)
    qt, qt_tail = _guarded((K, M), torch.uint8)
    st, st_tail = _guarded((G, K), torch.float32)
    fp8_quant_act(xd, q=q, s=s)
    fp8_quant_act_t(xd, qt=qt, st=st)
    torch.cuda.synchronize()
    _same(q, q_ref, "act codes"); _same(s, s_ref, "act scales")
    _same(qt, qt_ref, "act_t codes"); _same(st, st_ref, "act_t scales")
    for t, w in ((q_tail, "q"), (s_tail, "s"), (qt_tail, "qt"), (st_tail, "st")):
        _untouched(t, w)
    q2, q2_tail = _guarded((M, K), torch.uint8)
    qt2, qt2_tail = _guarded((K, M), torch.uint8)
    s2 = torch.empty(K // 128, M, dtype=torch.float32, device="cuda")
    st2 = torch.empty(G, K, dtype=torch.float32, device="cuda")
    fp8_quant_act_dual(xd, q=q2, s=s2, qt=qt2, st=st2)
    torch.cuda.synchronize()
    _same(q2, q_ref, "dual codes"); _same(s2, s_ref, "dual scales")
    _same(qt2, qt_ref, "dual t codes"); _same(st2, st_ref, "dual t scales")
    _untouched(q2_tail, "dual q"); _untouched(qt2_tail, "dual qt")
    assert fp8bw_last_device_error() == 0


def _layer(T, Din, Dout, seed):
    X = synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(seed, 0), outliers=True)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(seed, 1))
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(seed, 2))
    return X, W, dY


@pytest.mark.parametrize("T,Din,Dout", [
    (144, 512, 768),     # 2 row tiles, the second with 16 rows; 128x256 tiles would leave
                         # most SMs idle, so 128x128 tiles
    (1040, 256, 6400),   # 9 row tiles, last 16 rows; fprop with 128x256 tiles
    (16, 1024, 256),     # a single, 16-row tile
])
def test_fprop_dgrad_ragged_tokens(T, Din, Dout):
    X, W, dY = _layer(T, Din, Dout, seed=T + Din)
    qw, sw, _ = fp8_quant_weight(to_dev_bf16(W))
    qwr, swr, _ = oracle.quant_weight(W)
    for mode, src, N, K in ((FPROP, X, Dout, Din), (DGRAD, dY, Din, Dout)):
        a, sa = fp8_quant_act(to_dev_bf16(src))
        ar, sar = oracle.quant_act(src)
        _same(a, ar, "codes"); _same(sa, sar, "scales")
        out, tail = _guarded((T, N), torch.bfloat16)
        fp8_gemm_blockwise(mode, a, sa, qw, sw, T, N, K, out=out)
        torch.cuda.synchronize()
        _untouched(tail, f"mode {mode} output")
        y_ref, asum = oracle.gemm(mode, ar, sar, qwr, swr, T, N, K)
        check_gemm(bf16_dev_to_f64(out), y_ref, asum, f"mode {mode} T={T}")
    assert fp8bw_last_device_error() == 0


@pytest.mark.parametrize("T,Din,Dout", [
    (1040, 512, 384),    # single-CTA path, 9 reduction blocks, the last of 16 tokens
    (1040, 2048, 2048),  # CTA-pair path (64 pair tiles)
    (144, 640, 256),     # 128-wide tiles (N = 640), 2 reduction blocks
])
def test_wgrad_ragged_reduction(T, Din, Dout):
    X, W, dY = _layer(T, Din, Dout, seed=7 * T + Dout)
    a, sa = fp8_quant_act_t(to_dev_bf16(dY))
    b, sb = fp8_quant_act_t(to_dev_bf16(X))
    ar, sar = oracle.quant_act_t(dY)
    br, sbr = oracle.quant_act_t(X)
    for g, r in ((a, ar), (sa, sar), (b, br), (sb, sbr)):
        _same(g, r, "wgrad operands")
    y = bf16_dev_to_f64(fp8_gemm_blockwise(WGRAD, a, sa, b, sb, Dout, Din, T))
    y_ref, asum = oracle.gemm(WGRAD, ar, sar, br, sbr, Dout, Din, T)
    check_gemm(y, y_ref, asum, f"wgrad T={T}")
    # FP32 main grad over the same ragged reduction: prev + sum, then + sum again
    prev = (np.random.default_rng(T).standard_normal((Dout, Din)) * 1e-3).astype(np.float32)
    dw32 = torch.from_numpy(prev.copy()).cuda()
    fp8_gemm_wgrad_acc32(a, sa, b, sb, Dout, Din, T, dw32)
    y1 = dw32.cpu().numpy().astype(np.float64)
    fp8_gemm_wgrad_acc32(a, sa, b, sb, Dout, Din, T, dw32)
    y2 = dw32.cpu().numpy().astype(np.float64)
    p64 = prev.astype(np.float64)
    check_gemm(y1, p64 + y_ref, asum + np.abs(p64), "acc32 ragged once")
    check_gemm(y2, p64 + 2 * y_ref, 2 * asum + np.abs(p64), "acc32 ragged twice")
    assert fp8bw_last_device_error() == 0
