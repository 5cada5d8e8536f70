"""GPU parity of fp8_gemm_blockwise (fprop / dgrad / wgrad) against the CPU oracle's
FP64 GEMM over the oracle's own quantized operands.

The GPU GEMM consumes the GPU quantizers' output; those are checked bit-exact
against the oracle's first, so both sides see the same FP8 bytes and scales."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_fp8_linear_b200 import (DGRAD, FPROP, WGRAD, fp8_gemm_blockwise,
                                       fp8_gemm_wgrad_acc32, fp8_quant_act, fp8_quant_act_t,
                                       fp8_quant_weight, synth)
from tests._gpu import bf16_dev_to_f64, check_gemm, to_dev_bf16

pytestmark = pytest.mark.gpu


def _same(gpu: torch.Tensor, ref: np.ndarray):
    g = gpu.cpu().numpy()
    if ref.dtype == np.float32:
        assert np.array_equal(g.view(np.uint32), ref.view(np.uint32))
    else:
        assert np.array_equal(g, ref)


def _layer(T, Din, Dout, seed, outliers=True):
    X = synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(seed, 0), outliers=outliers)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(seed, 1))
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(seed, 2))
    return X, W, dY


def _rows(M, n):
    """A deterministic spread of rows touching every 128-row tile (first and last
    rows of tiles included)."""
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(M)
    base = np.concatenate([np.arange(0, M, 128), np.arange(127, M, 128)])
    extra = rng.choice(M, max(0, n - base.size), replace=False)
    return np.unique(np.concatenate([base, extra]))[:max(n, base.size)]


def _run_mode(mode, X, W, dY, rows=None):
    """Quantize on both sides, check the bytes, run the GEMM, return (y, y_ref, asum)."""
    T, Din = X.shape
    Dout = W.shape[0]
    if mode == FPROP:
        a_d, sa_d = fp8_quant_act(to_dev_bf16(X))
        b_d, sb_d, _ = fp8_quant_weight(to_dev_bf16(W))
        a, sa = oracle.quant_act(X)
        b, sb, _ = oracle.quant_weight(W)
        M, N, K = T, Dout, Din
    elif mode == DGRAD:
        a_d, sa_d = fp8_quant_act(to_dev_bf16(dY))
        b_d, sb_d, _ = fp8_quant_weight(to_dev_bf16(W))
        a, sa = oracle.quant_act(dY)
        b, sb, _ = oracle.quant_weight(W)
        M, N, K = T, Din, Dout
    else:
        a_d, sa_d = fp8_quant_act_t(to_dev_bf16(dY))
        b_d, sb_d = fp8_quant_act_t(to_dev_bf16(X))
        a, sa = oracle.quant_act_t(dY)
        b, sb = oracle.quant_act_t(X)
        M, N, K = Dout, Din, T
    for g, r in ((a_d, a), (sa_d, sa), (b_d, b), (sb_d, sb)):
        _same(g, r)
    y = bf16_dev_to_f64(fp8_gemm_blockwise(mode, a_d, sa_d, b_d, sb_d, M, N, K))
    y_ref, asum = oracle.gemm(mode, a, sa, b, sb, M, N, K, rows=rows)
    if rows is not None:
        y = y[rows]
    return y, y_ref, asum


@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
@pytest.mark.parametrize("T,Din,Dout", [
    (128, 1024, 1024),   # the single-fprop workload's shape (one row-tile)
    (384, 640, 896),     # N not a multiple of 256: the 128-wide tile path, ragged grid
    (256, 1152, 768),    # 3 tiles of 256 columns, odd number of reduction blocks
    (1024, 256, 2048),   # more column tiles, short reduction
])
def test_gemm_small_full(mode, T, Din, Dout):
    X, W, dY = _layer(T, Din, Dout, seed=T + Din + Dout + mode)
    y, y_ref, asum = _run_mode(mode, X, W, dY)
    check_gemm(y, y_ref, asum, f"mode {mode} {T}x{Din}x{Dout}")


@pytest.mark.parametrize("mode,T,Din,Dout", [
    (FPROP, 384, 256, 6400), (DGRAD, 384, 6400, 256), (WGRAD, 256, 6400, 384)])
def test_gemm_single_cta_wide_tiles(mode, T, Din, Dout):
    """M = 384 (not a multiple of 256), N = 6400, K = 256: the single-CTA path with
    128 x 256 tiles (75 of them, enough to keep that width); every output checked."""
    X, W, dY = _layer(T, Din, Dout, seed=4242 + mode)
    y, y_ref, asum = _run_mode(mode, X, W, dY)
    check_gemm(y, y_ref, asum, f"mode {mode} single-CTA 128x256 tiles")


def test_gemm_single_fprop_workload():
    """X[128x1024] ~ N(0,1), W[1024x1024] ~ N(0,0.02), seed 0: Y = X W^T, checked
    on every output."""
    X = synth.normal_bf16(128, 1024, 1.0, seed=synth.seed_for(0, 0))
    W = synth.normal_bf16(1024, 1024, 0.02, seed=synth.seed_for(0, 1))
    y, y_ref, asum = _run_mode(FPROP, X, W, None)
    check_gemm(y, y_ref, asum, "single fprop")


@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_many_tiles_per_cta(mode):
    """More tiles than SMs, so each persistent CTA walks several tiles and both TMEM
    buffers wrap many times; rows sampled across every row-tile."""
    T, Din, Dout = 2048, 1024, 3072
    X, W, dY = _layer(T, Din, Dout, seed=77 + mode)
    M = {FPROP: T, DGRAD: T, WGRAD: Dout}[mode]
    rows = _rows(M, 64)
    y, y_ref, asum = _run_mode(mode, X, W, dY, rows=rows)
    check_gemm(y, y_ref, asum, f"mode {mode} many tiles")


# Qwen3-1.7B linear shapes at M = 8192 tokens: (tokens, in, out)
FULL = {
    "qkv": (8192, 2048, 4096),
    "o": (8192, 2048, 2048),
    "gate_up": (8192, 2048, 12288),
    "down": (8192, 6144, 2048),
}


@pytest.mark.parametrize("name", list(FULL))
@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_full_size_sampled(name, mode):
    T, Din, Dout = FULL[name]
    X, W, dY = _layer(T, Din, Dout, seed=hash(name) % 1000 + 10 * mode)
    M = {FPROP: T, DGRAD: T, WGRAD: Dout}[mode]
    rows = _rows(M, 24)
    y, y_ref, asum = _run_mode(mode, X, W, dY, rows=rows)
    check_gemm(y, y_ref, asum, f"{name} mode {mode}")


# The MLP backward workload taken literally: one 6144-wide gate (or up) weight, so
# dgrad reduces over 6144 into dX[8192][2048] and wgrad gives dW[6144][2048] over 8192
# tokens (the down projection's dgrad and wgrad are the "down" rows above).
MLP_BWD = {"gate": (8192, 2048, 6144)}


@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_mlp_backward_shapes_sampled(mode):
    T, Din, Dout = MLP_BWD["gate"]
    X, W, dY = _layer(T, Din, Dout, seed=613 + mode)
    M = {FPROP: T, DGRAD: T, WGRAD: Dout}[mode]
    rows = _rows(M, 24)
    y, y_ref, asum = _run_mode(mode, X, W, dY, rows=rows)
    check_gemm(y, y_ref, asum, f"gate 6144 mode {mode}")


# The micro-batch sweep of a 28-layer step runs the same four linears at M = 4096, 16384
# and 32768 tokens (micro-batch 1, 4, 8 x sequence 4096): every linear at the smallest,
# one linear at each of the larger sizes (the wgrad reduction grows to 32768 tokens).
SWEEP = [(4096, name) for name in FULL] + [(16384, "qkv"), (32768, "down")]


@pytest.mark.parametrize("T,name", SWEEP)
@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_sweep_sizes_sampled(T, name, mode):
    _, Din, Dout = FULL[name]
    X, W, dY = _layer(T, Din, Dout, seed=T // 128 + 7 * mode + len(name))
    M = {FPROP: T, DGRAD: T, WGRAD: Dout}[mode]
    rows = _rows(M, 16)
    y, y_ref, asum = _run_mode(mode, X, W, dY, rows=rows)
    check_gemm(y, y_ref, asum, f"{name} mode {mode} M={T}")


@pytest.mark.parametrize("mode", [FPROP, DGRAD, WGRAD])
def test_gemm_zero_and_degenerate_inputs(mode):
    """All-zero activations give an exactly zero output; a single nonzero group
    gives a rank-one result the oracle reproduces."""
    T, Din, Dout = 256, 384, 512
    X, W, dY = _layer(T, Din, Dout, seed=5)
    Xz = np.zeros_like(X)
    dYz = np.zeros_like(dY)
    y, y_ref, asum = _run_mode(mode, Xz, W, dYz)
    assert np.all(y == 0) and np.all(y_ref == 0)
    X1 = Xz.copy(); X1[3, 128:256] = X[3, 128:256]
    dY1 = dYz.copy(); dY1[3, :128] = dY[3, :128]
    y, y_ref, asum = _run_mode(mode, X1, W, dY1)
    check_gemm(y, y_ref, asum, f"mode {mode} one group")


def test_gemm_deterministic():
    X, W, dY = _layer(1024, 2048, 2048, seed=9)
    qx, sx = fp8_quant_act(to_dev_bf16(X))
    qw, sw, _ = fp8_quant_weight(to_dev_bf16(W))
    y1 = fp8_gemm_blockwise(FPROP, qx, sx, qw, sw, 1024, 2048, 2048)
    y2 = fp8_gemm_blockwise(FPROP, qx, sx, qw, sw, 1024, 2048, 2048)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("T,Din,Dout", [
    (256, 384, 640),      # single-CTA path, N not a multiple of 256
    (1024, 768, 512),     # single-CTA path, 128x256 tiles
    (8192, 2048, 4096),   # CTA-pair path (the QKV weight gradient), rows sampled
])
def test_wgrad_fp32_accumulation(T, Din, Dout):
    """dW32 += wgrad sum in FP32 (gradient accumulation in FP32): starting from a
    seeded FP32 buffer, one call adds the oracle's sum, a second call adds it again."""
    X, W, dY = _layer(T, Din, Dout, seed=T + Din + Dout + 31)
    a_d, sa_d = fp8_quant_act_t(to_dev_bf16(dY))
    b_d, sb_d = fp8_quant_act_t(to_dev_bf16(X))
    a, sa = oracle.quant_act_t(dY)
    b, sb = oracle.quant_act_t(X)
    for g, r in ((a_d, a), (sa_d, sa), (b_d, b), (sb_d, sb)):
        _same(g, r)
    M, N, K = Dout, Din, T
    rows = _rows(M, 24) if M * N > 4 * 1024 * 1024 else None
    rng = np.random.default_rng(7)
    prev = (rng.standard_normal((M, N)) * 1e-3).astype(np.float32)
    dw = torch.from_numpy(prev.copy()).cuda()
    fp8_gemm_wgrad_acc32(a_d, sa_d, b_d, sb_d, M, N, K, dw)
    y1 = dw.cpu().numpy().astype(np.float64)
    fp8_gemm_wgrad_acc32(a_d, sa_d, b_d, sb_d, M, N, K, dw)
    y2 = dw.cpu().numpy().astype(np.float64)
    y_ref, asum = oracle.gemm(WGRAD, a, sa, b, sb, M, N, K, rows=rows)
    p64 = prev.astype(np.float64)
    if rows is not None:
        y1, y2, p64 = y1[rows], y2[rows], p64[rows]
    check_gemm(y1, p64 + y_ref, asum + np.abs(p64), "acc32 once")
    check_gemm(y2, p64 + 2 * y_ref, 2 * asum + np.abs(p64), "acc32 twice")



@pytest.mark.parametrize("T,Din,Dout", [
    (256, 384, 640),      # single-CTA path (vector atomic adds)
    (8192, 2048, 4096),   # CTA-pair path (TMA reduce-add), rows sampled
])
def test_wgrad_fp32_accumulation_overlapping_calls(T, Din, Dout):
    """Two fp8_gemm_wgrad_acc32 calls on two streams, free to overlap on the GPU, into
    one FP32 buffer: both sums must land (prev + 2 * sum), only their order may vary."""
    X, W, dY = _layer(T, Din, Dout, seed=T + Din + Dout + 57)
    a_d, sa_d = fp8_quant_act_t(to_dev_bf16(dY))
    b_d, sb_d = fp8_quant_act_t(to_dev_bf16(X))
    a, sa = oracle.quant_act_t(dY)
    b, sb = oracle.quant_act_t(X)
    M, N, K = Dout, Din, T
    rows = _rows(M, 24) if M * N > 4 * 1024 * 1024 else None
    rng = np.random.default_rng(11)
    prev = (rng.standard_normal((M, N)) * 1e-3).astype(np.float32)
    dw = torch.from_numpy(prev.copy()).cuda()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    start = torch.cuda.Event()
    start.record()
    for st in (s1, s2):
        st.wait_event(start)
        fp8_gemm_wgrad_acc32(a_d, sa_d, b_d, sb_d, M, N, K, dw, stream=st)
    torch.cuda.synchronize()
    y2 = dw.cpu().numpy().astype(np.float64)
    y_ref, asum = oracle.gemm(WGRAD, a, sa, b, sb, M, N, K, rows=rows)
    p64 = prev.astype(np.float64)
    if rows is not None:
        y2, p64 = y2[rows], p64[rows]
    check_gemm(y2, p64 + 2 * y_ref, 2 * asum + np.abs(p64), "acc32 on two streams")
