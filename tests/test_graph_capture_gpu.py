"""The library's calls can be captured in a CUDA graph: they only enqueue work on the
caller's stream (no synchronization, no allocation), so a layer captured once replays
with no host work per kernel.  One fprop layer (both quantizers and the GEMM, also
with the weight quantizer forked onto a second stream and joined before the GEMM) and
one training linear (dual quantizer of dY, dgrad and wgrad) are captured into static
buffers; replays must give the eager results bit for bit, also after the captured
input buffers receive new values."""
import pytest
import torch

from blockwise_fp8_linear_b200 import (DGRAD, FPROP, WGRAD, fp8_gemm_blockwise, fp8_quant_act,
                                       fp8_quant_act_dual, fp8_quant_weight,
                                       fp8bw_last_device_error, synth)
from tests._gpu import to_dev_bf16

pytestmark = pytest.mark.gpu


def _capture(fn):
    """Warm `fn` up on a side stream, then capture it (torch's recommended sequence)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        fn()
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("fork", [False, True])
@pytest.mark.parametrize("T,Din,Dout", [(128, 1024, 1024), (1024, 2048, 4096)])
def test_fprop_layer_replays_from_a_graph(T, Din, Dout, fork):
    X = to_dev_bf16(synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(T, 20), outliers=True))
    W = to_dev_bf16(synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(T, 21)))
    qx = torch.empty(T, Din, dtype=torch.uint8, device="cuda")
    sx = torch.empty(Din // 128, T, dtype=torch.float32, device="cuda")
    qw = torch.empty(Dout, Din, dtype=torch.uint8, device="cuda")
    sw = torch.empty(Dout // 128, Din // 128, dtype=torch.float32, device="cuda")
    Y = torch.empty(T, Dout, dtype=torch.bfloat16, device="cuda")

    branch = torch.cuda.Stream()

    def layer():
        if fork:  # the weight quantizer on a second stream, joined before the GEMM
            main = torch.cuda.current_stream()
            branch.wait_stream(main)
            with torch.cuda.stream(branch):
                fp8_quant_weight(W, q=qw, s=sw)
            fp8_quant_act(X, qx, sx)
            main.wait_stream(branch)
        else:
            fp8_quant_act(X, qx, sx)
            fp8_quant_weight(W, q=qw, s=sw)
        fp8_gemm_blockwise(FPROP, qx, sx, qw, sw, T, Dout, Din, out=Y)

    g = _capture(layer)
    for round_ in range(2):
        if round_:  # new values in the captured input buffers
            X.copy_(to_dev_bf16(synth.normal_bf16(T, Din, 3.0, seed=synth.seed_for(T, 22))))
            W.copy_(to_dev_bf16(synth.normal_bf16(Dout, Din, 0.05, seed=synth.seed_for(T, 23))))
        for t in (qx, sx, qw, sw, Y):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        eq, es = fp8_quant_act(X)
        ew, ews, _ = fp8_quant_weight(W)
        ey = fp8_gemm_blockwise(FPROP, eq, es, ew, ews, T, Dout, Din)
        torch.cuda.synchronize()
        assert torch.equal(qx, eq) and torch.equal(sx, es)
        assert torch.equal(qw, ew) and torch.equal(sw, ews)
        assert torch.equal(Y, ey)
    assert fp8bw_last_device_error() == 0


def test_backward_linear_replays_from_a_graph():
    T, Din, Dout = 1024, 2048, 2048
    X = to_dev_bf16(synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(T, 30), outliers=True))
    W = to_dev_bf16(synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(T, 31)))
    dY = to_dev_bf16(synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(T, 32)))
    _, _, qxt, sxt = fp8_quant_act_dual(X)
    qw, sw, _ = fp8_quant_weight(W)
    qd = torch.empty(T, Dout, dtype=torch.uint8, device="cuda")
    sd = torch.empty(Dout // 128, T, dtype=torch.float32, device="cuda")
    qdt = torch.empty(Dout, T, dtype=torch.uint8, device="cuda")
    sdt = torch.empty(T // 128, Dout, dtype=torch.float32, device="cuda")
    dX = torch.empty(T, Din, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(Dout, Din, dtype=torch.bfloat16, device="cuda")

    def backward():
        fp8_quant_act_dual(dY, qd, sd, qdt, sdt)
        fp8_gemm_blockwise(DGRAD, qd, sd, qw, sw, T, Din, Dout, out=dX)
        fp8_gemm_blockwise(WGRAD, qdt, sdt, qxt, sxt, Dout, Din, T, out=dW)

    g = _capture(backward)
    dY.copy_(to_dev_bf16(synth.normal_bf16(T, Dout, 2e-3, seed=synth.seed_for(T, 33))))
    for t in (qd, sd, qdt, sdt, dX, dW):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    eq, es, eqt, est = fp8_quant_act_dual(dY)
    edx = fp8_gemm_blockwise(DGRAD, eq, es, qw, sw, T, Din, Dout)
    edw = fp8_gemm_blockwise(WGRAD, eqt, est, qxt, sxt, Dout, Din, T)
    torch.cuda.synchronize()
    assert torch.equal(qd, eq) and torch.equal(sd, es)
    assert torch.equal(qdt, eqt) and torch.equal(sdt, est)
    assert torch.equal(dX, edx) and torch.equal(dW, edw)
    assert fp8bw_last_device_error() == 0
