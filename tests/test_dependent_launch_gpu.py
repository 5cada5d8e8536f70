"""Every kernel of the library is launched with programmatic stream serialization and
waits for its predecessor before touching memory.  These chains run several of them
back to back on one stream with no synchronization in between, each consuming the
previous one's output, and check the end result against the oracle fed with the
intermediate values read back afterwards (so a consumer that started before its
producer finished would show up as a mismatch)."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_fp8_linear_b200 import (DGRAD, FPROP, fp8_gemm_blockwise, fp8_quant_act,
                                       fp8_quant_act_dual, fp8_quant_weight,
                                       fp8bw_last_device_error, synth)
from tests._gpu import bf16_dev_to_f64, check_gemm, to_dev_bf16

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("T,D", [(256, 1024), (8192, 2048)])
def test_gemm_output_feeds_next_quantizer_and_gemm(T, D):
    """Y = X W1^T (GEMM) -> quantize Y (dual quantizer) -> Z = Y W2^T (GEMM), issued
    back to back; then both stages are recomputed by the oracle from the read-back Y."""
    X = synth.normal_bf16(T, D, 1.0, seed=synth.seed_for(T, 0), outliers=True)
    W1 = synth.normal_bf16(D, D, 0.02, seed=synth.seed_for(T, 1))
    W2 = synth.normal_bf16(D, D, 0.02, seed=synth.seed_for(T, 2))
    qw1, sw1, _ = fp8_quant_weight(to_dev_bf16(W1))
    qw2, sw2, _ = fp8_quant_weight(to_dev_bf16(W2))
    qx, sx = fp8_quant_act(to_dev_bf16(X))
    torch.cuda.synchronize()
    for _ in range(3):  # repeat, so later rounds overlap the previous round's tail
        Y = fp8_gemm_blockwise(FPROP, qx, sx, qw1, sw1, T, D, D)
        qy, sy, qyt, syt = fp8_quant_act_dual(Y)
        Z = fp8_gemm_blockwise(FPROP, qy, sy, qw2, sw2, T, D, D)
    torch.cuda.synchronize()
    assert fp8bw_last_device_error() == 0
    Yh = _u16(Y)
    qy_ref, sy_ref = oracle.quant_act(Yh)
    assert np.array_equal(qy.cpu().numpy(), qy_ref)
    assert np.array_equal(sy.cpu().numpy().view(np.uint32), sy_ref.view(np.uint32))
    qyt_ref, syt_ref = oracle.quant_act_t(Yh)
    assert np.array_equal(qyt.cpu().numpy(), qyt_ref)
    qw2_ref, sw2_ref, _ = oracle.quant_weight(W2)
    rows = None if T <= 256 else np.unique(np.concatenate([np.arange(0, T, 128),
                                                            np.arange(127, T, 128)]))
    z_ref, asum = oracle.gemm(FPROP, qy_ref, sy_ref, qw2_ref, sw2_ref, T, D, D, rows=rows)
    z = bf16_dev_to_f64(Z)
    check_gemm(z if rows is None else z[rows], z_ref, asum, "chained GEMM")


def test_dgrad_output_feeds_quantizer():
    """dX from DGRAD quantized straight away (the next layer's incoming gradient)."""
    T, Din, Dout = 1024, 2048, 1024
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(5, 2))
    W = synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(5, 1))
    qw, sw, _ = fp8_quant_weight(to_dev_bf16(W))
    qdy, sdy = fp8_quant_act(to_dev_bf16(dY))
    dX = fp8_gemm_blockwise(DGRAD, qdy, sdy, qw, sw, T, Din, Dout)
    q, s = fp8_quant_act(dX)
    torch.cuda.synchronize()
    assert fp8bw_last_device_error() == 0
    q_ref, s_ref = oracle.quant_act(_u16(dX))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
