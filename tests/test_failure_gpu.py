"""Failure detection on the GPU without a GPU fault: a bounded in-kernel wait that
nothing satisfies runs out, the host reads FP8BW_ETIMEOUT from the device error
word, the word clears, and the device keeps working."""
import numpy as np
import pytest

import oracle
import blockwise_fp8_linear_b200 as fb
from blockwise_fp8_linear_b200 import synth
from tests._gpu import bf16_dev_to_f64, check_gemm, to_dev_bf16

pytestmark = pytest.mark.gpu

FP8BW_OK, FP8BW_EINVAL, FP8BW_ETIMEOUT = 0, 1, 5


def test_bounded_wait_reports_timeout_and_device_stays_usable():
    assert fb.fp8bw_last_device_error() == FP8BW_OK
    fb.fp8bw_selftest_wait_timeout(20000)          # 20 ms wait on a barrier nobody arrives on
    assert fb.fp8bw_last_device_error() == FP8BW_ETIMEOUT
    assert fb.fp8bw_last_device_error() == FP8BW_OK   # read-and-clear
    # the context is intact: a GEMM right after still matches the oracle
    X = synth.normal_bf16(256, 512, 1.0, seed=41)
    W = synth.normal_bf16(256, 512, 0.02, seed=42)
    qx, sx = fb.fp8_quant_act(to_dev_bf16(X))
    qw, sw, _ = fb.fp8_quant_weight(to_dev_bf16(W))
    y = bf16_dev_to_f64(fb.fp8_gemm_blockwise(fb.FPROP, qx, sx, qw, sw, 256, 256, 512))
    a, sa = oracle.quant_act(X)
    b, sb, _ = oracle.quant_weight(W)
    y_ref, asum = oracle.gemm(oracle.FPROP, a, sa, b, sb, 256, 256, 512)
    check_gemm(y, y_ref, asum, "after timeout")
    assert fb.fp8bw_last_device_error() == FP8BW_OK


def test_selftest_rejects_bad_limits():
    for bad in (0, -5, 2_000_000):
        with pytest.raises(fb.Fp8bwError) as e:
            fb.fp8bw_selftest_wait_timeout(bad)
        assert e.value.status == FP8BW_EINVAL
