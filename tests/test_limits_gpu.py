"""GPU parity at the size limit of the ABI (FP8BW_MAX_DIM = 2^20 along one dimension):
the fused quantizer with 2^20 tokens or 2^20 features, fprop over 2^20 tokens, and
wgrad with a reduction of 2^20 tokens, each against the CPU oracle (codes and scales
bit-exact; GEMM outputs on rows that touch every row tile, within the tolerance)."""
import pytest

import oracle
from blockwise_fp8_linear_b200 import FPROP, WGRAD, fp8_quant_act_dual, synth
from tests._gpu import check_gemm, to_dev_bf16
from tests.test_gemm_gpu import _rows, _run_mode, _same

pytestmark = pytest.mark.gpu

LIMIT = 1 << 20


@pytest.mark.parametrize("M,K", [(128, LIMIT), (LIMIT, 128)])
def test_dual_quantizer_at_the_dimension_limit(M, K):
    x = synth.normal_bf16(M, K, 1.0, seed=synth.seed_for(40, M), outliers=True)
    q, s, qt, st = fp8_quant_act_dual(to_dev_bf16(x))
    qr, sr = oracle.quant_act(x)
    qtr, str_ = oracle.quant_act_t(x)
    for g, r in ((q, qr), (s, sr), (qt, qtr), (st, str_)):
        _same(g, r)


def test_fprop_over_the_token_limit():
    T, Din, Dout = LIMIT, 128, 256
    X = synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(43, 0), outliers=True)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(43, 1))
    y, y_ref, asum = _run_mode(FPROP, X, W, None, rows=_rows(T, 4096))
    check_gemm(y, y_ref, asum, "fprop, 2^20 tokens")


def test_wgrad_over_a_reduction_at_the_token_limit():
    T, Din, Dout = LIMIT, 128, 128
    X = synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(44, 0), outliers=True)
    W = synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(44, 1))
    dY = synth.normal_bf16(T, Dout, 1e-3, seed=synth.seed_for(44, 2))
    y, y_ref, asum = _run_mode(WGRAD, X, W, dY, rows=_rows(Dout, 4))
    check_gemm(y, y_ref, asum, "wgrad, reduction over 2^20 tokens")
