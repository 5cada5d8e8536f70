"""The C-ABI library loads without a GPU, exports every function include/fp8bw.h
declares, and rejects bad arguments before touching the device."""
import ctypes as C
import os
import re

import pytest

import blockwise_fp8_linear_b200 as fb
from blockwise_fp8_linear_b200 import build as fbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "fp8bw.h")


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return fb.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert {"fp8_quant_act", "fp8_quant_act_t", "fp8_quant_weight", "fp8_gemm_blockwise",
            "fp8bw_status_string", "fp8bw_last_device_error"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in fp8bw.h but not exported"


def test_status_strings_and_version(L):
    for st in range(7):
        assert fb.fp8bw_status_string(st).startswith("FP8BW_")
    assert "unknown" in fb.fp8bw_status_string(99)
    assert "sm_100a" in fb.fp8bw_version()


def test_argument_errors_before_any_launch(L):
    """Host-side validation order: null -> EINVAL, sizes -> ESHAPE, alignment ->
    EALIGN; none of these touch the device, so they work here without a GPU."""
    p = C.c_void_p(0x10000)   # never dereferenced: validation fails first
    odd = C.c_void_p(0x10008)
    nul = C.c_void_p(0)
    s = C.c_void_p(0)
    assert L.fp8_quant_act(nul, 128, 128, p, p, s) == 1
    assert L.fp8_quant_act(p, 100, 128, p, p, s) == 3
    assert L.fp8_quant_act(p, 128, 0, p, p, s) == 3
    assert L.fp8_quant_act(p, 128, (1 << 20) + 128, p, p, s) == 3
    assert L.fp8_quant_act(odd, 128, 128, p, p, s) == 2
    assert L.fp8_quant_act_t(p, 128, 129, p, p, s) == 3
    assert L.fp8_quant_act_t(p, 128, 128, p, odd, s) == 2
    assert L.fp8_quant_weight(p, 128, 128, nul, p, nul, s) == 1
    assert L.fp8_quant_weight(p, 128, 128, p, p, odd, s) == 2
    assert L.fp8_gemm_blockwise(3, p, p, p, p, p, 128, 128, 128, s) == 1
    assert L.fp8_gemm_blockwise(-1, p, p, p, p, p, 128, 128, 128, s) == 1
    assert L.fp8_gemm_blockwise(0, p, p, p, p, nul, 128, 128, 128, s) == 1
    assert L.fp8_gemm_blockwise(0, p, p, p, p, p, 128, 256, 200, s) == 3
    assert L.fp8_gemm_blockwise(1, p, odd, p, p, p, 128, 256, 256, s) == 2
    assert L.fp8_quant_act_dual(p, 128, 128, p, p, nul, p, s) == 1
    assert L.fp8_quant_act_dual(p, 128, 100, p, p, p, p, s) == 3
    assert L.fp8_gemm_wgrad_acc32(p, p, p, p, nul, 128, 128, 128, s) == 1
    assert L.fp8_gemm_wgrad_acc32(p, p, p, p, odd, 128, 128, 128, s) == 2
    assert L.fp8_quant_act_e8m0(nul, 128, 128, p, p, s) == 1
    assert L.fp8_quant_act_t_e8m0(p, 128, 200, p, p, s) == 3
    assert L.fp8_quant_act_dual_e8m0(p, 128, 128, p, p, p, odd, s) == 2
    assert L.fp8_quant_weight_e8m0(p, 128, 128, p, nul, nul, s) == 1
    assert L.fp8_gemm_blockwise_e8m0(5, p, p, p, p, p, 128, 128, 128, s) == 1
    assert L.fp8_gemm_blockwise_e8m0(2, p, p, p, p, p, 128, 128, 130, s) == 3
    assert L.fp8_gemm_blockwise_e8m0(0, p, odd, p, p, p, 128, 128, 128, s) == 2


def test_no_gpu_reports_cuda_error_not_crash(L):
    """With valid arguments and no usable device the call returns an error status."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = C.c_void_p(0x10000)
    assert L.fp8_quant_act(p, 128, 128, p, p, C.c_void_p(0)) in (4, 6)


def test_python_binding_validates_types():
    import torch
    with pytest.raises(TypeError):
        fb.fp8_quant_act(torch.zeros(128, 128, dtype=torch.bfloat16))  # CPU tensor
