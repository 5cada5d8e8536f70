"""Helpers shared by the GPU parity tests: host<->device marshalling and the GEMM
acceptance check (elementwise and normwise tolerances)."""
from __future__ import annotations

import numpy as np
import torch

# GEMM acceptance bar: |y - y_ref| <= 2^-7 |y_ref| + 1e-3 sum_k |ahat_k bhat_k|
# elementwise, and ||y - y_ref||_F / ||y_ref||_F <= 5e-3.  2^-7 covers the final
# BF16 rounding (half an ulp is <= 2^-8 relative) with a factor of two to spare; the
# absolute term covers FP32 accumulation and the rounding of the per-block scale
# product.
REL_TOL = 2.0 ** -7
ABS_TOL = 1e-3
NORM_TOL = 5e-3


def to_dev_bf16(x_u16: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x_u16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def bf16_dev_to_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


def check_gemm(y: np.ndarray, y_ref: np.ndarray, asum: np.ndarray, what: str = ""):
    err = np.abs(y - y_ref)
    bound = REL_TOL * np.abs(y_ref) + ABS_TOL * asum
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} elements out of tolerance; first at {tuple(i)}: "
            f"y={y[tuple(i)]!r} ref={y_ref[tuple(i)]!r} bound={bound[tuple(i)]!r}")
    nref = np.linalg.norm(y_ref)
    if nref > 0:
        rel = np.linalg.norm(y - y_ref) / nref
        assert rel <= NORM_TOL, f"{what}: normwise relative error {rel:.3e} > {NORM_TOL}"
    else:
        assert np.all(y == 0), f"{what}: reference is zero but output is not"
