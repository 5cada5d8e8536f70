"""Blockwise-FP8 Transformer linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI of ``libfp8bw.so`` (declared in
``include/fp8bw.h``).  Every function here only marshals arguments: it allocates
outputs with torch, checks dtypes and devices, and calls the C entry point of the
same name on the current CUDA stream.  All arithmetic runs in the CUDA kernels.
There is no CPU fallback: if the library is missing or the device is not sm_100,
the calls raise.

Method (Puro-2B, part 3/7, section 3.2 "FP8 Mixed-Precision Training"): E4M3
operands; activations and their gradients scaled per 128 neighbouring elements in
the summed (K) direction, weights per 128x128 tile; FP32
scales amax/448, and fprop / dgrad / wgrad GEMMs in FP8 with a BF16 result.
"""
from __future__ import annotations

import ctypes as C
import os

__all__ = [
    "FPROP", "DGRAD", "WGRAD", "Fp8bwError", "lib", "library_path",
    "fp8_quant_act", "fp8_quant_act_t", "fp8_quant_act_dual", "fp8_quant_weight",
    "fp8_gemm_blockwise", "fp8_gemm_wgrad_acc32",
    "fp8_quant_act_e8m0", "fp8_quant_act_t_e8m0", "fp8_quant_act_dual_e8m0",
    "fp8_quant_weight_e8m0", "fp8_gemm_blockwise_e8m0",
    "fp8bw_status_string", "fp8bw_last_device_error", "fp8bw_version",
    "fp8bw_selftest_wait_timeout",
    "linear_fprop", "linear_dgrad", "linear_wgrad",
]

FPROP, DGRAD, WGRAD = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libfp8bw.so")
_lib = None


class Fp8bwError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {fp8bw_status_string(status)} (status {status})")


def lib():
    """Load libfp8bw.so (built in-tree by ``python -m blockwise_fp8_linear_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"{library_path} is missing: build it with "
                "`python -m blockwise_fp8_linear_b200.build` (no CPU fallback exists)")
        L = C.CDLL(library_path)
        vp, i64, i32 = C.c_void_p, C.c_int64, C.c_int
        L.fp8_quant_act.argtypes = [vp, i64, i64, vp, vp, vp]
        L.fp8_quant_act_t.argtypes = [vp, i64, i64, vp, vp, vp]
        L.fp8_quant_act_dual.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.fp8_quant_weight.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.fp8_gemm_blockwise.argtypes = [i32, vp, vp, vp, vp, vp, i64, i64, i64, vp]
        L.fp8_gemm_wgrad_acc32.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
        L.fp8_quant_act_e8m0.argtypes = [vp, i64, i64, vp, vp, vp]
        L.fp8_quant_act_t_e8m0.argtypes = [vp, i64, i64, vp, vp, vp]
        L.fp8_quant_act_dual_e8m0.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.fp8_quant_weight_e8m0.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.fp8_gemm_blockwise_e8m0.argtypes = [i32, vp, vp, vp, vp, vp, i64, i64, i64, vp]
        for f in (L.fp8_quant_act, L.fp8_quant_act_t, L.fp8_quant_act_dual, L.fp8_quant_weight,
                  L.fp8_gemm_blockwise, L.fp8_gemm_wgrad_acc32, L.fp8_quant_act_e8m0,
                  L.fp8_quant_act_t_e8m0, L.fp8_quant_act_dual_e8m0, L.fp8_quant_weight_e8m0,
                  L.fp8_gemm_blockwise_e8m0):
            f.restype = i32
        L.fp8bw_status_string.argtypes = [i32]
        L.fp8bw_status_string.restype = C.c_char_p
        L.fp8bw_last_device_error.argtypes = [vp]
        L.fp8bw_last_device_error.restype = i32
        L.fp8bw_selftest_wait_timeout.argtypes = [i64, vp]
        L.fp8bw_selftest_wait_timeout.restype = i32
        L.fp8bw_version.argtypes = []
        L.fp8bw_version.restype = C.c_char_p
        _lib = L
    return _lib


def fp8bw_status_string(status: int) -> str:
    return lib().fp8bw_status_string(int(status)).decode()


def fp8bw_version() -> str:
    return lib().fp8bw_version().decode()


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise Fp8bwError(status, what)


def _need(t, dtype, ndim, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


def fp8bw_last_device_error(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device error word status."""
    return int(lib().fp8bw_last_device_error(_stream(stream)))


def fp8bw_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Run the bounded-wait self-test kernel (a wait that nothing satisfies)."""
    _check(lib().fp8bw_selftest_wait_timeout(int(limit_us), _stream(stream)),
           "fp8bw_selftest_wait_timeout")


def fp8_quant_act(x, q=None, s=None, stream=None):
    """X[M][K] bf16 -> (Q[M][K] uint8 E4M3 codes, S[K/128][M] float32)."""
    import torch
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if q is None else q
    s = torch.empty((K // 128, M), dtype=torch.float32, device=x.device) if s is None else s
    _check(lib().fp8_quant_act(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(), _stream(stream)),
           "fp8_quant_act")
    return q, s


def fp8_quant_act_t(x, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q^T[K][M] uint8, S^T[M/128][K] float32), groups along M."""
    import torch
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    qt = torch.empty((K, M), dtype=torch.uint8, device=x.device) if qt is None else qt
    st = torch.empty((M // 128, K), dtype=torch.float32, device=x.device) if st is None else st
    _check(lib().fp8_quant_act_t(x.data_ptr(), M, K, qt.data_ptr(), st.data_ptr(),
                                 _stream(stream)), "fp8_quant_act_t")
    return qt, st


def fp8_quant_act_dual(x, q=None, s=None, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q, S, Q^T, S^T): both layouts from one read of X."""
    import torch
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if q is None else q
    s = torch.empty((K // 128, M), dtype=torch.float32, device=x.device) if s is None else s
    qt = torch.empty((K, M), dtype=torch.uint8, device=x.device) if qt is None else qt
    st = torch.empty((M // 128, K), dtype=torch.float32, device=x.device) if st is None else st
    _check(lib().fp8_quant_act_dual(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(), qt.data_ptr(),
                                    st.data_ptr(), _stream(stream)), "fp8_quant_act_dual")
    return q, s, qt, st


def fp8_quant_weight(w, want_t: bool = False, q=None, s=None, qt=None, stream=None):
    """W[N][K] bf16 -> (Q[N][K] uint8, S[N/128][K/128] float32, Q^T[K][N] or None)."""
    import torch
    _need(w, torch.bfloat16, 2, "w")
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device) if q is None else q
    s = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device) if s is None else s
    if want_t and qt is None:
        qt = torch.empty((K, N), dtype=torch.uint8, device=w.device)
    _check(lib().fp8_quant_weight(w.data_ptr(), N, K, q.data_ptr(), s.data_ptr(),
                                  qt.data_ptr() if qt is not None else None, _stream(stream)),
           "fp8_quant_weight")
    return q, s, qt


def fp8_gemm_blockwise(mode: int, a, sa, b, sb, M: int, N: int, K: int, out=None, stream=None):
    """D[M][N] bf16 from FP8 operands and blockwise scales; see include/fp8bw.h for the
    operand layouts of FPROP, DGRAD and WGRAD."""
    import torch
    for t, dt, name in ((a, torch.uint8, "a"), (b, torch.uint8, "b"),
                        (sa, torch.float32, "sa"), (sb, torch.float32, "sb")):
        _need(t, dt, 2, name)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device) if out is None else out
    _check(lib().fp8_gemm_blockwise(int(mode), a.data_ptr(), sa.data_ptr(), b.data_ptr(),
                                    sb.data_ptr(), out.data_ptr(), M, N, K, _stream(stream)),
           "fp8_gemm_blockwise")
    return out


def fp8_gemm_wgrad_acc32(a, sa, b, sb, M: int, N: int, K: int, dw32, stream=None):
    """dw32[M][N] (float32, caller-owned) += the wgrad sum, kept in FP32 (no BF16
    rounding); a, sa, b, sb as for fp8_gemm_blockwise(WGRAD, ...)."""
    import torch
    for t, dt, name in ((a, torch.uint8, "a"), (b, torch.uint8, "b"),
                        (sa, torch.float32, "sa"), (sb, torch.float32, "sb"),
                        (dw32, torch.float32, "dw32")):
        _need(t, dt, 2, name)
    _check(lib().fp8_gemm_wgrad_acc32(a.data_ptr(), sa.data_ptr(), b.data_ptr(), sb.data_ptr(),
                                      dw32.data_ptr(), M, N, K, _stream(stream)),
           "fp8_gemm_wgrad_acc32")
    return dw32


# -- power-of-two (E8M0) scales: the MXFP8 form of the recipe --------------------

def fp8_quant_act_e8m0(x, q=None, s=None, stream=None):
    """X[M][K] bf16 -> (Q[M][K] uint8, S: E8M0 scale blocks [M/128][(K/128)*512] uint8,
    the tensor-core layout described in include/fp8bw.h)."""
    import torch
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if q is None else q
    s = torch.empty((M // 128, (K // 128) * 512), dtype=torch.uint8, device=x.device) if s is None else s
    _check(lib().fp8_quant_act_e8m0(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(),
                                    _stream(stream)), "fp8_quant_act_e8m0")
    return q, s


def fp8_quant_act_t_e8m0(x, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q^T[K][M] uint8, S^T: E8M0 scale blocks [K/128][(M/128)*512])."""
    import torch
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    qt = torch.empty((K, M), dtype=torch.uint8, device=x.device) if qt is None else qt
    st = torch.empty((K // 128, (M // 128) * 512), dtype=torch.uint8, device=x.device) if st is None else st
    _check(lib().fp8_quant_act_t_e8m0(x.data_ptr(), M, K, qt.data_ptr(), st.data_ptr(),
                                      _stream(stream)), "fp8_quant_act_t_e8m0")
    return qt, st


def fp8_quant_act_dual_e8m0(x, stream=None):
    """X[M][K] bf16 -> (Q, S, Q^T, S^T) with E8M0 scale codes, from one read of X."""
    import torch
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    dev = x.device
    q = torch.empty((M, K), dtype=torch.uint8, device=dev)
    s = torch.empty((M // 128, (K // 128) * 512), dtype=torch.uint8, device=dev)
    qt = torch.empty((K, M), dtype=torch.uint8, device=dev)
    st = torch.empty((K // 128, (M // 128) * 512), dtype=torch.uint8, device=dev)
    _check(lib().fp8_quant_act_dual_e8m0(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(),
                                         qt.data_ptr(), st.data_ptr(), _stream(stream)),
           "fp8_quant_act_dual_e8m0")
    return q, s, qt, st


def fp8_quant_weight_e8m0(w, want_t: bool = False, stream=None):
    """W[N][K] bf16 -> (Q[N][K], S: E8M0 scale blocks [N/128][(K/128)*512], Q^T or None)."""
    import torch
    _need(w, torch.bfloat16, 2, "w")
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    s = torch.empty((N // 128, (K // 128) * 512), dtype=torch.uint8, device=w.device)
    qt = torch.empty((K, N), dtype=torch.uint8, device=w.device) if want_t else None
    _check(lib().fp8_quant_weight_e8m0(w.data_ptr(), N, K, q.data_ptr(), s.data_ptr(),
                                       qt.data_ptr() if want_t else None, _stream(stream)),
           "fp8_quant_weight_e8m0")
    return q, s, qt


def fp8_gemm_blockwise_e8m0(mode: int, a, sa, b, sb, M: int, N: int, K: int, out=None,
                            stream=None):
    """fp8_gemm_blockwise with E8M0 scale blocks (from the *_e8m0 quantizers), applied by
    the block-scaled MMA."""
    import torch
    for t, dt, name in ((a, torch.uint8, "a"), (b, torch.uint8, "b"),
                        (sa, torch.uint8, "sa"), (sb, torch.uint8, "sb")):
        _need(t, dt, 2, name)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device) if out is None else out
    _check(lib().fp8_gemm_blockwise_e8m0(int(mode), a.data_ptr(), sa.data_ptr(), b.data_ptr(),
                                         sb.data_ptr(), out.data_ptr(), M, N, K, _stream(stream)),
           "fp8_gemm_blockwise_e8m0")
    return out


# -- the three GEMMs of the linear layer, composed from the entry points above ----

def linear_fprop(x, w, stream=None):
    """Y = X W^T with X[T][Din], W[Dout][Din] (bf16).  Returns (Y, saved) where saved
    holds the quantized weight for dgrad."""
    T, Din = x.shape
    Dout = w.shape[0]
    qx, sx = fp8_quant_act(x, stream=stream)
    qw, sw, _ = fp8_quant_weight(w, stream=stream)
    y = fp8_gemm_blockwise(FPROP, qx, sx, qw, sw, T, Dout, Din, stream=stream)
    return y, (qw, sw)


def linear_dgrad(dy, qw, sw, stream=None):
    """dX = dY W with dY[T][Dout] and the weight quantized by fp8_quant_weight."""
    T, Dout = dy.shape
    Din = qw.shape[1]
    qdy, sdy = fp8_quant_act(dy, stream=stream)
    return fp8_gemm_blockwise(DGRAD, qdy, sdy, qw, sw, T, Din, Dout, stream=stream)


def linear_wgrad(dy, x, stream=None):
    """dW = dY^T X with both operands quantized along the token dimension."""
    T, Dout = dy.shape
    Din = x.shape[1]
    qdyt, sdyt = fp8_quant_act_t(dy, stream=stream)
    qxt, sxt = fp8_quant_act_t(x, stream=stream)
    return fp8_gemm_blockwise(WGRAD, qdyt, sdyt, qxt, sxt, Dout, Din, T, stream=stream)
