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


def _validate(items):
    """Check the tensor arguments of one call before anything reaches the C ABI.
    items: (tensor or None, dtype, shape, name); None marks an output to allocate.
    Shapes are checked first, for every tensor, then dtype, contiguity and that all
    are CUDA tensors of one device.  A size that disagreed with the M, N, K handed to
    the C call would let a kernel read or write past an allocation, so every mismatch
    raises here (ValueError for shapes and devices, TypeError for kinds)."""
    import torch
    given = [(t, dt, shp, name) for t, dt, shp, name in items if t is not None]
    for t, _, shp, name in given:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch tensor")
        if tuple(t.shape) != tuple(int(d) for d in shp):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shp)}")
    for t, dt, _, name in given:
        if t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
    dev = given[0][0].device
    for t, _, _, name in given:
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev} (one device per call)")
    return dev


def _alloc(t, shape, dtype, device):
    import torch
    return torch.empty(shape, dtype=dtype, device=device) if t is None else t


def _dims(M, N=None, K=None):
    """Sizes must be positive multiples of 128 (the ABI rejects others; checked here
    so that buffer shapes derived from them are whole)."""
    for d in (M, N, K):
        if d is not None and (int(d) <= 0 or int(d) % 128):
            raise ValueError(f"size {d} is not a positive multiple of 128")


def _on(device):
    """Context that makes `device` current, so the call's stream and the current device
    match its buffers (the ABI rejects buffers of another device)."""
    import torch
    return torch.cuda.device(device)


def _tokens(M):
    """A token count (the M of the activation quantizers and of FPROP/DGRAD, the
    reduction K of WGRAD) may end in a partial group of 128: a positive multiple of
    16 (the 16-byte row stride of the token-major codes)."""
    if int(M) <= 0 or int(M) % 16:
        raise ValueError(f"token count {M} is not a positive multiple of 16")


def _x2(x, name, tokens=False):
    """Rows and columns of a 2-D input; with tokens=True the rows are a token count
    (a multiple of 16), else both are multiples of 128."""
    import torch
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor")
    M, K = x.shape
    if tokens:
        _tokens(M)
        _dims(K)
    else:
        _dims(M, K)
    return int(M), int(K)


def _groups(M):
    return (int(M) + 127) // 128


def fp8bw_last_device_error(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device error word status."""
    return int(lib().fp8bw_last_device_error(_stream(stream)))


def fp8bw_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Run the bounded-wait self-test kernel (a wait that nothing satisfies)."""
    _check(lib().fp8bw_selftest_wait_timeout(int(limit_us), _stream(stream)),
           "fp8bw_selftest_wait_timeout")


def fp8_quant_act(x, q=None, s=None, stream=None):
    """X[M][K] bf16 -> (Q[M][K] uint8 E4M3 codes, S[K/128][M] float32); M any
    multiple of 16 tokens."""
    import torch
    M, K = _x2(x, "x", tokens=True)
    dev = _validate([(x, torch.bfloat16, (M, K), "x"), (q, torch.uint8, (M, K), "q"),
                     (s, torch.float32, (K // 128, M), "s")])
    q = _alloc(q, (M, K), torch.uint8, dev)
    s = _alloc(s, (K // 128, M), torch.float32, dev)
    with _on(dev):
        _check(lib().fp8_quant_act(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(),
                                   _stream(stream)), "fp8_quant_act")
    return q, s


def fp8_quant_act_t(x, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q^T[K][M] uint8, S^T[ceil(M/128)][K] float32), groups along M
    (the last group holds the M mod 128 tokens present)."""
    import torch
    M, K = _x2(x, "x", tokens=True)
    dev = _validate([(x, torch.bfloat16, (M, K), "x"), (qt, torch.uint8, (K, M), "qt"),
                     (st, torch.float32, (_groups(M), K), "st")])
    qt = _alloc(qt, (K, M), torch.uint8, dev)
    st = _alloc(st, (_groups(M), K), torch.float32, dev)
    with _on(dev):
        _check(lib().fp8_quant_act_t(x.data_ptr(), M, K, qt.data_ptr(), st.data_ptr(),
                                     _stream(stream)), "fp8_quant_act_t")
    return qt, st


def fp8_quant_act_dual(x, q=None, s=None, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q, S, Q^T, S^T): both layouts from one read of X."""
    import torch
    M, K = _x2(x, "x", tokens=True)
    dev = _validate([(x, torch.bfloat16, (M, K), "x"), (q, torch.uint8, (M, K), "q"),
                     (s, torch.float32, (K // 128, M), "s"), (qt, torch.uint8, (K, M), "qt"),
                     (st, torch.float32, (_groups(M), K), "st")])
    q = _alloc(q, (M, K), torch.uint8, dev)
    s = _alloc(s, (K // 128, M), torch.float32, dev)
    qt = _alloc(qt, (K, M), torch.uint8, dev)
    st = _alloc(st, (_groups(M), K), torch.float32, dev)
    with _on(dev):
        _check(lib().fp8_quant_act_dual(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(),
                                        qt.data_ptr(), st.data_ptr(), _stream(stream)),
               "fp8_quant_act_dual")
    return q, s, qt, st


def fp8_quant_weight(w, want_t: bool = False, q=None, s=None, qt=None, stream=None):
    """W[N][K] bf16 -> (Q[N][K] uint8, S[N/128][K/128] float32, Q^T[K][N] or None)."""
    import torch
    N, K = _x2(w, "w")
    dev = _validate([(w, torch.bfloat16, (N, K), "w"), (q, torch.uint8, (N, K), "q"),
                     (s, torch.float32, (N // 128, K // 128), "s"),
                     (qt, torch.uint8, (K, N), "qt")])
    q = _alloc(q, (N, K), torch.uint8, dev)
    s = _alloc(s, (N // 128, K // 128), torch.float32, dev)
    if want_t:
        qt = _alloc(qt, (K, N), torch.uint8, dev)
    with _on(dev):
        _check(lib().fp8_quant_weight(w.data_ptr(), N, K, q.data_ptr(), s.data_ptr(),
                                      qt.data_ptr() if qt is not None else None,
                                      _stream(stream)), "fp8_quant_weight")
    return q, s, qt


def _gemm_shapes(mode: int, M: int, N: int, K: int, e8m0: bool = False):
    """Operand shapes of each GEMM mode (include/fp8bw.h): a, sa, b, sb."""
    if mode not in (FPROP, DGRAD, WGRAD):
        raise ValueError(f"mode must be FPROP, DGRAD or WGRAD, got {mode}")
    if e8m0:
        _dims(M, N, K)
    elif mode == WGRAD:   # the reduction runs over tokens
        _dims(M, N)
        _tokens(K)
    else:                 # M is the token count
        _tokens(M)
        _dims(N, K)
    a = (M, K)
    b = (K, N) if mode == DGRAD else (N, K)
    if not e8m0:
        sa = (_groups(K), M)
        sb = {FPROP: (N // 128, K // 128), DGRAD: (K // 128, N // 128), WGRAD: (_groups(K), N)}[mode]
    else:  # 512-byte scale blocks, one per 128 rows x 128-deep reduction block
        sa = (M // 128, (K // 128) * 512)
        sb = (K // 128, (N // 128) * 512) if mode == DGRAD else (N // 128, (K // 128) * 512)
    return a, sa, b, sb


def fp8_gemm_blockwise(mode: int, a, sa, b, sb, M: int, N: int, K: int, out=None, stream=None):
    """D[M][N] bf16 from FP8 operands and blockwise scales; see include/fp8bw.h for the
    operand layouts of FPROP, DGRAD and WGRAD."""
    import torch
    M, N, K = int(M), int(N), int(K)
    sh_a, sh_sa, sh_b, sh_sb = _gemm_shapes(mode, M, N, K)
    dev = _validate([(a, torch.uint8, sh_a, "a"), (sa, torch.float32, sh_sa, "sa"),
                     (b, torch.uint8, sh_b, "b"), (sb, torch.float32, sh_sb, "sb"),
                     (out, torch.bfloat16, (M, N), "out")])
    out = _alloc(out, (M, N), torch.bfloat16, dev)
    with _on(dev):
        _check(lib().fp8_gemm_blockwise(int(mode), a.data_ptr(), sa.data_ptr(), b.data_ptr(),
                                        sb.data_ptr(), out.data_ptr(), M, N, K, _stream(stream)),
               "fp8_gemm_blockwise")
    return out


def fp8_gemm_wgrad_acc32(a, sa, b, sb, M: int, N: int, K: int, dw32, stream=None):
    """dw32[M][N] (float32, caller-owned) += the wgrad sum, kept in FP32 (no BF16
    rounding); a, sa, b, sb as for fp8_gemm_blockwise(WGRAD, ...)."""
    import torch
    M, N, K = int(M), int(N), int(K)
    sh_a, sh_sa, sh_b, sh_sb = _gemm_shapes(WGRAD, M, N, K)
    if dw32 is None:
        raise TypeError("dw32 must be a caller-owned float32 tensor")
    dev = _validate([(a, torch.uint8, sh_a, "a"), (sa, torch.float32, sh_sa, "sa"),
                     (b, torch.uint8, sh_b, "b"), (sb, torch.float32, sh_sb, "sb"),
                     (dw32, torch.float32, (M, N), "dw32")])
    with _on(dev):
        _check(lib().fp8_gemm_wgrad_acc32(a.data_ptr(), sa.data_ptr(), b.data_ptr(),
                                          sb.data_ptr(), dw32.data_ptr(), M, N, K,
                                          _stream(stream)), "fp8_gemm_wgrad_acc32")
    return dw32


# -- power-of-two (E8M0) scales: the MXFP8 form of the recipe --------------------

def fp8_quant_act_e8m0(x, q=None, s=None, stream=None):
    """X[M][K] bf16 -> (Q[M][K] uint8, S: E8M0 scale blocks [M/128][(K/128)*512] uint8,
    the tensor-core layout described in include/fp8bw.h)."""
    import torch
    M, K = _x2(x, "x")
    ssh = (M // 128, (K // 128) * 512)
    dev = _validate([(x, torch.bfloat16, (M, K), "x"), (q, torch.uint8, (M, K), "q"),
                     (s, torch.uint8, ssh, "s")])
    q = _alloc(q, (M, K), torch.uint8, dev)
    s = _alloc(s, ssh, torch.uint8, dev)
    with _on(dev):
        _check(lib().fp8_quant_act_e8m0(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(),
                                        _stream(stream)), "fp8_quant_act_e8m0")
    return q, s


def fp8_quant_act_t_e8m0(x, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q^T[K][M] uint8, S^T: E8M0 scale blocks [K/128][(M/128)*512])."""
    import torch
    M, K = _x2(x, "x")
    tsh = (K // 128, (M // 128) * 512)
    dev = _validate([(x, torch.bfloat16, (M, K), "x"), (qt, torch.uint8, (K, M), "qt"),
                     (st, torch.uint8, tsh, "st")])
    qt = _alloc(qt, (K, M), torch.uint8, dev)
    st = _alloc(st, tsh, torch.uint8, dev)
    with _on(dev):
        _check(lib().fp8_quant_act_t_e8m0(x.data_ptr(), M, K, qt.data_ptr(), st.data_ptr(),
                                          _stream(stream)), "fp8_quant_act_t_e8m0")
    return qt, st


def fp8_quant_act_dual_e8m0(x, q=None, s=None, qt=None, st=None, stream=None):
    """X[M][K] bf16 -> (Q, S, Q^T, S^T) with E8M0 scale codes, from one read of X."""
    import torch
    M, K = _x2(x, "x")
    ssh, tsh = (M // 128, (K // 128) * 512), (K // 128, (M // 128) * 512)
    dev = _validate([(x, torch.bfloat16, (M, K), "x"), (q, torch.uint8, (M, K), "q"),
                     (s, torch.uint8, ssh, "s"), (qt, torch.uint8, (K, M), "qt"),
                     (st, torch.uint8, tsh, "st")])
    q = _alloc(q, (M, K), torch.uint8, dev)
    s = _alloc(s, ssh, torch.uint8, dev)
    qt = _alloc(qt, (K, M), torch.uint8, dev)
    st = _alloc(st, tsh, torch.uint8, dev)
    with _on(dev):
        _check(lib().fp8_quant_act_dual_e8m0(x.data_ptr(), M, K, q.data_ptr(), s.data_ptr(),
                                             qt.data_ptr(), st.data_ptr(), _stream(stream)),
               "fp8_quant_act_dual_e8m0")
    return q, s, qt, st


def fp8_quant_weight_e8m0(w, want_t: bool = False, q=None, s=None, qt=None, stream=None):
    """W[N][K] bf16 -> (Q[N][K], S: E8M0 scale blocks [N/128][(K/128)*512], Q^T or None)."""
    import torch
    N, K = _x2(w, "w")
    ssh = (N // 128, (K // 128) * 512)
    dev = _validate([(w, torch.bfloat16, (N, K), "w"), (q, torch.uint8, (N, K), "q"),
                     (s, torch.uint8, ssh, "s"), (qt, torch.uint8, (K, N), "qt")])
    q = _alloc(q, (N, K), torch.uint8, dev)
    s = _alloc(s, ssh, torch.uint8, dev)
    if want_t:
        qt = _alloc(qt, (K, N), torch.uint8, dev)
    with _on(dev):
        _check(lib().fp8_quant_weight_e8m0(w.data_ptr(), N, K, q.data_ptr(), s.data_ptr(),
                                           qt.data_ptr() if qt is not None else None,
                                           _stream(stream)), "fp8_quant_weight_e8m0")
    return q, s, qt


def fp8_gemm_blockwise_e8m0(mode: int, a, sa, b, sb, M: int, N: int, K: int, out=None,
                            stream=None):
    """fp8_gemm_blockwise with E8M0 scale blocks (from the *_e8m0 quantizers), applied by
    the block-scaled MMA."""
    import torch
    M, N, K = int(M), int(N), int(K)
    sh_a, sh_sa, sh_b, sh_sb = _gemm_shapes(mode, M, N, K, e8m0=True)
    dev = _validate([(a, torch.uint8, sh_a, "a"), (sa, torch.uint8, sh_sa, "sa"),
                     (b, torch.uint8, sh_b, "b"), (sb, torch.uint8, sh_sb, "sb"),
                     (out, torch.bfloat16, (M, N), "out")])
    out = _alloc(out, (M, N), torch.bfloat16, dev)
    with _on(dev):
        _check(lib().fp8_gemm_blockwise_e8m0(int(mode), a.data_ptr(), sa.data_ptr(),
                                             b.data_ptr(), sb.data_ptr(), out.data_ptr(), M, N, K,
                                             _stream(stream)), "fp8_gemm_blockwise_e8m0")
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
