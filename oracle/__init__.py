"""CPU oracle for the blockwise-FP8 linear layer (ctypes wrapper over plain C).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The product
library never imports it, and it imports nothing from the product.

Every function takes and returns numpy arrays.  BF16 tensors are carried as their
``uint16`` bit patterns.  The arithmetic lives in ``fp8bw_oracle.c``; see its header
for the definition each function follows (Puro-2B part 3/7, section 3.2).
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from .build import build_oracle

_lib = None

FPROP, DGRAD, WGRAD = 0, 1, 2


def _load():
    global _lib
    if _lib is None:
        lib = C.CDLL(build_oracle())
        lib.fp8o_e4m3_decode.restype = C.c_double
        lib.fp8o_e4m3_decode.argtypes = [C.c_uint8]
        lib.fp8o_e4m3_encode.restype = C.c_uint8
        lib.fp8o_e4m3_encode.argtypes = [C.c_float]
        lib.fp8o_e4m3_encode_array.restype = None
        lib.fp8o_e4m3_encode_array.argtypes = [C.c_void_p, C.c_int64, C.c_void_p]
        lib.fp8o_quantize_group.restype = C.c_float
        lib.fp8o_quantize_group.argtypes = [C.c_void_p, C.c_int64, C.c_int64,
                                            C.c_void_p, C.c_int64]
        for name in ("fp8o_quant_act", "fp8o_quant_act_t"):
            f = getattr(lib, name)
            f.restype = C.c_int
            f.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]
        lib.fp8o_quant_weight.restype = C.c_int
        lib.fp8o_quant_weight.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p,
                                          C.c_void_p, C.c_void_p]
        lib.fp8o_gemm.restype = C.c_int
        lib.fp8o_gemm.argtypes = [C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                  C.c_void_p, C.c_int64, C.c_int64, C.c_int64,
                                  C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int]
        lib.fp8o_max_threads.restype = C.c_int
        lib.fp8o_max_threads.argtypes = []
        lib.fp8o_e8m0_exponent.restype = C.c_int
        lib.fp8o_e8m0_exponent.argtypes = [C.c_float]
        lib.fp8o_quantize_group_e8m0.restype = C.c_uint8
        lib.fp8o_quantize_group_e8m0.argtypes = [C.c_void_p, C.c_int64, C.c_int64,
                                                 C.c_void_p, C.c_int64]
        for name in ("fp8o_quant_act_e8m0", "fp8o_quant_act_t_e8m0"):
            f = getattr(lib, name)
            f.restype = C.c_int
            f.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p]
        lib.fp8o_quant_weight_e8m0.restype = C.c_int
        lib.fp8o_quant_weight_e8m0.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p,
                                               C.c_void_p, C.c_void_p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def _u16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "BF16 tensors are passed as uint16 bit patterns"
    return x


def e4m3_decode(code: int) -> float:
    return _load().fp8o_e4m3_decode(int(code) & 0xFF)


def e4m3_decode_table() -> np.ndarray:
    """Value of each of the 256 codes (float64, NaN for 0x7F/0xFF)."""
    lib = _load()
    return np.array([lib.fp8o_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v: float) -> int:
    return int(_load().fp8o_e4m3_encode(float(np.float32(v))))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """fp8o_e4m3_encode over an array of float32 values (same shape, uint8)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().fp8o_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def quantize_group(x_bf16: np.ndarray):
    """One group of BF16 values -> (codes uint8, scale float32)."""
    x = _u16(x_bf16).ravel()
    q = np.empty(x.size, dtype=np.uint8)
    s = _load().fp8o_quantize_group(_ptr(x), 1, x.size, _ptr(q), 1)
    return q, np.float32(s)


def quant_act(x_bf16: np.ndarray):
    """X[M][K] -> (Q[M][K] uint8, S[K/128][M] float32); any token count M."""
    x = _u16(x_bf16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((K // 128, M), dtype=np.float32)
    rc = _load().fp8o_quant_act(_ptr(x), M, K, _ptr(q), _ptr(s))
    if rc:
        raise ValueError(f"oracle quant_act: bad sizes {M}x{K}")
    return q, s


def quant_act_t(x_bf16: np.ndarray):
    """X[M][K] -> (Q^T[K][M] uint8, S^T[ceil(M/128)][K] float32).  M may be any token
    count: the last token group holds M mod 128 tokens, its scale taken over them."""
    x = _u16(x_bf16)
    M, K = x.shape
    qt = np.empty((K, M), dtype=np.uint8)
    st = np.empty(((M + 127) // 128, K), dtype=np.float32)
    rc = _load().fp8o_quant_act_t(_ptr(x), M, K, _ptr(qt), _ptr(st))
    if rc:
        raise ValueError(f"oracle quant_act_t: bad sizes {M}x{K}")
    return qt, st


def quant_weight(w_bf16: np.ndarray, want_t: bool = False):
    """W[N][K] -> (Q[N][K], S[N/128][K/128], Q^T[K][N] or None)."""
    w = _u16(w_bf16)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // 128, K // 128), dtype=np.float32)
    qt = np.empty((K, N), dtype=np.uint8) if want_t else None
    rc = _load().fp8o_quant_weight(_ptr(w), N, K, _ptr(q), _ptr(s),
                                   _ptr(qt) if want_t else None)
    if rc:
        raise ValueError(f"oracle quant_weight: bad sizes {N}x{K}")
    return q, s, qt


# ---- power-of-two (E8M0) scales: the MXFP8 form of section 3.2 ----

def e8m0_exponent(amax: float) -> int:
    """Exponent e of the group scale 2^e: the smallest e with amax <= 448 * 2^e,
    clamped to [-127, 127]; -127 for amax = 0."""
    return int(_load().fp8o_e8m0_exponent(float(amax)))


def e8m0_to_float(codes) -> np.ndarray:
    """E8M0 codes (uint8, e + 127) -> the float32 scales 2^e (all exact)."""
    c = np.asarray(codes, dtype=np.int64)
    return np.ldexp(np.float32(1.0), (c - 127).astype(np.int32)).astype(np.float32)


def quantize_group_e8m0(x_bf16: np.ndarray):
    """One group of BF16 values -> (codes uint8, E8M0 scale code uint8)."""
    x = _u16(x_bf16).ravel()
    q = np.empty(x.size, dtype=np.uint8)
    c = _load().fp8o_quantize_group_e8m0(_ptr(x), 1, x.size, _ptr(q), 1)
    return q, np.uint8(c)


def quant_act_e8m0(x_bf16: np.ndarray):
    """X[M][K] -> (Q[M][K] uint8, S[K/128][M] uint8 E8M0 codes)."""
    x = _u16(x_bf16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((K // 128, M), dtype=np.uint8)
    if _load().fp8o_quant_act_e8m0(_ptr(x), M, K, _ptr(q), _ptr(s)):
        raise ValueError(f"oracle quant_act_e8m0: bad sizes {M}x{K}")
    return q, s


def quant_act_t_e8m0(x_bf16: np.ndarray):
    """X[M][K] -> (Q^T[K][M] uint8, S^T[M/128][K] uint8 E8M0 codes)."""
    x = _u16(x_bf16)
    M, K = x.shape
    qt = np.empty((K, M), dtype=np.uint8)
    st = np.empty((M // 128, K), dtype=np.uint8)
    if _load().fp8o_quant_act_t_e8m0(_ptr(x), M, K, _ptr(qt), _ptr(st)):
        raise ValueError(f"oracle quant_act_t_e8m0: bad sizes {M}x{K}")
    return qt, st


def quant_weight_e8m0(w_bf16: np.ndarray, want_t: bool = False):
    """W[N][K] -> (Q[N][K], S[N/128][K/128] uint8 E8M0 codes, Q^T[K][N] or None)."""
    w = _u16(w_bf16)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // 128, K // 128), dtype=np.uint8)
    qt = np.empty((K, N), dtype=np.uint8) if want_t else None
    if _load().fp8o_quant_weight_e8m0(_ptr(w), N, K, _ptr(q), _ptr(s),
                                      _ptr(qt) if want_t else None):
        raise ValueError(f"oracle quant_weight_e8m0: bad sizes {N}x{K}")
    return q, s, qt


def gemm(mode: int, a, sa, b, sb, M: int, N: int, K: int, rows=None, nthreads: int = 0):
    """Blockwise GEMM in FP64 over dequantized operands.

    Returns (y, asum), each [len(rows) or M][N] float64, where asum is
    sum_k |ahat*bhat| (the scale of the elementwise tolerance)."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rows.size
    else:
        nr = M
    y = np.empty((nr, N), dtype=np.float64)
    asum = np.empty((nr, N), dtype=np.float64)
    rc = _load().fp8o_gemm(mode, _ptr(a), _ptr(sa), _ptr(b), _ptr(sb), M, N, K,
                           _ptr(rows) if rows is not None else None, nr,
                           _ptr(y), _ptr(asum), int(nthreads))
    if rc:
        raise ValueError(f"oracle gemm: bad arguments mode={mode} {M}x{N}x{K}")
    return y, asum


def max_threads() -> int:
    return int(_load().fp8o_max_threads())
