"""Seeded synthetic BF16 inputs shaped like Qwen3-1.7B linear-layer operands.

This module only draws random numbers; it holds none of the quantization or GEMM
arithmetic.  The same bytes feed both the CUDA path and the CPU oracle.

Recipe (stated once, used everywhere):
  * A counter-based splitmix64 stream (Steele, Lea and Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014): element i of the stream with
    state ``s`` is ``mix(s + (i + 1) * 0x9E3779B97F4A7C15)``.
  * Standard normals by the Box-Muller transform on consecutive pairs:
    ``u1 = (v0 >> 11 + 1) * 2^-53`` in (0, 1], ``u2 = (v1 >> 11) * 2^-53`` in [0, 1),
    ``r = sqrt(-2 ln u1)``, giving ``r cos(2 pi u2)`` and ``r sin(2 pi u2)``.
  * Values are scaled by the standard deviation, outlier columns (1% of the input
    channels, chosen by a seeded permutation) are multiplied by 20, and the FP64
    result is rounded once to BF16 (round to nearest, ties to even).
  * The seed of tensor ``t`` of workload ``c`` is the first output of a stream with
    state ``c * 1000 + t``.

BF16 tensors are returned as numpy ``uint16`` bit patterns.
"""
from __future__ import annotations

import os

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream(state: int, start: int, count: int) -> np.ndarray:
    """Elements start .. start+count-1 of the splitmix64 stream with this state."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(state & 0xFFFFFFFFFFFFFFFF) + idx * GOLDEN
    return _mix(z)


def seed_for(workload: int, tensor: int) -> int:
    return int(stream(workload * 1000 + tensor, 0, 1)[0])


def standard_normal(seed: int, count: int, start: int = 0) -> np.ndarray:
    """count standard normals (float64); start must be even."""
    assert start % 2 == 0
    npairs = (count + 1) // 2
    v = stream(seed, start, 2 * npairs)
    u1 = ((v[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (v[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * np.pi * u2)
    out[1::2] = r * np.sin(2.0 * np.pi * u2)
    return out[:count]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round FP64 values once to BF16 (nearest, ties to even); return bit patterns.

    Valid for finite values whose BF16 rounding is a normal BF16 number or zero,
    which covers every value this generator draws."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    with np.errstate(over="ignore"):
        b = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f = b.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def outlier_columns(seed: int, ncols: int, frac: float = 0.01) -> np.ndarray:
    """floor(frac * ncols) column indices from a seeded permutation."""
    n = int(np.floor(frac * ncols))
    keys = stream(seed ^ 0x5DEECE66D, 0, ncols)
    return np.sort(np.argsort(keys, kind="stable")[:n])


def normal_bf16(rows: int, cols: int, std: float, seed: int,
                outliers: bool = False, outlier_gain: float = 20.0) -> np.ndarray:
    """[rows][cols] BF16 (uint16 bits) ~ N(0, std); with outliers, 1% of the
    columns are multiplied by outlier_gain before rounding to BF16."""
    total = rows * cols
    out = np.empty(total, dtype=np.uint16)
    gain = None
    if outliers:
        gain = np.ones(cols, dtype=np.float64)
        gain[outlier_columns(seed, cols)] = outlier_gain

    def fill(s):
        n = min(_CHUNK, total - s)
        z = standard_normal(seed, n, start=s) * std
        if gain is not None:
            z *= gain[(np.arange(s, s + n) % cols)]
        out[s:s + n] = f64_to_bf16_bits(z)

    starts = range(0, total, _CHUNK)
    if total > 4 * _CHUNK:
        # chunks are independent slices of the counter-based stream, so filling
        # them on several threads gives the same bytes
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    else:
        for s in starts:
            fill(s)
    return out.reshape(rows, cols)


def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
