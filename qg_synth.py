"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This module holds no arithmetic of the quantized GEMM itself: it only draws
bf16 matrices.  Both the CUDA path and the CPU oracle receive exactly the same
bf16 bits from here, so any difference between them comes from the method.

Recipe (the workloads of the quantized linear layer at LLM-decode shapes):

* counter-based splitmix64: word j of stream ``seed`` is
  ``mix64((seed << 48) + (j + 1) * 0x9E3779B97F4A7C15 mod 2**64)`` with the
  published splitmix64 finaliser (Steele, Lea, Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014);
* Box-Muller in fp64: normal i uses words 2i and 2i+1,
  ``u1 = ((w0 >> 11) + 0.5) * 2**-53``, ``u2 = (w1 >> 11) * 2**-53``,
  ``z = sqrt(-2 ln u1) * cos(2 pi u2)``;
* value = ``std * z`` rounded fp64 -> fp32 (round to nearest even) -> bf16
  (round to nearest even on the fp32 bits).

Activations A[M, K] use seed 0 and std 1; weights W[N, K] use seed 1 and
std 0.02.  Tests add structure on top (an all-zero row, a 100x outlier
channel) explicitly.
"""
from __future__ import annotations

import os

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

SEED_A = 0
SEED_W = 1
STD_A = 1.0
STD_W = 0.02


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_words(seed: int, start: int, count: int) -> np.ndarray:
    """Words ``start .. start+count-1`` of the counter-based stream ``seed``."""
    j = np.arange(start, start + count, dtype=np.uint64)
    base = np.uint64((int(seed) << 48) & 0xFFFFFFFFFFFFFFFF)
    with np.errstate(over="ignore"):
        return _mix64(base + (j + np.uint64(1)) * _GAMMA)


def normal_fp64(seed: int, count: int, start: int = 0) -> np.ndarray:
    """``count`` standard normals (fp64) starting at normal index ``start``."""
    w = splitmix64_words(seed, 2 * start, 2 * count)
    w0 = w[0::2]
    w1 = w[1::2]
    u1 = ((w0 >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    u2 = (w1 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    nan = np.isnan(x)
    r = np.where(nan, np.uint32(0x7FC0), r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_matrix(seed: int, rows: int, cols: int, std: float) -> np.ndarray:
    """A [rows, cols] matrix of bf16 values, returned as uint16 bit patterns.
    Large matrices are drawn in independent chunks on a thread pool; element
    i is always normal i of the stream, so the result does not depend on the
    chunking."""
    n = rows * cols
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 22

    def fill(start):
        cnt = min(chunk, n - start)
        z = normal_fp64(seed, cnt, start) * std
        out[start:start + cnt] = f32_to_bf16_bits(z.astype(np.float32))

    starts = range(0, n, chunk)
    if n <= chunk:
        fill(0)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4)) as ex:
            list(ex.map(fill, starts))
    return out.reshape(rows, cols)


def activations(M: int, K: int, seed: int = SEED_A) -> np.ndarray:
    """A ~ N(0, 1) as bf16 bits [M, K]."""
    return bf16_matrix(seed, M, K, STD_A)


def weights(N: int, K: int, seed: int = SEED_W) -> np.ndarray:
    """W ~ N(0, 0.02^2) as bf16 bits [N, K]."""
    return bf16_matrix(seed, N, K, STD_W)


def with_edge_rows(a_bits: np.ndarray) -> np.ndarray:
    """Test-only structure: row 0 all zero and, if there are >= 3 rows, row 2
    carries one channel scaled by 100 (an activation outlier)."""
    a = a_bits.copy()
    if a.shape[0] >= 1:
        a[0, :] = 0
    if a.shape[0] >= 3 and a.shape[1] >= 8:
        v = bf16_bits_to_f32(a[2:3, 5:6]) * np.float32(100.0)
        a[2, 5] = f32_to_bf16_bits(v)[0, 0]
    return a
