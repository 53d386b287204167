"""Bit-level number formats used by the quantized GEMM (oracle; test-only).

* E4M3 ("fp8 e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
  Exponent field 0 holds subnormals m * 2^-9; the all-ones pattern
  S.1111.111 is NaN; there is no infinity; the largest finite magnitude is
  1.75 * 2^8 = 448 (code 0x7E).  Source: OCP 8-bit Floating Point
  Specification (OFP8) rev 1.0, E4M3 encoding.  The linear backend's formats
  FP8_Dynamic and Block_FP8 ("Helion in the vLLM backend", first paragraph)
  and the NVFP4 block scales use it.
* E2M1 ("fp4"): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; the
  eight magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Source: OCP Microscaling
  Formats (MX) v1.0, FP4 E2M1 element type; used by ``mm_fp4 --use_nvfp4``
  in FlashInfer PR 3948.
* bf16 output rounding: round to nearest, ties to even, of the exact fp64
  value.

Encoders are nearest-value searches over the decode table (saturating to the
largest finite value, ties to the even code), independent of any hardware
conversion instruction.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def _e4m3_value(code: int) -> float:
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9          # subnormal: 0.mmm * 2^(1-7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def _e2m1_value(code: int) -> float:
    sign = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return sign * m * 0.5                # subnormal: 0.m * 2^(1-1)
    return sign * (1.0 + m / 2.0) * 2.0 ** (e - 1)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)

# Non-negative finite codes in increasing value order: for both formats the
# code of a non-negative value is its position (the encodings are monotone).
_E4M3_POS = E4M3_TABLE[:0x7F]           # codes 0x00 .. 0x7E
_E2M1_POS = E2M1_TABLE[:8]              # codes 0x0 .. 0x7


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def decode_e2m1(codes: np.ndarray) -> np.ndarray:
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


def _nearest_even(x: np.ndarray, pos_values: np.ndarray, sign_bit: int) -> np.ndarray:
    """Nearest representable value of |x| (saturating at the largest finite
    one), ties broken to the even code; the sign of x (including -0) sets the
    sign bit.  ``x`` must be finite."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), pos_values[-1])
    hi = np.searchsorted(pos_values, a, side="left")       # pos[hi-1] < a <= pos[hi]
    hi = np.minimum(hi, len(pos_values) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - pos_values[lo]
    d_hi = pos_values[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint16)
    code = np.where(np.signbit(x), code | sign_bit, code)
    return code.astype(np.uint8)


def encode_e4m3(x: np.ndarray) -> np.ndarray:
    """fp32/fp64 -> E4M3 code, round to nearest even, saturating to +-448."""
    return _nearest_even(x, _E4M3_POS, 0x80)


def encode_e2m1(x: np.ndarray) -> np.ndarray:
    """fp32/fp64 -> E2M1 code (0..15), round to nearest even, saturating to +-6."""
    return _nearest_even(x, _E2M1_POS, 0x8)


def bf16_round(y: np.ndarray) -> np.ndarray:
    """Exact fp64 values -> bf16 (nearest, ties to even), returned as fp64.

    bf16 keeps 8 significant bits and fp32's exponent range; values below
    2^-126 are rounded on the subnormal grid 2^-133; magnitudes that round
    above the largest finite bf16 become infinities.
    """
    y = np.asarray(y, dtype=np.float64)
    out = np.zeros_like(y)
    finite = np.isfinite(y) & (y != 0)
    yf = y[finite]
    _, e = np.frexp(yf)                                     # |yf| in [2^(e-1), 2^e)
    quantum_exp = np.maximum(e - 8, -133)
    q = np.ldexp(np.rint(np.ldexp(yf, -quantum_exp)), quantum_exp)  # rint: half to even
    q = np.where(np.abs(q) > 3.3895313892515355e38, np.copysign(np.inf, q), q)
    out[finite] = q
    out[~finite] = y[~finite]
    return out


def bf16_bits(y_rounded: np.ndarray) -> np.ndarray:
    """bf16-representable fp64 values -> their 16-bit patterns."""
    f = np.asarray(y_rounded, dtype=np.float64).astype(np.float32)   # exact
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_from_bits(bits: np.ndarray) -> np.ndarray:
    """16-bit bf16 patterns -> fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
