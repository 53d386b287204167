"""Dynamic quantisers of the quantized linear layer (oracle; test-only).

Each quantiser takes bf16 bit patterns (uint16) and returns codes plus the
scales that dequantise them: x ~= dec(code) * scale.  Whenever a float
decides an integer code the oracle takes that decision in fp32, the
precision the dynamic quantiser itself works in: the amax is exact, the
scale is the correctly rounded fp32 quotient, and so is x / scale.

Formats ("Helion in the vLLM backend", first paragraph, names the three 8-bit
formats; the recipes below are the plain readings of those names):

* FP8_Dynamic: per-token (activation rows) or per-channel (weight rows) e4m3,
  scale = amax / 448.
* W8A8_INT8: symmetric int8 per token / per channel, scale = amax / 127,
  code = round-half-even(x / scale) clamped to [-127, 127].
* Block_FP8: e4m3 with one scale per 1x128 activation group and per 128x128
  weight block, scale = amax(group or block) / 448.  The 128-wide groups are
  those of the "FP8 block-scaling GEMM" of TensorRT-LLM issue 16363.
* NVFP4 (FlashInfer PR 3948, ``mm_fp4 --use_nvfp4``): e2m1 codes with an e4m3
  scale per 16 consecutive K elements and one fp32 tensor scale.  The pages
  name the format but not its recipe; the reading used here (the pages fix
  no recipe, so this reading is pinned by hand-worked blocks derived from it
  and by invariants, not by values the pages print):
  g = amax(tensor) / (448 * 6); block scale s_b = e4m3((amax_b / 6) / g);
  code = e2m1(x / (dec(s_b) * g)), and code 0 wherever dec(s_b) == 0.

An all-zero row, group, block or tensor gets scale 1 and codes 0.
"""
from __future__ import annotations

import numpy as np

from .formats import decode_e4m3, encode_e2m1, encode_e4m3, bf16_from_bits

F32 = np.float32


def _amax_scale(amax: np.ndarray, qmax: float) -> np.ndarray:
    amax = np.asarray(amax, dtype=F32)
    safe = np.where(amax > 0, amax, F32(1.0))
    s = (safe / F32(qmax)).astype(F32)               # correctly rounded fp32 division
    return np.where(amax > 0, s, F32(1.0)).astype(F32)


def per_row_fp8(x_bits: np.ndarray):
    """FP8_Dynamic rows: returns (codes uint8 [R, K], scale fp32 [R])."""
    x = bf16_from_bits(x_bits)
    s = _amax_scale(np.abs(x).max(axis=1), 448.0)
    q = encode_e4m3((x / s[:, None]).astype(F32))
    return q, s


def per_row_int8(x_bits: np.ndarray):
    """W8A8_INT8 rows: returns (codes int8 [R, K], scale fp32 [R])."""
    x = bf16_from_bits(x_bits)
    s = _amax_scale(np.abs(x).max(axis=1), 127.0)
    r = np.rint((x / s[:, None]).astype(F32))          # rint: ties to even
    q = np.clip(r, -127, 127).astype(np.int8)
    return q, s


def act_groups_fp8(x_bits: np.ndarray, group: int = 128):
    """Block_FP8 activations: 1x128 groups.
    Returns (codes uint8 [M, K], scale fp32 [M, K/128])."""
    x = bf16_from_bits(x_bits)
    M, K = x.shape
    assert K % group == 0
    G = K // group
    xg = x.reshape(M, G, group)
    s = _amax_scale(np.abs(xg).max(axis=2), 448.0)            # [M, G]
    q = encode_e4m3((xg / s[:, :, None]).astype(F32)).reshape(M, K)
    return q, s


def weight_blocks_fp8(w_bits: np.ndarray, block: int = 128):
    """Block_FP8 weights: 128x128 blocks (the last row block may be short).
    Returns (codes uint8 [N, K], scale fp32 [ceil(N/128), K/128])."""
    w = bf16_from_bits(w_bits)
    N, K = w.shape
    assert K % block == 0
    G = K // block
    NB = (N + block - 1) // block
    s = np.empty((NB, G), dtype=F32)
    q = np.empty((N, K), dtype=np.uint8)
    for b in range(NB):
        rows = w[b * block:(b + 1) * block].reshape(-1, G, block)
        s[b] = _amax_scale(np.abs(rows).max(axis=(0, 2)), 448.0)
        q[b * block:(b + 1) * block] = encode_e4m3(
            (rows / s[b][None, :, None]).astype(F32)).reshape(-1, K)
    return q, s


def nvfp4(x_bits: np.ndarray, global_amax: float | None = None, sf_vec: int = 16):
    """NVFP4 tensor quantisation (reading stated in the module docstring).

    Returns (codes uint8 [R, K] one e2m1 code per element, block scale codes
    uint8 [R, K/16] e4m3, g fp32 scalar).  ``global_amax`` replaces the
    tensor's own amax when given (a static activation scale).
    The recipe is this module's reading (the pages give none).
    """
    x = bf16_from_bits(x_bits)
    R, K = x.shape
    assert K % sf_vec == 0
    amax_t = F32(np.abs(x).max()) if global_amax is None else F32(global_amax)
    g = F32(amax_t / F32(448.0 * 6.0)) if amax_t > 0 else F32(1.0)
    xb = x.reshape(R, K // sf_vec, sf_vec)
    amax_b = np.abs(xb).max(axis=2).astype(F32)
    t = ((amax_b / F32(6.0)).astype(F32) / g).astype(F32)
    sf = encode_e4m3(t)                                        # satfinite, nearest even
    d = (decode_e4m3(sf).astype(F32) * g).astype(F32)          # fp32 product
    zero = d == 0
    d_safe = np.where(zero, F32(1.0), d)
    q = encode_e2m1((xb / d_safe[:, :, None]).astype(F32))
    q = np.where(zero[:, :, None], np.uint8(0), q).reshape(R, K)
    return q, sf, g


def nvfp4_experts(w_bits: np.ndarray, experts: int, sf_vec: int = 16):
    """Stacked mixture-of-experts weights [experts * N, K]: every expert's
    N rows quantised by ``nvfp4`` as a tensor of its own (its own amax and
    tensor scale).  Returns (codes [experts * N, K], block scale codes
    [experts * N, K/16], g float32 [experts])."""
    R = w_bits.shape[0]
    assert R % experts == 0
    N = R // experts
    parts = [nvfp4(w_bits[e * N:(e + 1) * N], sf_vec=sf_vec) for e in range(experts)]
    q = np.concatenate([p[0] for p in parts], axis=0)
    sf = np.concatenate([p[1] for p in parts], axis=0)
    g = np.array([p[2] for p in parts], dtype=F32)
    return q, sf, g

