"""Helpers shared by the GPU parity tests: inputs to the device, the oracle
on the same bf16 bits, layout unpacking of the library's buffers, and the
tolerance of the quantized GEMM."""
from __future__ import annotations

import functools

import numpy as np
import torch

import precision_quantized_gemm_b200 as qg
import qg_synth
from oracle import formats as OF
from oracle import gemm as OG
from oracle import quant as OQ

FMT_NAMES = {qg.QG_FP8_DYNAMIC: "fp8", qg.QG_W8A8_INT8: "int8", qg.QG_BLOCK_FP8: "block", qg.QG_NVFP4: "nvfp4"}


@functools.lru_cache(maxsize=64)
def _acts(M, K, seed):
    return qg_synth.activations(M, K, seed)


@functools.lru_cache(maxsize=16)
def _weights(N, K, seed):
    return qg_synth.weights(N, K, seed)


def inputs(M, N, K, edge_rows=False, seed_a=qg_synth.SEED_A, seed_w=qg_synth.SEED_W):
    a = _acts(M, K, seed_a)
    if edge_rows:
        a = qg_synth.with_edge_rows(a)
    return a, _weights(N, K, seed_w)


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def unpack_nvfp4_codes(qbytes: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Packed e2m1 [rows, K/2] bytes (element 2j in the low nibble) -> codes [rows, K]."""
    b = qbytes.reshape(rows, K // 2)
    out = np.empty((rows, K), np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def unpack_sf_128x4(sf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """128x4 tiled e4m3 scale layout (see include/qgemm.h) -> logical [rows, K/16]."""
    C = ((K + 255) // 256) * 16
    r = np.arange(rows)[:, None]
    c = np.arange(K // 16)[None, :]
    atom = (r // 128) * (C // 4) + c // 4
    off = atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return sf[off]


def sf_padding_is_zero(sf: np.ndarray, rows: int, K: int) -> bool:
    C = ((K + 255) // 256) * 16
    R = ((rows + 127) // 128) * 128
    r = np.arange(R)[:, None]
    c = np.arange(C)[None, :]
    atom = (r // 128) * (C // 4) + c // 4
    off = atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    pad = (r >= rows) | (c >= K // 16)
    return bool(np.all(sf[off[np.broadcast_to(pad, off.shape)]] == 0))


def gpu_codes(fmt, op: qg.Operand):
    """The library's codes/scales of an operand as the oracle's logical arrays."""
    torch.cuda.synchronize()
    q = op.q.cpu().numpy()
    s = op.scale.cpu().numpy()
    rows, K = op.rows, op.K
    if fmt == qg.QG_NVFP4:
        return (unpack_nvfp4_codes(q, rows, K), unpack_sf_128x4(s, rows, K),
                np.float32(op.global_scale.cpu().numpy()[0]))
    sc = s.view(np.float32)
    if fmt == qg.QG_W8A8_INT8:
        return q.view(np.int8).reshape(rows, K), sc
    if fmt == qg.QG_BLOCK_FP8:
        g = K // 128
        nr = (rows + 127) // 128 if op.is_weight else rows
        return q.reshape(rows, K), sc.reshape(nr, g)
    return q.reshape(rows, K), sc


def oracle_quant(fmt, bits, is_weight):
    if fmt == qg.QG_FP8_DYNAMIC:
        return OQ.per_row_fp8(bits)
    if fmt == qg.QG_W8A8_INT8:
        return OQ.per_row_int8(bits)
    if fmt == qg.QG_BLOCK_FP8:
        return OQ.weight_blocks_fp8(bits) if is_weight else OQ.act_groups_fp8(bits)
    return OQ.nvfp4(bits)


def oracle_y(fmt, qa, qw):
    """Oracle y (fp64 values of the bf16 result) from oracle-quantised operands."""
    if fmt == qg.QG_FP8_DYNAMIC:
        return OG.fp8_dynamic(qa[0], qa[1], qw[0], qw[1])
    if fmt == qg.QG_W8A8_INT8:
        return OG.w8a8_int8(qa[0], qa[1], qw[0], qw[1])
    if fmt == qg.QG_BLOCK_FP8:
        return OG.block_fp8(qa[0], qa[1], qw[0], qw[1])
    return OG.nvfp4(qa[0], qa[1], qa[2], qw[0], qw[1], qw[2])


def tolerance_violations(y: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Mask of elements outside |y - ref| <= 0.01 |ref| + 0.01 rms(ref row)."""
    rms = np.sqrt(np.mean(ref.astype(np.float64) ** 2, axis=1, keepdims=True))
    return ~(np.abs(y.astype(np.float64) - ref) <= 0.01 * np.abs(ref) + 0.01 * rms)


def assert_within_tolerance(y: np.ndarray, ref: np.ndarray, what=""):
    bad = tolerance_violations(y, ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                             f"first at {tuple(i)}: got {y[tuple(i)]}, want {ref[tuple(i)]}")


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)
