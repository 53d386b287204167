"""Every configured shape against the oracle, in the configuration the
shipped table dispatches (the launch the bench times).

The workloads: FP8_Dynamic 16 x 2048 x 2048; W8A8_INT8 M in {1, 8, 32} at
4096^2; Block_FP8 M in {1, 4, 16, 32} x 4 (N, K); NVFP4 M in {1, 8, 64, 512} x
4 (N, K); the FP8_Dynamic and Block_FP8 sweep (M in {1 .. 32} x 12 (N, K)
pairs of the FlashInfer mm_fp4 shape list); Block_FP8 M in {4096, 16384} at
5120^2.

The whole CUDA output is produced.  The oracle computes a sample: token rows
0 (all zero), 2 (a 100x outlier channel), M/2 and M-1 against whole
128-channel blocks (first, middle and the ragged last).  Scales are local to
a weight row (per channel), a 128-row block (Block_FP8) or a 16-element block
with the tensor amax (NVFP4), so the oracle quantises only the sampled rows
and blocks, and the library's codes and scales of those rows are compared
bit for bit.  Over all of y: finite values and an exactly zero row 0."""
import os

import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
import qg_synth
from gpu_util import assert_within_tolerance, bf16_to_np, gpu_codes, oracle_y, to_dev_bf16
from oracle import formats as OF
from oracle import quant as OQ

pytestmark = pytest.mark.gpu

TABLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                     "precision_quantized_gemm_b200", "tables", "b200.qgt")
SWEEP_NK = [(896, 5120), (1024, 7168), (1280, 8192), (1792, 5120), (2560, 8192), (4096, 4096),
            (4608, 7168), (5120, 640), (5120, 2048), (6144, 4096), (7168, 2048), (8192, 8192)]
FAMILIES = [
    (qg.QG_FP8_DYNAMIC, [16], [(2048, 2048)]),
    (qg.QG_W8A8_INT8, [1, 8, 32], [(4096, 4096)]),
    (qg.QG_BLOCK_FP8, [1, 4, 16, 32], [(512, 7168), (4608, 7168), (5120, 640), (2560, 8192)]),
    (qg.QG_NVFP4, [1, 8, 64, 512], [(896, 1024), (1792, 5120), (5120, 2048), (1280, 8192)]),
    (qg.QG_FP8_DYNAMIC, [1, 2, 4, 8, 16, 32], SWEEP_NK),
    (qg.QG_BLOCK_FP8, [1, 2, 4, 8, 16, 32], SWEEP_NK),
    (qg.QG_BLOCK_FP8, [4096, 16384], [(5120, 5120)]),
]
# ordered by weight shape so that each weight matrix is drawn and quantised once
SHAPES = sorted({(f, M, N, K) for f, Ms, NKs in FAMILIES for (N, K) in NKs for M in Ms},
                key=lambda s: (s[2], s[3], s[0], s[1]))


@pytest.fixture(scope="module")
def table():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    t = qg.Table(TABLE) if os.path.exists(TABLE) else None
    yield t
    assert qg.qgemm_device_error() == qg.QG_OK


_WCACHE = {}


def _weights_dev(fmt, N, K):
    """bf16 weights (seeded generator) and the library's quantised operand,
    kept while the tests of one (N, K) run."""
    if _WCACHE.get("nk") != (N, K):
        _WCACHE.clear()
        torch.cuda.empty_cache()
        _WCACHE["nk"] = (N, K)
        _WCACHE["w"] = qg_synth.weights(N, K)
    if fmt not in _WCACHE:
        _WCACHE[fmt] = qg.quantize_weight(fmt, to_dev_bf16(_WCACHE["w"]))
    return _WCACHE["w"], _WCACHE[fmt]


def _rows(M):
    return sorted({r for r in (0, min(2, M - 1), M // 2, M - 1) if 0 <= r < M})


def _blocks(N):
    nb = (N + 127) // 128
    return sorted({0, nb // 2, nb - 1})


def _quant_rows(fmt, x_bits, rows, is_weight, tensor_amax=None):
    """The oracle's quantisation of the given rows only (scales are local to
    a row, a 128-row weight block or a 16-element block)."""
    sub = x_bits[rows]
    if fmt == qg.QG_FP8_DYNAMIC:
        return OQ.per_row_fp8(sub)
    if fmt == qg.QG_W8A8_INT8:
        return OQ.per_row_int8(sub)
    if fmt == qg.QG_BLOCK_FP8:
        return OQ.weight_blocks_fp8(sub) if is_weight else OQ.act_groups_fp8(sub)
    return OQ.nvfp4(sub, global_amax=tensor_amax)


def _tensor_amax(bits):
    return float(np.abs(OF.bf16_from_bits(bits)).max())


@pytest.mark.parametrize("shape", SHAPES, ids=[f"f{f}-{M}x{N}x{K}" for f, M, N, K in SHAPES])
def test_configured_shape_matches_the_oracle(table, shape):
    fmt, M, N, K = shape
    w, W = _weights_dev(fmt, N, K)
    a = qg_synth.with_edge_rows(qg_synth.activations(M, K))
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    cfg = table.dispatch(fmt, M, N, K)[0] if table is not None else qg.qgemm_default_config(fmt, M, N, K)
    y = qg.run(fmt, A, W, cfg)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    assert torch.count_nonzero(y[0]).item() == 0
    rows = _rows(M)
    blocks = _blocks(N)
    # oracle operands of the sampled token rows and weight blocks
    amax_a = _tensor_amax(a) if fmt == qg.QG_NVFP4 else None
    amax_w = _tensor_amax(w) if fmt == qg.QG_NVFP4 else None
    qa = _quant_rows(fmt, a, rows, False, amax_a)
    wrows = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in blocks])
    # library codes and scales at the same rows, bit for bit
    ga = gpu_codes(fmt, A)
    gw = gpu_codes(fmt, W)
    np.testing.assert_array_equal(ga[0][rows], qa[0])
    np.testing.assert_array_equal(np.asarray(ga[1])[rows], np.asarray(qa[1]))
    ref_parts = []
    for b in blocks:
        br = np.arange(b * 128, min(N, b * 128 + 128))
        qw = _quant_rows(fmt, w, br, True, amax_w)
        np.testing.assert_array_equal(gw[0][br], qw[0])
        if fmt == qg.QG_BLOCK_FP8:
            np.testing.assert_array_equal(np.asarray(gw[1])[b:b + 1], np.asarray(qw[1]))
        else:
            np.testing.assert_array_equal(np.asarray(gw[1])[br], np.asarray(qw[1]))
        if fmt == qg.QG_NVFP4:
            assert ga[2] == qa[2] and gw[2] == qw[2]
        ref_parts.append(oracle_y(fmt, qa, qw))
    ref = np.concatenate(ref_parts, axis=1)
    got = bf16_to_np(y)[np.ix_(rows, wrows)]
    assert_within_tolerance(got, ref, f"f{fmt} {M}x{N}x{K} cfg {cfg.as_dict()}")
