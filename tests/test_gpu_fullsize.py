"""GPU parity at the workloads' full sizes, in the launch configuration the
bench times (per-shape table dispatch, else the built-in default).

The whole CUDA output is produced; the oracle computes a sample of it (a few
token rows, including the all-zero row and the outlier row, against whole
128-channel blocks, one of them the ragged tail), and properties that hold
at any size are checked on all of it: the quantiser codes and scales are
bit-exact for the full tensors, no output is NaN or infinite, the all-zero
token row is exactly zero.
"""
import os

import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import (assert_within_tolerance, bf16_to_np, gpu_codes, inputs, oracle_quant, oracle_y,
                      to_dev_bf16)

pytestmark = pytest.mark.gpu

TABLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                     "precision_quantized_gemm_b200", "tables", "b200.qgt")

CASES = [  # (format, M, N, K): one per workload family, at its own sizes
    (qg.QG_FP8_DYNAMIC, 16, 2048, 2048),
    (qg.QG_W8A8_INT8, 1, 4096, 4096),
    (qg.QG_W8A8_INT8, 8, 4096, 4096),
    (qg.QG_W8A8_INT8, 32, 4096, 4096),
    (qg.QG_BLOCK_FP8, 16, 4608, 7168),
    (qg.QG_BLOCK_FP8, 4, 5120, 640),
    (qg.QG_BLOCK_FP8, 32, 2560, 8192),
    (qg.QG_NVFP4, 8, 1792, 5120),
    (qg.QG_NVFP4, 512, 5120, 2048),
    (qg.QG_NVFP4, 64, 1280, 8192),
    (qg.QG_FP8_DYNAMIC, 32, 8192, 8192),
    (qg.QG_BLOCK_FP8, 4096, 5120, 5120),
]


@pytest.fixture(scope="module")
def table():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return qg.Table(TABLE) if os.path.exists(TABLE) else None


def _cfg(table, fmt, M, N, K):
    if table is not None:
        return table.dispatch(fmt, M, N, K)[0]
    return qg.qgemm_default_config(fmt, M, N, K)


def _sample_rows(M):
    rows = {0, min(2, M - 1), M // 2, M - 1}       # zero row, outlier row, middle, last
    return sorted(r for r in rows if 0 <= r < M)


def _sample_cols(N):
    nb = (N + 127) // 128
    blocks = sorted({0, nb // 2, nb - 1})          # first, middle and the (ragged) last block
    return np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in blocks])


def _sub_weights(fmt, qw, cols):
    """Oracle weight operands (per-channel formats) restricted to channels `cols`."""
    if fmt == qg.QG_NVFP4:
        return qw[0][cols], qw[1][cols], qw[2]
    return qw[0][cols], qw[1][cols]


@pytest.mark.parametrize("fmt,M,N,K", CASES, ids=[f"{f}-{M}x{N}x{K}" for f, M, N, K in CASES])
def test_fullsize_sampled_parity(table, fmt, M, N, K):
    a, w = inputs(M, N, K, edge_rows=True)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    cfg = _cfg(table, fmt, M, N, K)
    y = qg.run(fmt, A, W, cfg)
    torch.cuda.synchronize()
    # properties over the whole output
    assert torch.isfinite(y.float()).all()
    assert torch.count_nonzero(y[0]).item() == 0                 # the all-zero token row
    # quantisers: bit-exact on the full tensors
    qa = oracle_quant(fmt, a, False)
    qw = oracle_quant(fmt, w, True)
    for g, o in zip(gpu_codes(fmt, A), qa):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(o))
    for g, o in zip(gpu_codes(fmt, W), qw):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(o))
    # sampled outputs against the oracle
    rows = _sample_rows(M)
    cols = _sample_cols(N)
    if fmt == qg.QG_NVFP4:
        qa_s = (qa[0][rows], qa[1][rows], qa[2])
    else:
        qa_s = (qa[0][rows], qa[1][rows])
    if fmt == qg.QG_BLOCK_FP8:
        blocks = sorted(set(int(c) // 128 for c in cols))
        ref = np.concatenate([oracle_y(fmt, qa_s, (qw[0][b * 128:min(N, b * 128 + 128)], qw[1][b:b + 1]))
                              for b in blocks], axis=1)
    else:
        ref = oracle_y(fmt, qa_s, _sub_weights(fmt, qw, cols))
    got = bf16_to_np(y)[np.ix_(rows, cols)]
    assert_within_tolerance(got, ref, f"{fmt} {M}x{N}x{K} cfg {cfg.as_dict()}")
