"""GPU parity of the decode ("skinny") kernel (qg_config.variant = 1):
warp-level MMAs with register accumulators, each CTA owning `rows` weight
rows over the whole of K and `tile_n` tokens, fed by a TMA ring.

Against the oracle on the same seeded inputs: bf16 outputs within the target
tolerance for FP8_Dynamic, W8A8_INT8 and Block_FP8; INT8 int32 accumulators
bit-exact; ragged N (inside a CTA and inside an 8-row fragment), ragged M
(several token tiles, the last partial), ragged K (the last K tile partly out
of range), rings that wrap several times, K groups with unequal tile counts,
and every rows / tile_n instantiation; two runs give the same bits."""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16
from oracle import gemm as OG

pytestmark = pytest.mark.gpu

FMTS = [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8]
IDS = {qg.QG_FP8_DYNAMIC: "fp8", qg.QG_W8A8_INT8: "int8", qg.QG_BLOCK_FP8: "block"}

CASES = [  # (M, N, K, tile_n, rows, stages)
    (1, 256, 512, 16, 32, 4),
    (5, 300, 1024, 16, 8, 8),         # N ragged inside an 8-row fragment
    (16, 1024, 2048, 16, 16, 8),      # ring of 8 over 16 K tiles
    (20, 512, 4096, 32, 64, 8),       # one K group, 32 tokens per CTA
    (33, 520, 1024, 16, 32, 4),       # three token tiles, the last partial
    (32, 768, 7168, 32, 32, 16),      # 56 K tiles through a ring of 16
    (8, 4096, 640, 16, 16, 8),        # 5 K tiles over 4 K groups
    (3, 24, 1024, 16, 32, 2),         # fewer weight rows than one CTA holds
    (2, 640, 8192, 16, 8, 64),        # K groups of 8 warps, deepest ring
    (64, 256, 2048, 32, 16, 8),       # two 32-token tiles
    # up to 8 tokens per CTA: the weight rows are the 16-row MMA operand
    (1, 256, 512, 8, 16, 8),
    (8, 1000, 2048, 8, 32, 8),        # ragged N, 4 K groups
    (3, 640, 4096, 8, 64, 8),         # 2 K groups, ring of 8 over 32 K tiles
    (13, 384, 1024, 8, 16, 16),       # two 8-token tiles, the last partial
]
RAGGED_K = [(4, 384, 528, 16, 32, 8), (9, 200, 1040, 16, 8, 8),   # K % 128 != 0 (8-bit per-row formats)
            (5, 272, 656, 8, 16, 8)]


def _cases():
    out = []
    for f in FMTS:
        for c in CASES:
            out.append((f, *c))
        if f != qg.QG_BLOCK_FP8:
            for c in RAGGED_K:
                out.append((f, *c))
    return out


ALL = _cases()


def _id(c):
    f, M, N, K, tn, rows, st = c
    return f"{IDS[f]}-M{M}-N{N}-K{K}-t{tn}-r{rows}-s{st}"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


@pytest.mark.parametrize("case", ALL, ids=[_id(c) for c in ALL])
def test_skinny_matches_the_oracle(case):
    fmt, M, N, K, tn, rows, st = case
    a, w = inputs(M, N, K, edge_rows=True)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    qa, qw = oracle_quant(fmt, a, False), oracle_quant(fmt, w, True)
    cfg = qg.skinny_config(tile_n=tn, rows=rows, stages=st)
    y = qg.run(fmt, A, W, cfg)
    assert_within_tolerance(bf16_to_np(y), oracle_y(fmt, qa, qw), _id(case))
    assert torch.count_nonzero(y[0]).item() == 0                  # the all-zero token row
    y2 = qg.run(fmt, A, W, cfg)
    assert torch.equal(y, y2)                                    # fixed summation order
    if fmt == qg.QG_W8A8_INT8:
        acc = qg.run(fmt, A, W, cfg, out_kind=qg.QG_OUT_ACC)
        np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), OG.acc_int8(qa[0], qw[0]))


def test_skinny_in_a_graph_after_the_quantiser():
    # the decode step as captured: quantise the activations, then the skinny
    # GEMM waits for them through programmatic dependent launch
    fmt, M, N, K = qg.QG_W8A8_INT8, 8, 4096, 4096
    a, w = inputs(M, N, K, edge_rows=True)
    layer_w = to_dev_bf16(w)
    layer = qg.Linear(fmt, layer_w)
    step = qg.GraphStep(layer, M, cfg=qg.skinny_config(16, 32, 32))
    outs = []
    for _ in range(3):
        step.A.copy_(to_dev_bf16(a))
        outs.append(step.replay().clone())
    torch.cuda.synchronize()
    ref = oracle_y(fmt, oracle_quant(fmt, a, False), oracle_quant(fmt, w, True))
    for y in outs:
        assert_within_tolerance(bf16_to_np(y), ref, "graph step")
        assert torch.equal(y, outs[0])
