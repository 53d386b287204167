"""GPU parity of the persistent kernel (qg_config.variant = 2): the 8-bit
formats in the standard orientation, one CTA per SM walking the 128 x tile_n
output tiles (FP8_Dynamic / W8A8_INT8 with two TMEM accumulators, Block_FP8
with its promotion's group buffers).

Its MMAs accumulate each tile's K tiles in the tile kernel's order and its
epilogue applies the same fp32 arithmetic, so y is bitwise that of the tile
kernel (variant 0) with the same tile_n; and within the target tolerance of
the oracle.  Shapes cover one tile, several tiles per CTA (more tiles than
SMs), ragged M and N, K with a partial last tile, a wider output row (columns
past N untouched), and rings shallower than a tile's K tiles."""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import FMT_NAMES, assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16

pytestmark = pytest.mark.gpu

CASES = [  # (format, M, N, K, tile_n, stages)
    (qg.QG_FP8_DYNAMIC, 128, 256, 512, 256, 2),       # one tile
    (qg.QG_FP8_DYNAMIC, 300, 520, 1024, 128, 3),      # ragged M and N
    (qg.QG_W8A8_INT8, 1000, 2048, 2048, 256, 3),
    (qg.QG_W8A8_INT8, 4096, 5120, 512, 256, 2),       # 640 tiles: several per CTA
    (qg.QG_FP8_DYNAMIC, 2048, 4096, 1024, 128, 4),    # 512 tiles of 128
    (qg.QG_W8A8_INT8, 129, 392, 272, 128, 2),         # K % 128 != 0: a partial last K tile
    (qg.QG_FP8_DYNAMIC, 520, 1536, 4096, 256, 3),
    # Block_FP8: promotion into register accumulators, group buffers shared by consecutive tiles
    (qg.QG_BLOCK_FP8, 300, 640, 1024, 256, 3),
    (qg.QG_BLOCK_FP8, 2048, 2560, 2048, 256, 3),       # 320 tiles: several per CTA
    (qg.QG_BLOCK_FP8, 1000, 1152, 512, 128, 3),
    (qg.QG_BLOCK_FP8, 4096, 5120, 5120, 256, 3),
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


def _id(c):
    return f"{FMT_NAMES[c[0]]}-M{c[1]}-N{c[2]}-K{c[3]}-t{c[4]}-s{c[5]}"


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_persistent_matches_the_tile_kernel_and_oracle(case):
    fmt, M, N, K, tn, st = case
    a, w = inputs(M, N, K)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    ldy = N + 16
    buf = torch.full((M, ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = buf[:, :N]
    qg.run(fmt, A, W, qg.persist_config(tile_n=tn, stages=st), out=y)
    # the tile kernel stages its output tile in the ring: at least 3 stages
    y_tile = qg.run(fmt, A, W, qg.make_config(split_k=1, swap_ab=0, tile_n=tn, stages=max(st, 3), reduce_mode=0))
    torch.cuda.synchronize()
    assert torch.isnan(buf[:, N:]).all(), "a store crossed the row's last channel"
    assert torch.equal(y, y_tile)
    assert torch.equal(y, qg.run(fmt, A, W, qg.persist_config(tile_n=tn, stages=st)))
    rows = np.arange(M) if M <= 600 else np.random.default_rng(M).choice(M, 24, replace=False)
    qa, qw = oracle_quant(fmt, a[rows], False), oracle_quant(fmt, w, True)
    assert_within_tolerance(bf16_to_np(y[torch.from_numpy(rows).cuda()]), oracle_y(fmt, qa, qw), _id(case))


def test_persistent_refuses_what_it_does_not_cover():
    fmt, M, N, K = qg.QG_W8A8_INT8, 256, 512, 512
    a, w = inputs(M, N, K)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    with pytest.raises(qg.QGemmError):                 # raw accumulators: the tile store is bf16 only
        qg.run(fmt, A, W, qg.persist_config(), out_kind=qg.QG_OUT_ACC)
    An = qg.quantize_act(qg.QG_NVFP4, to_dev_bf16(a))
    Wn = qg.quantize_weight(qg.QG_NVFP4, to_dev_bf16(w))
    with pytest.raises(qg.QGemmError):                 # the 8-bit formats only
        qg.run(qg.QG_NVFP4, An, Wn, qg.persist_config())


def test_persistent_in_a_graph_after_the_quantiser():
    # programmatic dependent launch: the kernel reads the activations (and
    # their scales) only after the quantiser that writes them has completed
    fmt, M, N, K = qg.QG_FP8_DYNAMIC, 2048, 2048, 1024
    a, w = inputs(M, N, K)
    layer = qg.Linear(fmt, to_dev_bf16(w))
    step = qg.GraphStep(layer, M, cfg=qg.persist_config(256, 3))
    outs = []
    for _ in range(3):
        step.A.copy_(to_dev_bf16(a))
        outs.append(step.replay().clone())
    torch.cuda.synchronize()
    rows = np.random.default_rng(1).choice(M, 16, replace=False)
    ref = oracle_y(fmt, oracle_quant(fmt, a[rows], False), oracle_quant(fmt, w, True))
    for y in outs:
        assert torch.equal(y, outs[0])
        assert_within_tolerance(bf16_to_np(y[torch.from_numpy(rows).cuda()]), ref, "graph step")
