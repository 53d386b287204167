"""GPU parity of the CTA-pair kernel (qg_config.variant = 3): Block_FP8 in the
standard orientation, clusters of two CTAs walking output tiles of 256 tokens
x tile_n channels (128 or 256) with one cta_group::2 MMA per K step.

Each group's partial is the same MMA sum as the tile kernel's, and the
promotion applies the same fp32 arithmetic in the same group order, so y is
bitwise that of the tile kernel (variant 0) with the same tile_n; and within
the target tolerance of the oracle.  Shapes cover one pair tile, an odd CTA
whose rows all lie beyond M, ragged N inside one CTA's half of the weight
rows, several tiles per pair (more tiles than SM pairs), a wider output row
(columns past N untouched) and rings of 3 to 8 stages."""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16

pytestmark = pytest.mark.gpu

FMT = qg.QG_BLOCK_FP8
CASES = [  # (M, N, K, tile_n, stages)
    (256, 256, 256, 256, 4),        # one pair tile
    (300, 200, 640, 256, 4),        # the odd CTA of the second row block: rows 384.. > M
    (260, 392, 1024, 128, 3),       # ragged N inside the odd CTA's weight half
    (1024, 768, 2048, 128, 8),
    (4096, 1024, 1024, 256, 6),     # 64 tiles: one per pair
    (4096, 5120, 1024, 256, 3),     # 320 tiles over the SM pairs: several per pair
    (520, 1160, 5120, 256, 6),      # long K, ragged N (the last tile's second slice)
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


def _id(c):
    return f"M{c[0]}-N{c[1]}-K{c[2]}-t{c[3]}-s{c[4]}"


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_pair_matches_the_tile_kernel_and_oracle(case):
    M, N, K, tn, st = case
    a, w = inputs(M, N, K)
    A = qg.quantize_act(FMT, to_dev_bf16(a))
    W = qg.quantize_weight(FMT, to_dev_bf16(w))
    ldy = N + 16
    buf = torch.full((M, ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = buf[:, :N]
    qg.run(FMT, A, W, qg.pair_config(tile_n=tn, stages=st), out=y)
    y_tile = qg.run(FMT, A, W, qg.make_config(split_k=1, swap_ab=0, tile_n=tn, stages=3, reduce_mode=0))
    torch.cuda.synchronize()
    assert torch.isnan(buf[:, N:]).all(), "a store crossed the row's last channel"
    assert torch.equal(y, y_tile)
    assert torch.equal(y, qg.run(FMT, A, W, qg.pair_config(tile_n=tn, stages=st)))
    rows = np.arange(M) if M <= 600 else np.random.default_rng(M).choice(M, 24, replace=False)
    qa, qw = oracle_quant(FMT, a[rows], False), oracle_quant(FMT, w, True)
    assert_within_tolerance(bf16_to_np(y[torch.from_numpy(rows).cuda()]), oracle_y(FMT, qa, qw), _id(case))


def test_pair_refuses_what_it_does_not_cover():
    M, N, K = 256, 512, 512
    a, w = inputs(M, N, K)
    A = qg.quantize_act(FMT, to_dev_bf16(a))
    W = qg.quantize_weight(FMT, to_dev_bf16(w))
    with pytest.raises(qg.QGemmError):                 # raw accumulators: the tile store is bf16 only
        qg.run(FMT, A, W, qg.pair_config(), out_kind=qg.QG_OUT_ACC)
    with pytest.raises(qg.QGemmError):                 # the output row pitch must suit a tensor map
        qg.run(FMT, A, W, qg.pair_config(), out=torch.empty(M, N + 4, dtype=torch.bfloat16, device="cuda")[:, :N])
    A8 = qg.quantize_act(qg.QG_FP8_DYNAMIC, to_dev_bf16(a))
    W8 = qg.quantize_weight(qg.QG_FP8_DYNAMIC, to_dev_bf16(w))
    with pytest.raises(qg.QGemmError):                 # Block_FP8 only
        qg.run(qg.QG_FP8_DYNAMIC, A8, W8, qg.pair_config())


def test_pair_in_a_graph_after_the_quantiser():
    # programmatic dependent launch: the promotion reads the activation
    # scales only after the quantiser that writes them has completed
    M, N, K = 2048, 2048, 1024
    a, w = inputs(M, N, K)
    layer = qg.Linear(FMT, to_dev_bf16(w))
    step = qg.GraphStep(layer, M, cfg=qg.pair_config(256, 4))
    outs = []
    for _ in range(3):
        step.A.copy_(to_dev_bf16(a))
        outs.append(step.replay().clone())
    torch.cuda.synchronize()
    rows = np.random.default_rng(1).choice(M, 16, replace=False)
    ref = oracle_y(FMT, oracle_quant(FMT, a[rows], False), oracle_quant(FMT, w, True))
    for y in outs:
        assert torch.equal(y, outs[0])
        assert_within_tolerance(bf16_to_np(y[torch.from_numpy(rows).cuda()]), ref, "graph step")
