"""GPU parity of the TMA-store epilogue, through the C ABI.

Launches in the standard orientation with split_k = 1, tile_n >= 64 and bf16
output write their tile through a tensor map of y (128-byte swizzled boxes of
64 channels).  The switch qgemm_set_tma_store(0) restores the thread stores;
both must give the same bits, the tensor map must clip at M and N (a wider
output row keeps its other columns), and the result is within the target
tolerance of the oracle."""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import FMT_NAMES, assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16

pytestmark = pytest.mark.gpu

CASES = [  # (format, M, N, K, tile_n, stages): ragged M and N, every tile width the path takes
    (qg.QG_FP8_DYNAMIC, 200, 328, 512, 64, 3),
    (qg.QG_FP8_DYNAMIC, 300, 520, 1024, 256, 3),
    (qg.QG_W8A8_INT8, 129, 392, 512, 128, 4),
    (qg.QG_W8A8_INT8, 256, 1024, 2048, 256, 4),
    (qg.QG_BLOCK_FP8, 136, 384, 1024, 128, 3),
    (qg.QG_BLOCK_FP8, 260, 640, 512, 256, 3),
    (qg.QG_NVFP4, 144, 328, 1024, 128, 4),
    (qg.QG_NVFP4, 384, 1280, 2048, 64, 4),
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    qg.qgemm_set_tma_store(True)
    assert qg.qgemm_device_error() == qg.QG_OK


def _id(c):
    return f"{FMT_NAMES[c[0]]}-M{c[1]}-N{c[2]}-K{c[3]}-t{c[4]}"


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_tma_store_matches_thread_stores_and_oracle(case):
    fmt, M, N, K, tn, st = case
    a, w = inputs(M, N, K)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    cfg = qg.make_config(split_k=1, swap_ab=0, tile_n=tn, stages=st, reduce_mode=0)
    ldy = N + 24                               # a wider row: columns N .. ldy keep their sentinel
    outs = []
    for tma in (True, False):
        qg.qgemm_set_tma_store(tma)
        buf = torch.full((M, ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
        y = buf[:, :N]
        qg.run(fmt, A, W, cfg, out=y)
        torch.cuda.synchronize()
        assert torch.isnan(buf[:, N:]).all(), "a store crossed the row's last channel"
        outs.append(y.clone())
    qg.qgemm_set_tma_store(True)
    assert torch.equal(outs[0], outs[1])
    ref = oracle_y(fmt, oracle_quant(fmt, a, False), oracle_quant(fmt, w, True))
    assert_within_tolerance(bf16_to_np(outs[0]), ref, _id(case))


def test_tma_store_covers_a_multi_wave_grid():
    # more tiles than SMs: every CTA's boxes land where the thread stores put them
    fmt, M, N, K = qg.QG_W8A8_INT8, 2048, 5120, 512
    a, w = inputs(M, N, K)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    cfg = qg.make_config(split_k=1, swap_ab=0, tile_n=128, stages=4, reduce_mode=0)
    ys = []
    for tma in (True, False):
        qg.qgemm_set_tma_store(tma)
        ys.append(qg.run(fmt, A, W, cfg))
    qg.qgemm_set_tma_store(True)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1])
    rows = np.random.default_rng(3).choice(M, 16, replace=False)
    qa, qw = oracle_quant(fmt, a[rows], False), oracle_quant(fmt, w, True)
    assert_within_tolerance(bf16_to_np(ys[0][torch.from_numpy(rows).cuda()]), oracle_y(fmt, qa, qw), "multi-wave")
