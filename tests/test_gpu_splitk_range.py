"""Split-K over its whole range ("Helion in the vLLM backend", third
paragraph: split_k is a power of two up to 256) against the oracle.

K is long enough that every one of 32 ... 256 splits keeps a whole 128-byte
K tile (K = 32768 for the 8-bit formats, 65536 for NVFP4), and the partials
meet in the workspace (reduce_mode 1: second pass, 2: last-arriving CTA;
clusters stop at 8).  INT8 accumulators are bit-exact against the oracle's
int64 sums, bf16 outputs are within the target tolerance, and both modes give
the same bits (partials summed in split order)."""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16
from oracle import gemm as OG

pytestmark = pytest.mark.gpu

SPLITS = [32, 64, 128, 256]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


def _setup(fmt, M, N, K):
    a, w = inputs(M, N, K, edge_rows=True)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    return A, W, oracle_quant(fmt, a, False), oracle_quant(fmt, w, True)


CASES = []
for fmt, K in ((qg.QG_W8A8_INT8, 32768), (qg.QG_FP8_DYNAMIC, 32768), (qg.QG_BLOCK_FP8, 32768), (qg.QG_NVFP4, 65536)):
    for sk in SPLITS:
        CASES.append((fmt, 4, 256, K, sk, 1, 16))          # Swap-AB decode tile
CASES += [(qg.QG_FP8_DYNAMIC, 136, 256, 32768, 32, 0, 128),  # standard orientation, two token tiles
          (qg.QG_W8A8_INT8, 130, 384, 32768, 256, 0, 64)]


def _id(c):
    fmt, M, N, K, sk, swap, tn = c
    return f"f{fmt}-M{M}-N{N}-K{K}-s{sk}-sw{swap}-t{tn}"


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_large_split_matches_the_oracle_in_both_workspace_modes(case):
    fmt, M, N, K, sk, swap, tn = case
    A, W, qa, qw = _setup(fmt, M, N, K)
    ref = oracle_y(fmt, qa, qw)
    ys = []
    for mode in (1, 2):
        # two stages hold a Swap-AB slice; the standard orientation's output
        # tile (128 x (tile_n + 4) words, staged in the idle ring) needs three
        cfg = qg.make_config(split_k=sk, swap_ab=swap, tile_n=tn, stages=2 if swap else 3, reduce_mode=mode)
        y = qg.run(fmt, A, W, cfg)
        assert_within_tolerance(bf16_to_np(y), ref, f"{_id(case)} mode {mode}")
        ys.append(y)
        if fmt == qg.QG_W8A8_INT8:
            acc = qg.run(fmt, A, W, cfg, out_kind=qg.QG_OUT_ACC)
            np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), OG.acc_int8(qa[0], qw[0]))
    assert torch.equal(ys[0], ys[1])
    assert qg.qgemm_device_error() == qg.QG_OK


def test_split_beyond_the_k_tiles_is_refused():
    # K = 4096 has 32 tiles of 128 bytes: split 64 would leave empty slices
    fmt, M, N, K = qg.QG_FP8_DYNAMIC, 4, 256, 4096
    A, W, _, _ = _setup(fmt, M, N, K)
    cfg = qg.make_config(split_k=64, swap_ab=1, tile_n=16, stages=2, reduce_mode=1)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = qg.qgemm_run(fmt, A.c, W.c, M, N, K, cfg, None, 0, y.data_ptr(), N, qg.QG_OUT_BF16, qg._stream(None))
    assert st == qg.QG_ERR_UNSUPPORTED
