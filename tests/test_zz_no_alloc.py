"""qgemm_run_noalloc: the split-K GEMM for callers that cannot allocate.

Some callers of this library cannot allocate device memory on the GEMM path
(an engine whose memory planner reserved all device memory up front, a plugin
host that passes only input and output buffers).  qgemm_run_noalloc runs the
same kernel as qgemm_run but takes the split-K scratch from a fixed array
inside the library.  These tests call it through the C ABI and check, on two
calls in a row, that its output matches qgemm_run given a caller-owned
workspace, within the tolerance of the parity tests; they also check that a
configuration needing more scratch than the array holds is refused.
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import bf16_to_np, inputs, to_dev_bf16, tolerance_violations

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield


def _operands(fmt, M, N, K):
    a, w = inputs(M, N, K, edge_rows=True)
    return qg.quantize_act(fmt, to_dev_bf16(a)), qg.quantize_weight(fmt, to_dev_bf16(w))


@pytest.mark.parametrize("fmt,M,N,K,split,mode", [
    (qg.QG_W8A8_INT8, 8, 4096, 4096, 8, 2),     # last-arriving CTA: partials + tile counters
    (qg.QG_FP8_DYNAMIC, 32, 2048, 2048, 4, 1),  # second pass: partials only
    (qg.QG_BLOCK_FP8, 4, 512, 7168, 8, 2),
])
def test_noalloc_matches_run_with_workspace(fmt, M, N, K, split, mode):
    A, W = _operands(fmt, M, N, K)
    cfg = qg.make_config(split_k=split, swap_ab=1, tile_n=16 if M <= 16 else 32, stages=4,
                         reduce_mode=mode)
    ref = qg.run(fmt, A, W, cfg)                                     # caller-owned workspace
    ref_np = bf16_to_np(ref)
    stream = qg._stream(None)
    for call in range(2):                                            # two calls in a row
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = qg.qgemm_run_noalloc(fmt, A.c, W.c, M, N, K, cfg, y.data_ptr(), N, qg.QG_OUT_BF16, stream)
        assert st == qg.QG_OK, qg.status_string(st)
        torch.cuda.synchronize()
        bad = tolerance_violations(bf16_to_np(y), ref_np)
        assert not bad.any(), f"call {call}: {int(bad.sum())} elements differ from qgemm_run"
        # the same kernel sums the same partials in the same split order
        assert torch.equal(y, ref), f"call {call}: not bitwise equal to qgemm_run"
    assert qg.qgemm_device_error() == qg.QG_OK


def test_noalloc_int8_accumulators_bit_exact_twice():
    fmt, M, N, K = qg.QG_W8A8_INT8, 5, 1024, 2048
    A, W = _operands(fmt, M, N, K)
    cfg = qg.make_config(split_k=4, swap_ab=1, tile_n=16, stages=4, reduce_mode=2)
    ref = qg.run(fmt, A, W, cfg, out_kind=qg.QG_OUT_ACC)
    for _ in range(2):
        acc = torch.zeros(M, N, dtype=torch.int32, device="cuda")
        assert qg.qgemm_run_noalloc(fmt, A.c, W.c, M, N, K, cfg, acc.data_ptr(), N, qg.QG_OUT_ACC,
                                    qg._stream(None)) == qg.QG_OK
        torch.cuda.synchronize()
        assert torch.equal(acc, ref)


def test_noalloc_refuses_scratch_beyond_its_maximum():
    fmt, M, N, K = qg.QG_FP8_DYNAMIC, 32, 16384, 4096
    A = qg.Operand(fmt, False, M, K)                 # contents unused: refused before any launch
    W = qg.Operand(fmt, True, N, K)
    cfg = qg.make_config(split_k=8, swap_ab=1, tile_n=32, stages=4, reduce_mode=1)
    assert qg.qgemm_workspace_size(fmt, M, N, K, cfg) > (8 << 20)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    assert qg.qgemm_run_noalloc(fmt, A.c, W.c, M, N, K, cfg, y.data_ptr(), N, qg.QG_OUT_BF16,
                                qg._stream(None)) == qg.QG_ERR_WORKSPACE
