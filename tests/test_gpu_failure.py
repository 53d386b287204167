"""Failure detection on the GPU without a fault: every in-kernel wait of the
library is bounded, and an expired wait sets the device error word, which
the host reads (QG_ERR_DEVICE_TIMEOUT) while the context stays usable.

The self-test kernel waits, with the library's own bounded wait and a 1 ms
limit, on an mbarrier that nothing arrives on (no copy or MMA in flight).
After it returns the error is reported once and cleared, and a GEMM runs
correctly on the same context, also with a short wait limit set."""
import time

import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    assert qg.qgemm_device_error() == qg.QG_OK
    yield
    qg.qgemm_set_wait_limit(0)


def test_expired_wait_is_reported_once_and_the_context_stays_usable():
    t0 = time.perf_counter()
    assert qg.qgemm_selftest_wait_expiry(1_000_000) == qg.QG_OK        # 1 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert qg.qgemm_device_error() == qg.QG_ERR_DEVICE_TIMEOUT
    assert qg.qgemm_device_error() == qg.QG_OK                        # read and cleared
    fmt, M, N, K = qg.QG_W8A8_INT8, 8, 1024, 2048
    a, w = inputs(M, N, K, edge_rows=True)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    y = qg.run(fmt, A, W, qg.make_config(split_k=4, swap_ab=1, tile_n=16, stages=4, reduce_mode=0))
    assert_within_tolerance(bf16_to_np(y), oracle_y(fmt, oracle_quant(fmt, a, False), oracle_quant(fmt, w, True)),
                            "GEMM after an expired wait")
    assert qg.qgemm_device_error() == qg.QG_OK


def test_short_wait_limit_does_not_disturb_healthy_launches():
    qg.qgemm_set_wait_limit(20_000_000)                                  # 20 ms
    try:
        fmt, M, N, K = qg.QG_FP8_DYNAMIC, 16, 2048, 2048
        a, w = inputs(M, N, K, edge_rows=True)
        A = qg.quantize_act(fmt, to_dev_bf16(a))
        W = qg.quantize_weight(fmt, to_dev_bf16(w))
        for cfg in (qg.make_config(8, 1, 16, 4, 0), qg.make_config(4, 1, 16, 4, 2), qg.make_config(1, 0, 128, 4, 0)):
            y = qg.run(fmt, A, W, cfg)
            assert_within_tolerance(bf16_to_np(y), oracle_y(fmt, oracle_quant(fmt, a, False),
                                                            oracle_quant(fmt, w, True)), f"{cfg.as_dict()}")
        assert qg.qgemm_device_error() == qg.QG_OK
    finally:
        qg.qgemm_set_wait_limit(0)


def test_selftest_rejects_limits_out_of_range():
    assert qg.qgemm_selftest_wait_expiry(0) == qg.QG_ERR_INVALID_ARG
    assert qg.qgemm_selftest_wait_expiry(10 ** 9) == qg.QG_ERR_INVALID_ARG
