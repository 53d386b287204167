"""GPU test of the ahead-of-time tuner ("Helion in the vLLM backend", third
paragraph: an autotuner picks the configuration per shape; HeliosTune's
protocol: select on one timing pass, record the time of an independent
second pass).

qgemm_tune_ranked times the scorer's top 4 configurations of two small
shapes into a fresh table.  Every tuned entry must dispatch as an exact hit,
its configuration must compute the oracle's result within the tolerance,
and the time it records must be the second pass's (not the selection pass's
time of the same candidate, which the tuner's candidate log holds)."""
import os

import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16

pytestmark = pytest.mark.gpu

SHAPES = [(qg.QG_FP8_DYNAMIC, [4, 32], (2048, 2048)), (qg.QG_W8A8_INT8, [8], (1024, 4096))]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


FIELDS = ("split_k", "swap_ab", "tile_n", "stages", "reduce_mode", "variant", "rows")


def _log_rows(path):
    """Candidate log lines: fmt M N K, the configuration fields, the time."""
    rows = []
    for line in open(path):
        f = line.split()
        rows.append((tuple(int(x) for x in f[:-1]), float(f[-1])))
    return rows


def _table_rows(path):
    out = {}
    for line in open(path).read().splitlines()[2:]:
        f = line.split()
        out[tuple(int(x) for x in f[:4])] = (tuple(int(x) for x in f[4:-1]), float(f[-1]))
    return out


def test_tune_ranked_writes_validated_entries_timed_on_a_second_pass(tmp_path):
    log = str(tmp_path / "cands.txt")
    saved = str(tmp_path / "tuned.qgt")
    t = qg.Table()
    qg.qgemm_set_tune_log(log)
    try:
        for fmt, Ms, NK in SHAPES:
            t.tune(fmt, Ms, [NK], budget_s_per_shape=20.0, verbose=False, top_n=4)
    finally:
        qg.qgemm_set_tune_log(None)
    t.save(saved)
    entries = _table_rows(saved)
    cands = _log_rows(log)
    assert len(entries) == sum(len(Ms) for _, Ms, _ in SHAPES)
    for fmt, Ms, (N, K) in SHAPES:
        for M in Ms:
            cfg, hit = t.dispatch(fmt, M, N, K)
            assert hit == 1
            key = (fmt, M, N, K)
            fields, us = entries[key]
            assert cfg.as_dict() == dict(zip(FIELDS, fields))
            # the winner was timed in the selection pass (the log) ...
            timed = [t1 for (k, t1) in cands if k[:4] == key and k[4:] == fields]
            assert len(timed) == 1
            # the scorer's top 4, plus up to four of the other kernel variant
            assert 1 <= len([1 for (k, _) in cands if k[:4] == key]) <= 8
            # ... and the table holds an independent second measurement of it
            assert us > 0 and us != timed[0]
            assert 0.5 < us / timed[0] < 2.0
            # the tuned configuration computes the oracle's result
            a, w = inputs(M, N, K, edge_rows=True)
            A = qg.quantize_act(fmt, to_dev_bf16(a))
            W = qg.quantize_weight(fmt, to_dev_bf16(w))
            y = qg.run(fmt, A, W, cfg)
            ref = oracle_y(fmt, oracle_quant(fmt, a, False), oracle_quant(fmt, w, True))
            assert_within_tolerance(bf16_to_np(y), ref, f"tuned fmt {fmt} M {M} {cfg.as_dict()}")
    # the saved table loads back with the same entries
    t2 = qg.Table(saved)
    assert len(t2) == len(entries)
