"""GPU tests of the table policy (TensorRT-LLM issue 16363's shape-gated
selection, as configuration fallbacks inside one library):

* the validation gate keeps every entry of the shipped table, and removes an
  entry the kernels refuse on this device, after which dispatch answers that
  shape with the scored default;
* the identity gate ignores a table recorded on another device;
* a shape dispatched from a medium-M bucket computes within tolerance of the
  oracle.
"""
import os

import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16

pytestmark = pytest.mark.gpu
SHIPPED = os.path.join(os.path.dirname(qg.__file__), "tables", "b200.qgt")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


def test_validation_gate_keeps_the_shipped_table():
    t = qg.Table(SHIPPED)
    n = len(t)
    checked, rejected = t.validate()
    assert checked == n and rejected == 0 and len(t) == n


def test_validation_gate_rejects_a_refused_entry(tmp_path):
    t = qg.Table()
    good = qg.make_config(split_k=4, swap_ab=1, tile_n=16, stages=4, reduce_mode=0)
    # syntactically valid, but its 8-stage ring of 256-wide tiles exceeds the
    # shared memory of one CTA: qgemm_run refuses it on this device
    refused = qg.make_config(split_k=1, swap_ab=0, tile_n=256, stages=8, reduce_mode=0)
    t.put(qg.QG_FP8_DYNAMIC, 8, 1024, 2048, good, 1.0)
    t.put(qg.QG_FP8_DYNAMIC, 256, 1024, 2048, refused, 1.0)
    checked, rejected = t.validate()
    assert (checked, rejected) == (2, 1) and len(t) == 1
    c, hit = t.dispatch(qg.QG_FP8_DYNAMIC, 256, 1024, 2048)
    assert hit == 0 and c.as_dict() == qg.qgemm_default_config(qg.QG_FP8_DYNAMIC, 256, 1024, 2048).as_dict()
    c, hit = t.dispatch(qg.QG_FP8_DYNAMIC, 8, 1024, 2048)
    assert hit == 1 and c.as_dict() == good.as_dict()


def test_identity_gate_ignores_a_table_from_another_device(tmp_path):
    p = tmp_path / "other.qgt"
    p.write_text("qgemm-table 1\ndevice Some_Other_GPU sms 132\n1 8 4096 4096 2 1 32 3 0 9.0\n")
    c, hit = qg.Table(str(p)).dispatch(qg.QG_W8A8_INT8, 8, 4096, 4096)
    assert hit == -1
    assert c.as_dict() == qg.qgemm_default_config(qg.QG_W8A8_INT8, 8, 4096, 4096).as_dict()
    name = torch.cuda.get_device_name().replace(" ", "_")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    p.write_text(f"qgemm-table 1\ndevice {name} sms {sms}\n1 8 4096 4096 2 1 32 3 0 9.0\n")
    c, hit = qg.Table(str(p)).dispatch(qg.QG_W8A8_INT8, 8, 4096, 4096)
    assert hit == 1 and c.as_dict() == qg.make_config(2, 1, 32, 3, 0).as_dict()


@pytest.mark.parametrize("fmt", [qg.QG_FP8_DYNAMIC, qg.QG_BLOCK_FP8], ids=["fp8", "block"])
def test_medium_m_bucket_dispatch_parity(fmt):
    t = qg.Table(SHIPPED)
    M, N, K = 200, 1792, 5120            # between the tuned 128 and 256 buckets
    cfg, hit = t.dispatch(fmt, M, N, K)
    assert hit in (0, 2)
    a, w = inputs(M, N, K, edge_rows=True)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    y = qg.run(fmt, A, W, cfg)
    assert_within_tolerance(bf16_to_np(y), oracle_y(fmt, oracle_quant(fmt, a, False), oracle_quant(fmt, w, True)),
                            f"fmt {fmt} M {M} via {cfg.as_dict()}")
