"""GPU parity of the GEMM with fused activation quantisation
(qgemm_run_fused_act), through the C ABI.

* y (bf16) is bitwise equal to qgemm_quantize_act followed by qgemm_run with
  the same configuration: the kernel must produce the same codes and scales
  and accumulate in the same order.  Covered for FP8_Dynamic, W8A8_INT8 and
  Block_FP8 over unsplit launches, cluster split-K (2, 4 and 8 CTAs swapping
  partial amaxes through distributed shared memory), workspace split-K
  (Block_FP8), rings that wrap, several token tiles, ragged N, ragged K and a
  padded activation row stride;
* the activation scales the kernel reports are bitwise those of the oracle;
* y is within |y - y_ref| <= 0.01 |y_ref| + 0.01 rms(y_ref row) of the
  oracle, and INT8 int32 accumulators are bit-exact;
* a captured one-launch decode step replays to the two-launch step's bits.
"""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, inputs, oracle_quant, oracle_y, to_dev_bf16
from oracle import gemm as OG

pytestmark = pytest.mark.gpu

FMTS = [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8]
IDS = {qg.QG_FP8_DYNAMIC: "fp8", qg.QG_W8A8_INT8: "int8", qg.QG_BLOCK_FP8: "block"}

# (M, N, K, split_k, tile_n, reduce_mode, stages, row padding of A in elements)
CASES = [
    (1, 256, 512, 1, 16, 0, 4, 0),
    (5, 384, 1024, 2, 16, 0, 4, 0),
    (16, 300, 1024, 4, 16, 0, 6, 0),      # ragged N
    (32, 640, 2048, 8, 32, 0, 8, 0),      # 8-CTA cluster
    (33, 130, 512, 1, 16, 0, 4, 0),       # three token tiles, the last with one token
    (8, 512, 2048, 4, 16, 0, 2, 0),       # two-stage ring, wrapping twice per CTA
    (1, 384, 4096, 2, 16, 0, 3, 0),       # 16 K tiles per CTA: units past the register cache
    (48, 256, 1024, 2, 64, 0, 4, 0),      # 64-token tile
    (100, 256, 1024, 1, 128, 0, 3, 0),    # 128-token tile (Block_FP8: 8 epilogue warps)
    (4, 256, 4096, 1, 16, 0, 4, 0),       # 32 K tiles over 4 stages
    (12, 256, 1024, 2, 16, 0, 4, 24),     # padded row stride
    (20, 512, 2048, 4, 32, 1, 8, 0),      # workspace split-K, second pass
    (16, 300, 1024, 4, 16, 2, 6, 0),      # workspace split-K, last CTA
]
RAGGED_K = [                              # K % 128 != 0 (FP8_Dynamic, W8A8_INT8)
    (3, 256, 1040, 2, 16, 0, 4, 0),
    (7, 200, 400, 1, 16, 0, 4, 0),
]


def _all_cases():
    out = []
    for f in FMTS:
        for c in CASES + (RAGGED_K if f != qg.QG_BLOCK_FP8 else []):
            out.append((f,) + c)
    return out


ALL = _all_cases()


def _id(c):
    f, M, N, K, sk, tn, rm, st, pad = c
    return f"{IDS[f]}-M{M}-N{N}-K{K}-s{sk}-t{tn}-r{rm}-st{st}-pad{pad}"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability() == (10, 0), "GPU tests need an sm_100 device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


def _activations(a_bits, pad):
    """bf16 [M, K] on the device, optionally inside a wider row stride."""
    a = to_dev_bf16(a_bits)
    if pad == 0:
        return a
    M, K = a.shape
    wide = torch.zeros(M, K + pad, dtype=torch.bfloat16, device=a.device)
    wide[:, :K] = a
    return wide[:, :K]


def _scale_buffer(fmt, M, K):
    n = M * (K // 128) if fmt == qg.QG_BLOCK_FP8 else M
    return torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")


def _supported(fmt, sk, rm):
    return fmt == qg.QG_BLOCK_FP8 or sk == 1 or rm == 0


@pytest.mark.parametrize("case", ALL, ids=[_id(c) for c in ALL])
def test_fused_equals_quantize_then_run(case):
    fmt, M, N, K, sk, tn, rm, st, pad = case
    cfg = qg.make_config(split_k=sk, swap_ab=1, tile_n=tn, stages=st, reduce_mode=rm)
    a, w = inputs(M, N, K, edge_rows=M >= 3)
    A = _activations(a, pad)
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    if not _supported(fmt, sk, rm):
        with pytest.raises(qg.QGemmError) as e:
            qg.run_fused(fmt, A, W, cfg)
        assert e.value.status == qg.QG_ERR_UNSUPPORTED
        return
    Aq = qg.quantize_act(fmt, A)
    y_two = qg.run(fmt, Aq, W, cfg)
    sc = _scale_buffer(fmt, M, K)
    y = qg.run_fused(fmt, A, W, cfg, act_scale_out=sc)
    y_again = qg.run_fused(fmt, A, W, cfg)
    torch.cuda.synchronize()
    assert torch.equal(y, y_two), _id(case)
    assert torch.equal(y, y_again), _id(case)
    qa = oracle_quant(fmt, a, False)
    qw = oracle_quant(fmt, w, True)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32),
                                  np.ascontiguousarray(qa[1], dtype=np.float32).reshape(-1).view(np.uint32))
    assert_within_tolerance(bf16_to_np(y), oracle_y(fmt, qa, qw), _id(case))


INT8 = [c for c in ALL if c[0] == qg.QG_W8A8_INT8 and _supported(c[0], c[4], c[6])]


@pytest.mark.parametrize("case", INT8, ids=[_id(c) for c in INT8])
def test_fused_int8_accumulators_bit_exact(case):
    fmt, M, N, K, sk, tn, rm, st, pad = case
    cfg = qg.make_config(split_k=sk, swap_ab=1, tile_n=tn, stages=st, reduce_mode=rm)
    a, w = inputs(M, N, K, edge_rows=M >= 3)
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    acc = qg.run_fused(fmt, _activations(a, pad), W, cfg, out_kind=qg.QG_OUT_ACC)
    qa = oracle_quant(fmt, a, False)
    qw = oracle_quant(fmt, w, True)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), OG.acc_int8(qa[0], qw[0]))


@pytest.mark.parametrize("fmt", FMTS, ids=[IDS[f] for f in FMTS])
def test_fused_graph_step_matches_two_launch_step(fmt):
    M, N, K = 8, 1024, 2048
    a, w = inputs(M, N, K, edge_rows=True)
    layer = qg.Linear(fmt, to_dev_bf16(w))
    cfg = qg.make_config(split_k=4, swap_ab=1, tile_n=16, stages=4, reduce_mode=0)
    two = layer.capture(M, cfg=cfg)
    one = qg.GraphStep(layer, M, cfg=cfg, fused=True)
    for g in (two, one):
        g.A.copy_(to_dev_bf16(a))
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(one.Y, two.Y)


@pytest.mark.parametrize("fmt", FMTS, ids=[IDS[f] for f in FMTS])
def test_graph_step_host_io_and_captured_sequence(fmt):
    """A step with host I/O in its graph returns, in pinned host memory, the
    bits of the device-only step; steps captured back to back in one graph
    (capture_steps) give each step's own result."""
    N, K = 1024, 2048
    a1, w = inputs(1, N, K)
    a8, _ = inputs(8, N, K, edge_rows=True)
    layer = qg.Linear(fmt, to_dev_bf16(w))
    dev_only = {m: layer.capture(m) for m in (1, 8)}
    host = {m: qg.GraphStep(layer, m, host_io=True) for m in (1, 8)}
    for m, a in ((1, a1), (8, a8)):
        dev_only[m].A.copy_(to_dev_bf16(a))
        dev_only[m].replay()
        host[m].A_host.copy_(to_dev_bf16(a).cpu())
    torch.cuda.synchronize()
    seq = qg.capture_steps([host[1], host[8]])
    seq.replay()
    torch.cuda.synchronize()
    for m in (1, 8):
        assert torch.equal(host[m].Y_host, dev_only[m].Y.cpu())
    # a single step's own graph with host I/O agrees as well
    for m in (1, 8):
        host[m].Y_host.zero_()
        out = host[m].replay()
        torch.cuda.synchronize()
        assert torch.equal(out, dev_only[m].Y.cpu())
