"""GPU parity of the grouped (mixture-of-experts) GEMM, qgemm_run_grouped,
through the C ABI: every expert's rows of y are bitwise those of qgemm_run on
that expert's slice of A and W with the same configuration (same K split,
same accumulation order), and within the target tolerance of the oracle;
INT8 accumulators are bit-exact.  Routings cover experts without tokens,
experts with several token tiles, one expert holding every token, and split-K
through a cluster and through a second pass."""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import assert_within_tolerance, bf16_to_np, oracle_quant, to_dev_bf16
import qg_synth
from oracle import gemm as OG
from oracle import quant as OQ

pytestmark = pytest.mark.gpu

FMTS = [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8]
# the oracle's plain GEMM per format and its weight rows per scale
ORACLE_GEMM = {qg.QG_FP8_DYNAMIC: (OG.fp8_dynamic, 1), qg.QG_W8A8_INT8: (OG.w8a8_int8, 1),
               qg.QG_BLOCK_FP8: (OG.block_fp8, 128)}
IDS = {qg.QG_FP8_DYNAMIC: "fp8", qg.QG_W8A8_INT8: "int8", qg.QG_BLOCK_FP8: "block"}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


ROUTINGS = {  # tokens per expert
    "sparse": [3, 0, 1, 0, 0, 5, 2, 0],
    "one-expert": [0, 0, 37, 0],
    "multi-tile": [17, 40, 0, 16, 1, 33],
    "uniform": [2] * 16,
    # every expert's count is 1 mod 16: the routing needs exactly the grid's
    # floor((T - a) / tile_n) + a token tiles at tile_n = 16
    "tight": [17, 17, 1, 1],
    # the most experts a launch takes: every 32-expert chunk of the scan
    "e256": np.random.default_rng(5).multinomial(200, [1 / 256] * 256).tolist(),
}
CASES = [  # (routing, N, K, split_k, tile_n, reduce_mode, stages)
    ("sparse", 256, 1024, 1, 16, 0, 4),
    ("one-expert", 384, 512, 1, 16, 0, 4),
    ("multi-tile", 256, 2048, 4, 16, 0, 4),
    ("multi-tile", 128, 1024, 2, 32, 1, 4),
    ("uniform", 256, 1024, 2, 16, 0, 3),
    ("tight", 256, 512, 1, 16, 0, 4),
    ("tight", 128, 1024, 2, 16, 1, 4),
    ("e256", 128, 512, 1, 16, 0, 4),
]
ALL = [(f,) + c for f in FMTS for c in CASES]


def _id(c):
    return f"{IDS[c[0]]}-{c[1]}-N{c[2]}-K{c[3]}-s{c[4]}-t{c[5]}-r{c[6]}"


def _view(op: qg.Operand, fmt, row0, rows, K, is_weight):
    """An operand of rows [row0, row0 + rows) of `op` (pointer offsets only)."""
    q = op.q.data_ptr() + row0 * K
    if fmt == qg.QG_BLOCK_FP8:
        per_row = K // 128 * 4
        s = op.scale.data_ptr() + (row0 // 128 if is_weight else row0) * per_row
    else:
        s = op.scale.data_ptr() + row0 * 4
    return qg.qg_operand(q, s, op.global_scale.data_ptr(), rows, K)


@pytest.mark.parametrize("case", ALL, ids=[_id(c) for c in ALL])
def test_grouped_matches_per_expert_runs_and_oracle(case):
    fmt, routing, N, K, sk, tn, rm, st = case
    counts = ROUTINGS[routing]
    E, T = len(counts), sum(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    a = qg_synth.activations(T, K)
    w = qg_synth.weights(E * N, K)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    offsets = torch.from_numpy(offs).cuda()
    cfg = qg.make_config(split_k=sk, swap_ab=1, tile_n=tn, stages=st, reduce_mode=rm)
    y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    qg.run_grouped(fmt, A, W, offsets, N, cfg, out=y)
    y_again = qg.run_grouped(fmt, A, W, offsets, N, cfg)
    torch.cuda.synchronize()
    assert torch.equal(y, y_again)
    qa = oracle_quant(fmt, a, False)
    qw = oracle_quant(fmt, w, True)
    gemm_fn, w_rows_per_scale = ORACLE_GEMM[fmt]
    ref = OG.grouped(gemm_fn, qa[0], qa[1], qw[0], qw[1], offs, N, w_rows_per_scale)
    ws = qg.Workspace()
    for e in range(E):
        m0, m = int(offs[e]), counts[e]
        if m == 0:
            continue
        ye = torch.empty(m, N, dtype=torch.bfloat16, device="cuda")
        Ae, We = _view(A, fmt, m0, m, K, False), _view(W, fmt, e * N, N, K, True)
        wsp, wsb = ws.get(qg.qgemm_workspace_size(fmt, m, N, K, cfg))
        qg.check(qg.qgemm_run(fmt, Ae, We, m, N, K, cfg, wsp, wsb, ye.data_ptr(), N, 0, qg._stream(None)))
        torch.cuda.synchronize()
        assert torch.equal(y[m0:m0 + m], ye), f"expert {e}"
        assert_within_tolerance(bf16_to_np(y[m0:m0 + m]), ref[m0:m0 + m], f"{_id(case)} expert {e}")


def test_grouped_int8_accumulators_bit_exact():
    fmt, counts, N, K = qg.QG_W8A8_INT8, ROUTINGS["multi-tile"], 256, 2048
    E, T = len(counts), sum(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    a, w = qg_synth.activations(T, K), qg_synth.weights(E * N, K)
    A, W = qg.quantize_act(fmt, to_dev_bf16(a)), qg.quantize_weight(fmt, to_dev_bf16(w))
    cfg = qg.make_config(split_k=4, swap_ab=1, tile_n=16, stages=4, reduce_mode=0)
    acc = qg.run_grouped(fmt, A, W, torch.from_numpy(offs).cuda(), N, cfg, out_kind=qg.QG_OUT_ACC).cpu().numpy()
    qa, qw = oracle_quant(fmt, a, False), oracle_quant(fmt, w, True)
    for e in range(E):
        m0, m1 = int(offs[e]), int(offs[e + 1])
        if m1 > m0:
            np.testing.assert_array_equal(acc[m0:m1].astype(np.int64),
                                          OG.acc_int8(qa[0][m0:m1], qw[0][e * N:(e + 1) * N]))


# ------------------------------------------------------------------- NVFP4 --
# NVFP4 grouped launches: activations quantised with the per-expert scale
# layout (each expert's block scales start on a 128-row atom), weights one
# tensor per expert (a tensor scale each).
NVF4_ROUTINGS = dict(ROUTINGS, big=[300, 0, 129, 5, 200])
NVF4_CASES = [  # (routing, N, K, split_k, tile_n, reduce_mode, stages)
    ("sparse", 256, 1024, 1, 16, 0, 4),        # T = 11 <= 16: one tile per expert
    ("multi-tile", 256, 2048, 1, 64, 0, 4),
    ("multi-tile", 128, 1024, 2, 64, 1, 4),    # second-pass reduction
    ("big", 256, 1024, 2, 128, 0, 4),          # experts over 128 tokens: several atoms
    ("big", 128, 512, 1, 256, 0, 3),           # 256-token tiles: two atoms
    ("e256", 128, 512, 1, 64, 0, 4),
]


def _nvf4_id(c):
    return f"nvfp4-{c[0]}-N{c[1]}-K{c[2]}-s{c[3]}-t{c[4]}-r{c[5]}"


def _expert_rows(counts):
    """First scale row of every expert in the per-expert layout."""
    rows, r = [], 0
    for c in counts:
        rows.append(r)
        r += (c + 127) // 128 * 128
    return rows, r


@pytest.mark.parametrize("case", NVF4_CASES, ids=[_nvf4_id(c) for c in NVF4_CASES])
def test_grouped_nvfp4_matches_per_expert_runs_and_oracle(case):
    routing, N, K, sk, tn, rm, st = case
    fmt = qg.QG_NVFP4
    counts = NVF4_ROUTINGS[routing]
    E, T = len(counts), sum(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    a = qg_synth.activations(T, K)
    w = qg_synth.weights(E * N, K)
    offsets = torch.from_numpy(offs).cuda()
    A = qg.quantize_act_grouped(fmt, to_dev_bf16(a), offsets)
    W = qg.quantize_weight_grouped(fmt, to_dev_bf16(w), E)
    cfg = qg.make_config(split_k=sk, swap_ab=1, tile_n=tn, stages=st, reduce_mode=rm)
    y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    qg.run_grouped(fmt, A, W, offsets, N, cfg, out=y)
    y_again = qg.run_grouped(fmt, A, W, offsets, N, cfg)
    torch.cuda.synchronize()
    assert torch.equal(y, y_again)
    qa = OQ.nvfp4(a)
    qw = OQ.nvfp4_experts(w, E)
    # the tensor scales are the oracle's fp32 quotients
    assert float(A.global_scale[0]) == float(qa[2])
    assert np.array_equal(W.global_scale[:E].cpu().numpy(), qw[2])
    ref = OG.grouped_nvfp4(qa[0], qa[1], qa[2], qw[0], qw[1], qw[2], offs, N)
    C = (K + 255) // 256 * 16
    rows, _ = _expert_rows(counts)
    qbw, sbw = qg.qgemm_operand_bytes(fmt, 1, N, K)
    ws = qg.Workspace()
    for e in range(E):
        m0, m = int(offs[e]), counts[e]
        if m == 0:
            continue
        Ae = qg.qg_operand(A.q.data_ptr() + m0 * K // 2, A.scale.data_ptr() + rows[e] * C,
                           A.global_scale.data_ptr(), m, K)
        We = qg.qg_operand(W.q.data_ptr() + e * qbw, W.scale.data_ptr() + e * sbw,
                           W.global_scale.data_ptr() + 4 * e, N, K)
        ye = torch.empty(m, N, dtype=torch.bfloat16, device="cuda")
        wsp, wsb = ws.get(qg.qgemm_workspace_size(fmt, m, N, K, cfg))
        qg.check(qg.qgemm_run(fmt, Ae, We, m, N, K, cfg, wsp, wsb, ye.data_ptr(), N, 0, qg._stream(None)))
        torch.cuda.synchronize()
        assert torch.equal(y[m0:m0 + m], ye), f"expert {e}"
        assert_within_tolerance(bf16_to_np(y[m0:m0 + m]), ref[m0:m0 + m], f"{_nvf4_id(case)} expert {e}")


@pytest.mark.parametrize("routing", ["sparse", "big", "e256"])
def test_grouped_nvfp4_activation_layout_is_each_experts_plain_layout(routing):
    # with one static amax, expert e's codes and block scales are bitwise those
    # of the plain quantiser on its own tokens, placed at its first atom; the
    # scale rows past the last expert's atoms are zero
    fmt, K = qg.QG_NVFP4, 512
    counts = NVF4_ROUTINGS[routing]
    E, T = len(counts), sum(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    a = to_dev_bf16(qg_synth.activations(T, K))
    amax = torch.tensor([3.0], dtype=torch.float32, device="cuda")
    G = qg.quantize_act_grouped(fmt, a, torch.from_numpy(offs).cuda(), static_amax=amax)
    torch.cuda.synchronize()
    C = (K + 255) // 256 * 16
    rows, used = _expert_rows(counts)
    for e in range(E):
        m0, m = int(offs[e]), counts[e]
        if m == 0:
            continue
        P = qg.quantize_act(fmt, a[m0:m0 + m], static_amax=amax)
        torch.cuda.synchronize()
        assert torch.equal(G.q[m0 * K // 2:(m0 + m) * K // 2], P.q), f"expert {e} codes"
        nb = P.scale.numel()
        assert torch.equal(G.scale[rows[e] * C:rows[e] * C + nb], P.scale), f"expert {e} scales"
        assert float(G.global_scale[0]) == float(P.global_scale[0])
    assert int(G.scale[used * C:].count_nonzero()) == 0
