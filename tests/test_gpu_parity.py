"""GPU parity of the CUDA path with the CPU oracle, through the C ABI.

* quantisers: codes and scales bit-exact for all four formats, activations
  and weights, including an all-zero row, a 100x outlier and ragged sizes;
* INT8 int32 accumulators bit-exact for every orientation / split / reduce
  mode;
* bf16 outputs within |y - y_ref| <= 0.01 |y_ref| + 0.01 rms(y_ref row) for
  every format and variant (Standard, Split-K in both reduction modes,
  Swap-AB), at sizes spanning several tiles plus ragged tails.
"""
import numpy as np
import pytest
import torch

import precision_quantized_gemm_b200 as qg
from gpu_util import (assert_within_tolerance, bf16_to_np, gpu_codes, inputs, oracle_quant, oracle_y,
                      sf_padding_is_zero, to_dev_bf16)
from oracle import gemm as OG

pytestmark = pytest.mark.gpu

FMTS = [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8, qg.QG_NVFP4]
IDS = ["fp8", "int8", "block", "nvfp4"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability() == (10, 0), "GPU tests need an sm_100 device"
    qg.lib()
    yield
    assert qg.qgemm_device_error() == qg.QG_OK


def _k_for(fmt, K):
    return K


# ------------------------------------------------------------- quantisers --
@pytest.mark.parametrize("fmt", FMTS, ids=IDS)
@pytest.mark.parametrize("M,K", [(1, 256), (5, 1024), (32, 4096), (3, 8192)])
def test_act_quant_bit_exact(fmt, M, K):
    a, _ = inputs(M, 8, K, edge_rows=True)
    op = qg.quantize_act(fmt, to_dev_bf16(a))
    got = gpu_codes(fmt, op)
    want = oracle_quant(fmt, a, False)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(w))
    if fmt == qg.QG_NVFP4:
        assert sf_padding_is_zero(op.scale.cpu().numpy(), M, K)


@pytest.mark.parametrize("fmt", FMTS, ids=IDS)
@pytest.mark.parametrize("N,K", [(128, 256), (200, 512), (1024, 2048)])
def test_weight_quant_bit_exact(fmt, N, K):
    _, w = inputs(1, N, K)
    op = qg.quantize_weight(fmt, to_dev_bf16(w))
    got = gpu_codes(fmt, op)
    want = oracle_quant(fmt, w, True)
    for g, ww in zip(got, want):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(ww))


def _tie_rows(fmt, rows, K, seed):
    """bf16 rows whose amax fixes the scale to a power of two and whose other
    elements sit exactly on, or one bf16 step beside, a rounding tie of the
    code format (int8: k + 1/2; e4m3: midpoints of normal and subnormal
    codes), times the scale: every unit needs the quantisers' exact path."""
    rng = np.random.default_rng(seed)
    if fmt == qg.QG_W8A8_INT8:
        ties = np.arange(-127, 127) + 0.5
        qmax = 127.0
    else:
        mids = [(1 + (2 * j + 1) / 16) * 2.0 ** e for e in range(-6, 8) for j in range(8)]
        mids += [(2 * j + 1) * 2.0 ** -10 for j in range(7)]
        ties = np.array(mids + [-m for m in mids])
        qmax = 448.0
    out = np.empty((rows, K), np.float32)
    for r in range(rows):
        scale = 2.0 ** int(rng.integers(-3, 3))
        v = rng.choice(ties, size=K) * scale
        nudge = rng.integers(-1, 2, size=K)                 # -1, 0, +1 bf16 steps
        bits = (v.astype(np.float32).view(np.uint32) >> 16).astype(np.int64) + nudge * (v != 0)
        v = (bits.astype(np.uint32) << 16).view(np.float32)
        # the scale is fixed by the format's maximum times the power of two,
        # once per 128-element group (covers per-row and per-group scales)
        v[::128] = qmax * scale
        out[r] = v
    return (out.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("fmt", [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8], ids=["fp8", "int8", "block"])
def test_quant_codes_on_rounding_ties(fmt):
    a = _tie_rows(fmt, 7, 1024, seed=11)
    op = qg.quantize_act(fmt, to_dev_bf16(a))
    for g, w in zip(gpu_codes(fmt, op), oracle_quant(fmt, a, False)):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(w))
    w_bits = _tie_rows(fmt, 256, 512, seed=12)
    if fmt == qg.QG_BLOCK_FP8:                            # one power-of-two scale per 128x128 block
        w_bits = w_bits.copy()
        for nb in range(2):
            w_bits[nb * 128:(nb + 1) * 128] = w_bits[nb * 128]
    wop = qg.quantize_weight(fmt, to_dev_bf16(w_bits))
    for g, w in zip(gpu_codes(fmt, wop), oracle_quant(fmt, w_bits, True)):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(w))


def test_act_quant_with_row_stride():
    a, _ = inputs(4, 8, 512)
    big = np.zeros((4, 640), np.uint16)
    big[:, :512] = a
    t = to_dev_bf16(big)[:, :512]
    op = qg.quantize_act(qg.QG_FP8_DYNAMIC, t)
    got = gpu_codes(qg.QG_FP8_DYNAMIC, op)
    want = oracle_quant(qg.QG_FP8_DYNAMIC, a, False)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])


def test_nvfp4_static_amax():
    a, _ = inputs(4, 8, 512)
    amax = torch.tensor([3.0], dtype=torch.float32, device="cuda")
    op = qg.quantize_act(qg.QG_NVFP4, to_dev_bf16(a), static_amax=amax)
    got = gpu_codes(qg.QG_NVFP4, op)
    from oracle import quant as OQ
    want = OQ.nvfp4(a, global_amax=3.0)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(np.asarray(g), np.asarray(w))


# ------------------------------------------------------------------ GEMMs --
def _setup(fmt, M, N, K, edge_rows=True):
    a, w = inputs(M, N, K, edge_rows=edge_rows)
    A = qg.quantize_act(fmt, to_dev_bf16(a))
    W = qg.quantize_weight(fmt, to_dev_bf16(w))
    qa = oracle_quant(fmt, a, False)
    qw = oracle_quant(fmt, w, True)
    return A, W, qa, qw


SWAP_CASES = [  # (M, N, K, split_k, tile_n, reduce_mode, stages); reduce 0 cluster, 1 second pass, 2 last CTA
    (1, 256, 512, 1, 16, 0, 4),
    (5, 384, 1024, 2, 16, 0, 4),
    (16, 300, 1024, 4, 16, 2, 6),
    (20, 512, 2048, 4, 32, 1, 8),
    (32, 640, 2048, 8, 32, 0, 8),
    (32, 640, 2048, 8, 32, 2, 8),
    (48, 256, 1024, 2, 64, 0, 4),
    (33, 130, 512, 1, 16, 0, 4),      # two token tiles, ragged N
    (3, 260, 4096, 16, 16, 2, 4),     # split beyond the cluster limit
    (8, 512, 2048, 4, 16, 0, 2),      # two-stage ring, wrapping twice per CTA
    (1, 384, 4096, 2, 16, 0, 3),      # three-stage ring, ragged wrap
    (100, 512, 2048, 2, 128, 0, 4),   # wide token tiles: cluster pull reduction
    (130, 384, 1024, 1, 128, 0, 4),   # two wide token tiles, ragged
    (64, 256, 1024, 2, 128, 2, 4),    # wide tile, last-CTA reduction
    (200, 256, 1024, 1, 256, 0, 3),   # widest token tile
]
STD_CASES = [
    (128, 256, 512, 1, 128, 0, 4),
    (200, 384, 1024, 2, 64, 0, 4),
    (256, 512, 1024, 1, 256, 0, 3),
    (130, 300, 2048, 4, 128, 1, 4),
    (150, 256, 2048, 4, 128, 0, 4),
    (150, 256, 2048, 2, 256, 0, 3),
    (140, 200, 1024, 2, 64, 2, 4),
    (260, 520, 2048, 1, 256, 0, 3),   # wide tile: Block_FP8 promotes with 8 epilogue warps
    (200, 300, 1024, 2, 256, 0, 3),
    (140, 300, 1024, 2, 128, 2, 4),   # last-CTA reduction of a 128-wide tile
    (140, 300, 1024, 2, 128, 0, 4),   # cluster pull reduction of a 128-wide tile, ragged M and N
    (260, 384, 2048, 8, 128, 0, 4),   # pull over eight CTAs, 16 rows owned each
    (150, 520, 2048, 2, 256, 0, 4),   # 256-wide pull, four-stage ring
]


def _cases(fmt):
    out = []
    for (M, N, K, sk, tn, rm, st) in SWAP_CASES:
        if fmt == qg.QG_NVFP4 and tn < 64 and M > tn:
            continue
        out.append((M, N, K, qg.make_config(split_k=sk, swap_ab=1, tile_n=tn, stages=st, reduce_mode=rm)))
    for (M, N, K, sk, tn, rm, st) in STD_CASES:
        out.append((M, N, K, qg.make_config(split_k=sk, swap_ab=0, tile_n=tn, stages=st, reduce_mode=rm)))
    return out


ALL_CASES = [(f, *c) for f in FMTS for c in _cases(f)]


def _case_id(c):
    f, M, N, K, cfg = c
    return f"{IDS[f]}-M{M}-N{N}-K{K}-s{cfg.split_k}-sw{cfg.swap_ab}-t{cfg.tile_n}-r{cfg.reduce_mode}"


@pytest.mark.parametrize("case", ALL_CASES, ids=[_case_id(c) for c in ALL_CASES])
def test_gemm_bf16_within_tolerance(case):
    fmt, M, N, K, cfg = case
    if fmt == qg.QG_NVFP4 and K % 32:
        pytest.skip("NVFP4 needs K % 32 == 0")
    A, W, qa, qw = _setup(fmt, M, N, K)
    y = qg.run(fmt, A, W, cfg)
    ref = oracle_y(fmt, qa, qw)
    assert_within_tolerance(bf16_to_np(y), ref, _case_id(case))


INT8_ACC_CASES = [c for c in ALL_CASES if c[0] == qg.QG_W8A8_INT8]


@pytest.mark.parametrize("case", INT8_ACC_CASES, ids=[_case_id(c) for c in INT8_ACC_CASES])
def test_int8_accumulators_bit_exact(case):
    fmt, M, N, K, cfg = case
    A, W, qa, qw = _setup(fmt, M, N, K)
    acc = qg.run(fmt, A, W, cfg, out_kind=qg.QG_OUT_ACC)
    want = OG.acc_int8(qa[0], qw[0])
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), want)


def test_fp8_raw_accumulators_exact_without_split():
    # unsplit fp32 accumulation of e4m3 products: check against exact sums
    # within fp32 accumulation error
    A, W, qa, qw = _setup(qg.QG_FP8_DYNAMIC, 16, 256, 1024)
    acc = qg.run(qg.QG_FP8_DYNAMIC, A, W, qg.make_config(split_k=1, swap_ab=1, tile_n=16, stages=4),
                 out_kind=qg.QG_OUT_ACC).cpu().numpy().astype(np.float64)
    exact = OG.acc_e4m3(qa[0], qw[0])
    scale = np.abs(exact).max()
    assert np.max(np.abs(acc - exact)) <= 1e-5 * scale


@pytest.mark.parametrize("fmt", FMTS, ids=IDS)
def test_default_config_parity(fmt):
    A, W, qa, qw = _setup(fmt, 8, 1024, 2048)
    y = qg.run(fmt, A, W)
    assert_within_tolerance(bf16_to_np(y), oracle_y(fmt, qa, qw), IDS[fmt])


def test_split_k_deterministic_and_modes_agree():
    fmt = qg.QG_FP8_DYNAMIC
    A, W, _, _ = _setup(fmt, 16, 512, 4096)
    ys = [qg.run(fmt, A, W, qg.make_config(split_k=8, swap_ab=1, tile_n=16, stages=6, reduce_mode=r))
          for r in (0, 1, 2, 0, 2)]
    for y in ys[1:]:
        assert torch.equal(ys[0], y)     # fixed split order: every mode, every run, same bits


@pytest.mark.parametrize("fmt", [qg.QG_FP8_DYNAMIC, qg.QG_BLOCK_FP8, qg.QG_NVFP4], ids=["fp8", "block", "nvfp4"])
@pytest.mark.parametrize("sk", [2, 4, 8])
def test_wide_tile_cluster_reduction_agrees_with_workspace_modes(fmt, sk):
    # standard orientation, 128-wide tiles: the cluster's pull reduction sums
    # in the same split order as the two workspace reductions
    A, W, _, _ = _setup(fmt, 200, 384, 4096)
    ys = [qg.run(fmt, A, W, qg.make_config(split_k=sk, swap_ab=0, tile_n=128, stages=4, reduce_mode=r))
          for r in (0, 1, 2)]
    for y in ys[1:]:
        assert torch.equal(ys[0], y)


def test_swap_and_standard_agree_int8_bitwise():
    fmt = qg.QG_W8A8_INT8
    A, W, _, _ = _setup(fmt, 128, 256, 1024)
    ys = qg.run(fmt, A, W, qg.make_config(split_k=1, swap_ab=1, tile_n=128, stages=4), out_kind=qg.QG_OUT_ACC)
    yt = qg.run(fmt, A, W, qg.make_config(split_k=2, swap_ab=0, tile_n=128, stages=4), out_kind=qg.QG_OUT_ACC)
    assert torch.equal(ys, yt)
