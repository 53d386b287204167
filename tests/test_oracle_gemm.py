"""Pins of the oracle's contraction and epilogues.

* integer special case: codes holding small integers that e4m3 / e2m1 / int8
  represent exactly, with unit scales, reduce to the textbook integer matmul;
* brute force on tiny shapes with a differently written loop (k outermost,
  python scalars), including non-uniform scales, so a transposed operand, a
  wrong scale index or a dropped term fails;
* Swap-AB identity (W . A^T)^T == A . W^T exactly;
* Split-K invariant: the K-slice partial sums add up exactly to the unsplit sum;
* scale invariants: an A row times 2^k scales that y row by 2^k exactly; a
  negated W row negates that y column;
* Block_FP8 with all group scales of a row / block equal reduces to
  FP8_Dynamic with those scales.
"""
import numpy as np
import pytest

import qg_synth
from oracle import formats as F
from oracle import gemm as G
from oracle import quant as Q


def _bits(x):
    return qg_synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _int_codes_e4m3(rng, shape, lo=-16, hi=16):
    v = rng.integers(lo, hi + 1, size=shape).astype(np.float64)
    return F.encode_e4m3(v), v


def test_integer_special_case_reduces_to_integer_matmul():
    rng = np.random.default_rng(0)
    qa, va = _int_codes_e4m3(rng, (7, 96))
    qw, vw = _int_codes_e4m3(rng, (5, 96))
    ref = va.astype(np.int64) @ vw.astype(np.int64).T
    one_a = np.ones(7, np.float32)
    one_w = np.ones(5, np.float32)
    assert np.array_equal(G.acc_e4m3(qa, qw), ref.astype(np.float64))
    y = G.fp8_dynamic(qa, one_a, qw, one_w)
    assert np.array_equal(y, F.bf16_round(ref.astype(np.float64)))
    ia = rng.integers(-127, 128, size=(7, 96)).astype(np.int8)
    iw = rng.integers(-127, 128, size=(5, 96)).astype(np.int8)
    ref_i = ia.astype(np.int64) @ iw.astype(np.int64).T
    assert np.array_equal(G.acc_int8(ia, iw), ref_i)
    # e2m1 half-integers with unit block scales (code 0x38 = 1.0) and g = 1
    v4 = rng.choice(F.E2M1_TABLE[:16], size=(3, 64))
    w4 = rng.choice(F.E2M1_TABLE[:16], size=(4, 64))
    q4a, q4w = F.encode_e2m1(v4), F.encode_e2m1(w4)
    ones_a = np.full((3, 4), 0x38, np.uint8)
    ones_w = np.full((4, 4), 0x38, np.uint8)
    ref4 = (np.rint(v4 * 2).astype(np.int64) @ np.rint(w4 * 2).astype(np.int64).T) / 4.0
    assert np.array_equal(G.nvfp4(q4a, ones_a, 1.0, q4w, ones_w, 1.0), F.bf16_round(ref4))


def _loop_fp8(qa, sa, qw, sw):
    M, K = qa.shape
    N = qw.shape[0]
    acc = [[0.0] * N for _ in range(M)]
    for k in range(K):                       # k outermost
        for m in range(M):
            a = float(F.E4M3_TABLE[qa[m, k]])
            for n in range(N):
                acc[m][n] += a * float(F.E4M3_TABLE[qw[n, k]])
    return np.array([[acc[m][n] * float(sa[m]) * float(sw[n]) for n in range(N)] for m in range(M)])


def test_brute_force_tiny_fp8_with_scales():
    a = qg_synth.bf16_matrix(0, 3, 64, 1.0)
    w = qg_synth.bf16_matrix(1, 4, 64, 0.02)
    qa, sa = Q.per_row_fp8(a)
    qw, sw = Q.per_row_fp8(w)
    ref = F.bf16_round(_loop_fp8(qa, sa, qw, sw))
    assert np.array_equal(G.fp8_dynamic(qa, sa, qw, sw), ref)


def test_brute_force_tiny_int8_with_scales():
    a = qg_synth.bf16_matrix(0, 4, 48, 1.0)
    w = qg_synth.bf16_matrix(1, 3, 48, 0.02)
    qa, sa = Q.per_row_int8(a)
    qw, sw = Q.per_row_int8(w)
    ref = np.zeros((4, 3))
    for k in range(48):
        for m in range(4):
            for n in range(3):
                ref[m, n] += int(qa[m, k]) * int(qw[n, k])
    ref = ref * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    assert np.array_equal(G.w8a8_int8(qa, sa, qw, sw), F.bf16_round(ref))


def test_brute_force_tiny_block_fp8():
    a = qg_synth.bf16_matrix(0, 2, 256, 1.0)
    w = qg_synth.bf16_matrix(1, 130, 256, 0.02)       # two row blocks, one ragged
    qa, sa = Q.act_groups_fp8(a)
    qw, sw = Q.weight_blocks_fp8(w)
    ref = np.zeros((2, 130))
    for m in range(2):
        for n in range(130):
            for g in range(2):
                p = 0.0
                for k in range(g * 128, (g + 1) * 128):
                    p += F.E4M3_TABLE[qa[m, k]] * F.E4M3_TABLE[qw[n, k]]
                ref[m, n] += p * float(sa[m, g]) * float(sw[n // 128, g])
    assert np.array_equal(G.block_fp8(qa, sa, qw, sw), F.bf16_round(ref))


def test_brute_force_tiny_nvfp4():
    a = qg_synth.bf16_matrix(0, 2, 64, 1.0)
    w = qg_synth.bf16_matrix(1, 3, 64, 0.02)
    qa, sfa, ga = Q.nvfp4(a)
    qw, sfw, gw = Q.nvfp4(w)
    ref = np.zeros((2, 3))
    for m in range(2):
        for n in range(3):
            for k in range(64):
                ref[m, n] += (F.E2M1_TABLE[qa[m, k]] * F.E4M3_TABLE[sfa[m, k // 16]]
                              * F.E2M1_TABLE[qw[n, k]] * F.E4M3_TABLE[sfw[n, k // 16]])
    # every product has at most 12 significant bits between 2^-20 and 2^23,
    # so both sums are exact in fp64 and the same number; the tensor scales
    # multiply in the same order, so the bf16 results are identical
    ref = ref * float(ga) * float(gw)
    got = G.nvfp4(qa, sfa, ga, qw, sfw, gw)
    assert np.array_equal(got, F.bf16_round(ref))


def test_swap_ab_identity_is_exact():
    a = qg_synth.bf16_matrix(0, 5, 384, 1.0)
    w = qg_synth.bf16_matrix(1, 33, 384, 0.02)
    qa, _ = Q.per_row_fp8(a)
    qw, _ = Q.per_row_fp8(w)
    assert np.array_equal(G.swap_ab(qa, qw), G.acc_e4m3(qa, qw))
    ia, _ = Q.per_row_int8(a)
    iw, _ = Q.per_row_int8(w)
    assert np.array_equal(G.swap_ab(ia, iw, G.acc_int8), G.acc_int8(ia, iw))


@pytest.mark.parametrize("splits", [2, 4, 8, 16])
def test_split_k_sum_equals_unsplit(splits):
    a = qg_synth.bf16_matrix(0, 4, 2048, 1.0)
    w = qg_synth.bf16_matrix(1, 16, 2048, 0.02)
    qa, _ = Q.per_row_fp8(a)
    qw, _ = Q.per_row_fp8(w)
    parts = G.split_k_partials(qa, qw, splits)
    total = parts[0].copy()
    for p in parts[1:]:
        total += p
    assert np.array_equal(total, G.acc_e4m3(qa, qw))
    ia, _ = Q.per_row_int8(a)
    iw, _ = Q.per_row_int8(w)
    parts = G.split_k_partials(ia, iw, splits, G.acc_int8)
    assert np.array_equal(sum(parts), G.acc_int8(ia, iw))


def _fp8_y(a, w):
    qa, sa = Q.per_row_fp8(a)
    qw, sw = Q.per_row_fp8(w)
    return G.fp8_dynamic(qa, sa, qw, sw)


@pytest.mark.parametrize("fmt", ["fp8", "int8", "block", "nvfp4"])
def test_scale_invariants(fmt):
    a = qg_synth.bf16_matrix(0, 4, 256, 1.0)
    w = qg_synth.bf16_matrix(1, 8, 256, 0.02)

    def run(a_bits, w_bits):
        if fmt == "fp8":
            return _fp8_y(a_bits, w_bits)
        if fmt == "int8":
            qa, sa = Q.per_row_int8(a_bits)
            qw, sw = Q.per_row_int8(w_bits)
            return G.w8a8_int8(qa, sa, qw, sw)
        if fmt == "block":
            qa, sa = Q.act_groups_fp8(a_bits)
            qw, sw = Q.weight_blocks_fp8(w_bits)
            return G.block_fp8(qa, sa, qw, sw)
        # nvfp4: the tensor scale is global, so scale the whole tensor
        qa, sfa, ga = Q.nvfp4(a_bits)
        qw, sfw, gw = Q.nvfp4(w_bits)
        return G.nvfp4(qa, sfa, ga, qw, sfw, gw)

    y = run(a, w)
    xa = F.bf16_from_bits(a).copy()
    if fmt == "nvfp4":
        y2 = run(_bits(xa * np.float32(4.0)), w)
        assert np.array_equal(y2, y * 4.0)
    else:
        xa[1] *= np.float32(2.0 ** 5)
        y2 = run(_bits(xa), w)
        assert np.array_equal(y2[1], y[1] * 32.0)
        assert np.array_equal(np.delete(y2, 1, 0), np.delete(y, 1, 0))
    xw = F.bf16_from_bits(w).copy()
    xw[3] = -xw[3]
    y3 = run(a, _bits(xw))
    assert np.array_equal(y3[:, 3], -y[:, 3])
    if fmt != "block":   # block scales are shared by 128 rows: the rest must not move
        assert np.array_equal(np.delete(y3, 3, 1), np.delete(y, 3, 1))


def test_block_fp8_reduces_to_fp8_dynamic_with_uniform_scales():
    rng = np.random.default_rng(3)
    qa = F.encode_e4m3(rng.uniform(-448, 448, (3, 256)))
    qw = F.encode_e4m3(rng.uniform(-448, 448, (128, 256)))
    sa = np.array([0.5, 2.0, 0.125], np.float32)
    sw = np.float32(0.25)
    y_block = G.block_fp8(qa, np.repeat(sa[:, None], 2, 1), qw, np.full((1, 2), sw, np.float32))
    y_dyn = G.fp8_dynamic(qa, sa, qw, np.full(128, sw, np.float32))
    assert np.array_equal(y_block, y_dyn)


# ---------------------------------------------------- grouped (MoE) GEMM --
def test_grouped_with_one_expert_is_the_plain_gemm():
    a = qg_synth.bf16_matrix(0, 5, 128, 1.0)
    w = qg_synth.bf16_matrix(1, 12, 128, 0.02)
    qa, sa = Q.per_row_int8(a)
    qw, sw = Q.per_row_int8(w)
    y = G.grouped(G.w8a8_int8, qa, sa, qw, sw, np.array([0, 5]), 12)
    assert np.array_equal(y, G.w8a8_int8(qa, sa, qw, sw))


def test_grouped_brute_force_routing_with_an_empty_expert():
    # 3 experts x N = 4 channels; tokens 0-1 -> expert 0, none -> expert 1,
    # tokens 2-4 -> expert 2: every y row uses its own expert's weight rows
    a = qg_synth.bf16_matrix(0, 5, 64, 1.0)
    w = qg_synth.bf16_matrix(1, 12, 64, 0.02)
    qa, sa = Q.per_row_fp8(a)
    qw, sw = Q.per_row_fp8(w)
    offsets = np.array([0, 2, 2, 5])
    expert_of = [0, 0, 2, 2, 2]
    ref = np.zeros((5, 4))
    for t in range(5):
        e = expert_of[t]
        for n in range(4):
            s = 0.0
            for k in range(64):
                s += F.E4M3_TABLE[qa[t, k]] * F.E4M3_TABLE[qw[e * 4 + n, k]]
            ref[t, n] = s * float(sa[t]) * float(sw[e * 4 + n])
    assert np.array_equal(G.grouped(G.fp8_dynamic, qa, sa, qw, sw, offsets, 4), F.bf16_round(ref))


def test_grouped_block_scales_follow_the_expert():
    # Block_FP8 with 128-row weight blocks: swapping the two experts' weights
    # (rows and block scales) swaps which tokens see which weights
    a = qg_synth.bf16_matrix(0, 6, 256, 1.0)
    w = qg_synth.bf16_matrix(1, 256, 256, 0.02)
    qa, sa = Q.act_groups_fp8(a)
    qw, sw = Q.weight_blocks_fp8(w)
    offsets = np.array([0, 4, 6])
    y = G.grouped(G.block_fp8, qa, sa, qw, sw, offsets, 128, w_rows_per_scale=128)
    assert np.array_equal(y[:4], G.block_fp8(qa[:4], sa[:4], qw[:128], sw[:1]))
    assert np.array_equal(y[4:], G.block_fp8(qa[4:], sa[4:], qw[128:], sw[1:]))
    qw_s = np.concatenate([qw[128:], qw[:128]])
    sw_s = np.concatenate([sw[1:], sw[:1]])
    y_s = G.grouped(G.block_fp8, qa, sa, qw_s, sw_s, offsets, 128, w_rows_per_scale=128)
    assert np.array_equal(y_s[:4], G.block_fp8(qa[:4], sa[:4], qw[128:], sw[1:]))
    assert not np.array_equal(y_s[:4], y[:4])


def test_grouped_nvfp4_brute_force_with_per_expert_tensor_scales():
    # 3 experts x N = 4 channels, tokens 0-2 -> expert 0, none -> expert 1,
    # tokens 3-4 -> expert 2; each y element is summed here token by token,
    # element by element, with its own expert's block scales and tensor scale
    a = qg_synth.bf16_matrix(0, 5, 64, 1.0)
    w = qg_synth.bf16_matrix(1, 12, 64, 0.02)
    w[8:] = qg_synth.f32_to_bf16_bits(qg_synth.bf16_bits_to_f32(w[8:]) * np.float32(64.0))   # expert 2: other amax
    qa, sfa, ga = Q.nvfp4(a)
    qw, sfw, gw = Q.nvfp4_experts(w, 3)
    offsets = np.array([0, 3, 3, 5])
    expert_of = [0, 0, 0, 2, 2]
    ref = np.zeros((5, 4))
    for t in range(5):
        e = expert_of[t]
        for n in range(4):
            s = 0.0
            for k in range(64):
                s += (F.E2M1_TABLE[qa[t, k]] * F.E4M3_TABLE[sfa[t, k // 16]] *
                      F.E2M1_TABLE[qw[e * 4 + n, k]] * F.E4M3_TABLE[sfw[e * 4 + n, k // 16]])
            ref[t, n] = s * float(ga) * float(gw[e])
    y = G.grouped_nvfp4(qa, sfa, ga, qw, sfw, gw, offsets, 4)
    assert np.array_equal(y, F.bf16_round(ref))


def test_nvfp4_experts_scale_each_expert_by_its_own_amax():
    # expert 1 is expert 0 times 2^5: the same codes and block scales, a
    # tensor scale 2^5 larger, each tensor scale amax_e / 2688 in fp32
    # (a single scale over the stack would change expert 0's block scales)
    w0 = qg_synth.bf16_matrix(3, 16, 64, 0.02)
    w1 = qg_synth.f32_to_bf16_bits(qg_synth.bf16_bits_to_f32(w0) * np.float32(32.0))
    q, sf, g = Q.nvfp4_experts(np.concatenate([w0, w1]), 2)
    assert np.array_equal(q[:16], q[16:]) and np.array_equal(sf[:16], sf[16:])
    assert g[1] == np.float32(32.0) * g[0]
    amax0 = np.float32(np.abs(qg_synth.bf16_bits_to_f32(w0)).max())
    assert g[0] == np.float32(amax0 / np.float32(2688.0))
    q_all, sf_all, _ = Q.nvfp4(np.concatenate([w0, w1]))
    assert not np.array_equal(sf_all[:16], sf[:16])


def test_grouped_nvfp4_with_one_expert_is_the_plain_gemm():
    a = qg_synth.bf16_matrix(0, 6, 128, 1.0)
    w = qg_synth.bf16_matrix(1, 8, 128, 0.02)
    qa, sfa, ga = Q.nvfp4(a)
    qw, sfw, gw = Q.nvfp4_experts(w, 1)
    qw1, sfw1, gw1 = Q.nvfp4(w)
    assert np.array_equal(qw, qw1) and np.array_equal(sfw, sfw1) and gw[0] == gw1
    y = G.grouped_nvfp4(qa, sfa, ga, qw, sfw, gw, np.array([0, 6]), 8)
    assert np.array_equal(y, G.nvfp4(qa, sfa, ga, qw1, sfw1, gw1))
