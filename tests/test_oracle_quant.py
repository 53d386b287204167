"""Pins of the oracle's quantisers (closed forms, invariants, special cases).

* the amax element of a row maps to the format's extreme code (+-448 / +-127);
* scaling a row by 2^k leaves its codes unchanged and scales its scale by 2^k;
* reconstruction error bounds (|x - q s| <= s/2 for int8; within half an
  e4m3 spacing of x/s for fp8);
* all-zero rows give scale 1 and codes 0;
* a Block_FP8 group whose values equal one whole row reduces to per-token;
* NVFP4: block scales never exceed 448, element codes stay within +-6, the
  tensor scale and the 2^k invariance hold.
"""
import numpy as np
import pytest

import qg_synth
from oracle import formats as F
from oracle import quant as Q


def _bits(x):
    return qg_synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _act(M, K, seed=0):
    return qg_synth.bf16_matrix(seed, M, K, 1.0)


def test_per_row_fp8_extreme_and_zero_row():
    a = qg_synth.with_edge_rows(_act(5, 256))
    q, s = Q.per_row_fp8(a)
    x = F.bf16_from_bits(a)
    assert s[0] == 1.0 and np.all(q[0] == 0)
    for r in range(1, 5):
        k = np.argmax(np.abs(x[r]))
        assert F.E4M3_TABLE[q[r, k]] == np.copysign(448.0, x[r, k])
        assert s[r] == np.float32(np.abs(x[r]).max()) / np.float32(448.0)


def test_per_row_int8_bounds_and_extreme():
    a = qg_synth.with_edge_rows(_act(6, 512, seed=3))
    q, s = Q.per_row_int8(a)
    x = F.bf16_from_bits(a).astype(np.float64)
    assert s[0] == 1.0 and np.all(q[0] == 0)
    assert q.min() >= -127 and q.max() <= 127
    err = np.abs(x - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 1e-6))
    for r in range(1, 6):
        k = np.argmax(np.abs(x[r]))
        assert abs(int(q[r, k])) == 127


@pytest.mark.parametrize("fn", [Q.per_row_fp8, Q.per_row_int8, Q.act_groups_fp8])
def test_power_of_two_row_scaling(fn):
    a = _act(4, 256, seed=5)
    x = F.bf16_from_bits(a)
    q0, s0 = fn(a)
    for k in (-6, 3, 10):
        q1, s1 = fn(_bits(x * np.float32(2.0 ** k)))
        assert np.array_equal(q0, q1)
        assert np.array_equal(s1, (s0 * np.float32(2.0 ** k)).astype(np.float32))


def test_fp8_reconstruction_within_half_spacing():
    a = _act(8, 1024, seed=11)
    q, s = Q.per_row_fp8(a)
    x = F.bf16_from_bits(a).astype(np.float64)
    r = x / s[:, None].astype(np.float64)
    d = F.decode_e4m3(q)
    pos = F.E4M3_TABLE[:0x7F]
    idx = np.clip(np.searchsorted(pos, np.abs(d)), 1, len(pos) - 1)
    spacing = np.maximum(pos[np.minimum(idx + 1, len(pos) - 1)] - pos[idx], pos[idx] - pos[idx - 1])
    assert np.all(np.abs(r - d) <= spacing / 2 + 1e-4 * np.abs(r))


def test_block_act_groups_reduce_to_per_token_when_k_is_one_group():
    a = _act(6, 128, seed=13)
    qg, sg = Q.act_groups_fp8(a)
    qt, st = Q.per_row_fp8(a)
    assert np.array_equal(qg, qt) and np.array_equal(sg[:, 0], st)


def test_weight_blocks_match_row_quant_on_one_row_block_with_equal_amax():
    # A 128x128 block whose rows all share the block amax: per-block and
    # per-channel scales coincide, so the codes must coincide too.
    w = qg_synth.bf16_matrix(1, 128, 128, 0.02)
    x = F.bf16_from_bits(w).copy()
    m = np.abs(x).max()
    x[:, 0] = m                                   # every row now has amax == m
    wb = _bits(x)
    qb, sb = Q.weight_blocks_fp8(wb)
    qr, sr = Q.per_row_fp8(wb)
    assert np.all(sr == sb[0, 0]) and np.array_equal(qb, qr)


def test_weight_blocks_ragged_rows():
    w = qg_synth.bf16_matrix(1, 200, 256, 0.02)
    q, s = Q.weight_blocks_fp8(w)
    assert s.shape == (2, 2)
    x = F.bf16_from_bits(w)
    assert s[1, 1] == np.float32(np.abs(x[128:, 128:]).max()) / np.float32(448.0)


def test_nvfp4_structure_and_invariance():
    a = qg_synth.with_edge_rows(_act(6, 512, seed=17))
    q, sf, g = Q.nvfp4(a)
    x = F.bf16_from_bits(a)
    assert g == np.float32(np.abs(x).max()) / np.float32(2688.0)
    sfv = F.decode_e4m3(sf)
    assert np.all(sfv >= 0) and sfv.max() <= 448.0
    assert np.all(q[0] == 0)
    # the tensor amax element lands on +-6 with block scale 448
    r, k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert sfv[r, k // 16] == 448.0 and abs(F.E2M1_TABLE[q[r, k]]) == 6.0
    # dequantised value within half an e2m1 step (relative to block scale)
    deq = F.decode_e2m1(q) * np.repeat(sfv, 16, axis=1) * float(g)
    step = np.repeat(sfv, 16, axis=1) * float(g)       # spacing <= 2 * scale at the top
    assert np.all(np.abs(deq - x) <= step + 1e-12)
    # 2^k invariance of codes; the tensor scale absorbs the factor
    q2, sf2, g2 = Q.nvfp4(_bits(x * np.float32(8.0)))
    assert np.array_equal(q, q2) and np.array_equal(sf, sf2) and g2 == g * np.float32(8.0)


def test_nvfp4_static_global_scale():
    a = _act(2, 64, seed=19)
    q, sf, g = Q.nvfp4(a, global_amax=1000.0)
    assert g == np.float32(1000.0) / np.float32(2688.0)


# ---------------------------------------------------------------------------
# Hand-derived rounding decisions.  The reading of the quantisers rounds the
# fp32 quotient x / s half to even ("Helion in the vLLM backend", first
# paragraph, names W8A8_INT8; the symmetric int8 recipe rounds to nearest,
# and the tie rule is the reading stated with the oracle).  Every expected
# code below is worked out by hand in the comments, not by the oracle.

def _int8_tie_row(scale_num):
    """One row whose amax is 127 * scale_num, so that s = amax / 127 is
    exactly scale_num, followed by the values (k + 1/2) * scale_num for
    k = -127 .. 126 (each a tie of the fp32 quotient x / s)."""
    ks = np.arange(-127, 127)
    vals = np.concatenate([[127.0], ks + 0.5]) * scale_num
    return vals, ks


@pytest.mark.parametrize("scale_num", [1.0, 2.0, 0.25])
def test_int8_ties_round_half_to_even(scale_num):
    # scale_num = 1: the row [127, -126.5, ..., 126.5]; amax 127 gives
    # s = 127 / 127 = 1 exactly, and x / s = k + 1/2 is a tie between k and
    # k + 1.  Half to even picks the even one of the two: 0.5 -> 0,
    # 1.5 -> 2, 2.5 -> 2, -0.5 -> 0, -1.5 -> -2, 125.5 -> 126, -126.5 -> -126.
    # Half away from zero would give 1, 2, 3, -1, -2, 126, -127 instead.
    # scale_num = 2 (amax 254, s = 2) and 0.25 (amax 31.75, s = 0.25): the
    # same quotients, every value exact in bf16 (at most 8 significant bits).
    vals, ks = _int8_tie_row(scale_num)
    a = _bits(vals[None, :])
    assert np.array_equal(F.bf16_from_bits(a)[0].astype(np.float64), vals)   # exact in bf16
    q, s = Q.per_row_int8(a)
    assert s[0] == np.float32(scale_num)
    want = np.where(ks % 2 == 0, ks, ks + 1)         # the even one of k and k + 1
    assert q[0, 0] == 127
    assert np.array_equal(q[0, 1:].astype(np.int64), want)
    # sign symmetry: -x gives -code at every tie
    qn, _ = Q.per_row_int8(_bits(-vals[None, :]))
    assert np.array_equal(qn[0].astype(np.int64), -q[0].astype(np.int64))


def test_int8_one_ulp_either_side_of_a_tie():
    # s = 1 (amax 127).  Around the tie 2.5 the bf16 neighbours are
    # 2.5 - 2^-6 and 2.5 + 2^-6 (bf16 keeps 8 significant bits, so the
    # spacing in [2, 4) is 2^-6): they round to 2 and 3, while 2.5 itself
    # goes to 2.  Around -0.5 (spacing 2^-8 above 0.5 in magnitude, 2^-9
    # below): -0.5 - 2^-8 goes to -1, -0.5 + 2^-9 to 0, -0.5 itself to 0.
    # Around 63.5 (spacing 2^-2 in [32, 64)): 63.25 -> 63, 63.5 -> 64,
    # 63.75 -> 64.
    vals = np.array([127.0, 2.5 - 2 ** -6, 2.5, 2.5 + 2 ** -6, -0.5 - 2 ** -8, -0.5, -0.5 + 2 ** -9,
                     63.25, 63.5, 63.75])
    a = _bits(vals[None, :])
    assert np.array_equal(F.bf16_from_bits(a)[0].astype(np.float64), vals)
    q, s = Q.per_row_int8(a)
    assert s[0] == 1.0
    assert q[0].tolist() == [127, 2, 2, 3, -1, 0, 0, 63, 64, 64]


# NVFP4 hand-worked blocks.  Reading (stated with the oracle): g =
# amax(tensor) / (448 * 6); block scale code = e4m3_RNE_satfinite((amax_b /
# 6) / g); code = e2m1_RNE_satfinite(x / (dec(block scale) * g)); code 0
# wherever the block scale decodes to 0.  e2m1 magnitudes in code order:
# 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7, sign bit 8).  e4m3 codes near 14:
# 0x56 = 1.110b * 2^3 = 14, 0x57 = 15, 0x58 = 16.
NVFP4_ROW0 = [6, 5, -5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, -0.25, 0, 4.5, 2.75, 1.125, -6, 0.625]
NVFP4_ROW1 = [87, 70, 49, 35, 24.5, 17.5, 10.5, 3.5, -87, 7, 21, 42, 56, 0, -3.5, 28]
NVFP4_ROW2 = [6 * 2 ** -10, 2 ** -8, -(2 ** -8), 2 ** -9, 0, 3 * 2 ** -10, -6 * 2 ** -10, 2 ** -10,
              0, 0, 0, 0, 0, 0, 0, 2 ** -8]


def _nvfp4_hand_tensor():
    return np.array([np.array(NVFP4_ROW0) * 448.0, NVFP4_ROW1, NVFP4_ROW2])


def test_nvfp4_hand_worked_blocks():
    x = _nvfp4_hand_tensor()
    a = _bits(x)
    assert np.array_equal(F.bf16_from_bits(a).astype(np.float64), x)   # every value exact in bf16
    q, sf, g = Q.nvfp4(a)
    # tensor amax = 6 * 448 = 2688, so g = 2688 / 2688 = 1 exactly.
    assert g == np.float32(1.0)
    # Row 0: amax_b = 2688, (2688 / 6) / 1 = 448 -> e4m3 0x7E (448), d = 448
    # and x / d is the listed multiple exactly.  Codes: 6 -> 7; 5 is the tie
    # of 4 (code 6, even) and 6 (code 7) -> 6; -5 -> 8 | 6 = 14; 3.5, tie of
    # 3 (5) and 4 (6) -> 6; 2.5, tie of 2 (4) and 3 (5) -> 4; 1.75, tie of
    # 1.5 (3) and 2 (4) -> 4; 1.25, tie of 1 (2) and 1.5 (3) -> 2; 0.75, tie
    # of 0.5 (1) and 1 (2) -> 2; 0.25, tie of 0 (0) and 0.5 (1) -> 0; -0.25
    # -> -0 = 8 (the sign of x sets the sign bit); 0 -> 0; 4.5 -> 4 (6);
    # 2.75 -> 3 (5); 1.125 -> 1 (2); -6 -> 15; 0.625 -> 0.5 (1).
    # Row 1: amax_b = 87, 87 / 6 = 14.5, the tie of 14 (0x56, even mantissa)
    # and 15 (0x57) -> 0x56, d = 14 (a rounded-up scale would be 15).  x / 14:
    # 87 -> 6.21.. saturates to 6 (7); 70 -> 5, tie -> 4 (6); 49 -> 3.5 -> 4
    # (6); 35 -> 2.5 -> 2 (4); 24.5 -> 1.75 -> 2 (4); 17.5 -> 1.25 -> 1 (2);
    # 10.5 -> 0.75 -> 1 (2); 3.5 -> 0.25 -> 0 (0); -87 -> 15; 7 -> 0.5 (1);
    # 21 -> 1.5 (3); 42 -> 3 (5); 56 -> 4 (6); 0 -> 0; -3.5 -> -0 (8);
    # 28 -> 2 (4).
    # Row 2: amax_b = 6 * 2^-10, (amax_b / 6) / 1 = 2^-10, half of the
    # smallest e4m3 subnormal 2^-9: the tie of 0 (code 0, even) and 2^-9
    # (code 1) -> code 0, which decodes to 0, so every element code is 0
    # (without that rule x / 0 would saturate the non-zero elements to +-6).
    assert sf[:, 0].tolist() == [0x7E, 0x56, 0x00]
    assert q[0].tolist() == [7, 6, 14, 6, 4, 4, 2, 2, 0, 8, 0, 6, 5, 2, 15, 1]
    assert q[1].tolist() == [7, 6, 6, 4, 4, 2, 2, 0, 15, 1, 3, 5, 6, 0, 8, 4]
    assert q[2].tolist() == [0] * 16
