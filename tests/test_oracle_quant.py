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
