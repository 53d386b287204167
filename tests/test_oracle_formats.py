"""Pins of the oracle's number formats against facts outside the oracle.

* the OCP OFP8 E4M3 and OCP MX E2M1 tables (golden fixtures with citations);
* exhaustive structure of all 256 E4M3 codes (2 NaN codes, max 448, min
  subnormal 2^-9, 126 distinct positive finite non-zero values, monotone);
* torch's own float8_e4m3fn conversion (a library routine) for every code
  and for 2^20 random fp32 values inside the finite range;
* hand-derived round-half-to-even cases at every midpoint;
* torch's fp32 -> bf16 conversion for the output rounding.
"""
import os

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            rows.append((c, float(v)))
    return rows


def test_e2m1_table_matches_mx_spec():
    for code, v in _read_table("e2m1_values.txt"):
        got = F.E2M1_TABLE[int(code)]
        assert got == v and np.signbit(got) == np.signbit(v), (code, got, v)


def test_e4m3_landmarks_match_ofp8_spec():
    for code, v in _read_table("e4m3_landmarks.txt"):
        got = F.E4M3_TABLE[int(code, 16)]
        if np.isnan(v):
            assert np.isnan(got), code
        else:
            assert got == v and np.signbit(got) == np.signbit(v), (code, got, v)


def test_e4m3_exhaustive_structure():
    t = F.E4M3_TABLE
    nan_codes = [c for c in range(256) if np.isnan(t[c])]
    assert nan_codes == [0x7F, 0xFF]
    fin = t[~np.isnan(t)]
    assert fin.max() == 448.0 and fin.min() == -448.0
    pos = fin[fin > 0]
    assert len(np.unique(pos)) == 126 and pos.min() == 2.0 ** -9
    # monotone on each sign half, mirror-symmetric
    assert np.all(np.diff(t[0x00:0x7F]) > 0)
    assert np.all(np.diff(t[0x80:0xFF]) < 0)
    assert np.array_equal(np.abs(t[0x00:0x7F]), np.abs(t[0x80:0xFF]))


def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (ref == F.E4M3_TABLE) | (np.isnan(ref) & np.isnan(F.E4M3_TABLE))
    assert same.all()


def test_encode_every_representable_value():
    for c in range(256):
        v = F.E4M3_TABLE[c]
        if np.isnan(v):
            continue
        assert F.encode_e4m3(np.array([v]))[0] == c, hex(c)
    for c in range(16):
        assert F.encode_e2m1(np.array([F.E2M1_TABLE[c]]))[0] == c, c


def test_encode_midpoints_round_half_to_even():
    # e4m3: between consecutive positive codes c and c+1, the midpoint must go
    # to whichever of the two codes is even (its mantissa LSB is 0).
    pos = F.E4M3_TABLE[:0x7F]
    for c in range(0x7E):
        mid = (pos[c] + pos[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert F.encode_e4m3(np.array([mid]))[0] == want, hex(c)
        assert F.encode_e4m3(np.array([-mid]))[0] == (want | 0x80), hex(c)
    # e2m1 ties, derived by hand from the MX table
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0,
             7.0: 6.0, 100.0: 6.0, 0.2: 0.0, 0.3: 0.5, 5.1: 6.0}
    for x, v in cases.items():
        assert F.E2M1_TABLE[F.encode_e2m1(np.array([x]))[0]] == v, x
        assert F.E2M1_TABLE[F.encode_e2m1(np.array([-x]))[0]] == -v, x


def test_encode_saturates_and_keeps_sign_of_zero():
    assert F.encode_e4m3(np.array([1e6]))[0] == 0x7E
    assert F.encode_e4m3(np.array([-1e6]))[0] == 0xFE
    assert F.encode_e4m3(np.array([464.0]))[0] == 0x7E     # beyond max: satfinite
    assert F.encode_e4m3(np.array([-0.0]))[0] == 0x80
    assert F.encode_e4m3(np.array([-1e-9]))[0] == 0x80     # rounds to -0
    assert F.encode_e2m1(np.array([-0.1]))[0] == 0x8


def test_encode_e4m3_matches_torch_on_random_fp32():
    rng = np.random.default_rng(1234)
    # log-uniform magnitudes across the whole e4m3 range incl. subnormals
    mag = np.exp2(rng.uniform(-12, np.log2(448.0), size=1 << 20))
    x = (mag * rng.choice([-1.0, 1.0], size=mag.shape)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.encode_e4m3(x)
    assert np.array_equal(got, ref)


def test_encode_error_within_half_gap():
    rng = np.random.default_rng(7)
    x = rng.uniform(-448, 448, size=1 << 16)
    d = F.decode_e4m3(F.encode_e4m3(x))
    pos = F.E4M3_TABLE[:0x7F]
    idx = np.clip(np.searchsorted(pos, np.abs(x)), 1, len(pos) - 1)
    half_gap = (pos[idx] - pos[idx - 1]) / 2
    assert np.all(np.abs(np.abs(x) - np.abs(d)) <= half_gap + 1e-300)


def test_bf16_round_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(99)
    x = (rng.standard_normal(1 << 18) * np.exp2(rng.integers(-40, 40, 1 << 18))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = F.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_round_ties_and_fp64_precision():
    one = 1.0
    ulp = 2.0 ** -7
    assert F.bf16_round(np.array([one + ulp / 2]))[0] == one                  # tie -> even
    assert F.bf16_round(np.array([one + 3 * ulp / 2]))[0] == one + 2 * ulp    # tie -> even (up)
    # just above a tie must round up: only exact fp64 rounding sees this
    assert F.bf16_round(np.array([one + ulp / 2 + 2.0 ** -40]))[0] == one + ulp
    assert F.bf16_round(np.array([-(one + ulp / 2 + 2.0 ** -40)]))[0] == -(one + ulp)
    assert F.bf16_round(np.array([0.0]))[0] == 0.0
