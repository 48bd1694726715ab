"""Pins for the oracle's scalar codecs (fp16, bf16, FP8 e4m3, FP4 e2m1).

Each codec is written in the oracle from its format definition; here it is
checked against something other than itself:
  * fp16  -- numpy's IEEE binary16 conversion (library routine), plus
             hand-picked ties, subnormals and overflow;
  * bf16  -- torch's fp32 -> bfloat16 conversion (library routine);
  * e4m3  -- all 256 codes decoded against the OCP FP8 value formula typed
             out here, and encoding against torch's float8_e4m3fn conversion
             for in-range values, plus saturation;
  * e2m1  -- the eight magnitudes of the OCP FP4 format and brute-force
             nearest-value search with ties to the even code.
"""
import math

import numpy as np
import pytest
import torch

pytestmark = []


def test_f16_against_numpy(orc):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 4000),
        np.array([0.0, -0.0, 1.0, 65504.0, 65519.0, 65520.0, 70000.0, 2.0 ** -24, 2.0 ** -25,
                  1.5 * 2.0 ** -25, 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11], np.float32),
    ])
    for v in vals:
        want = np.array([v], np.float64).astype(np.float16).view(np.uint16)[0]
        assert orc.f16_bits(float(v)) == int(want), v
    for b in list(range(0, 0x7C00, 97)) + [1, 0x3FF, 0x400, 0x7BFF]:
        assert orc.f16_value(b) == float(np.array([b], np.uint16).view(np.float16)[0])


def test_f16_ties_hand(orc):
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: ties to the even mantissa (1.0).
    assert orc.f16_bits(1.0 + 2.0 ** -11) == 0x3C00
    # 1 + 3*2^-11 lies halfway between 1+2^-10 (odd) and 1+2^-9 (even).
    assert orc.f16_bits(1.0 + 3 * 2.0 ** -11) == 0x3C02
    # smallest subnormal 2^-24 = 0x0001; half of it ties to zero
    assert orc.f16_bits(2.0 ** -24) == 0x0001
    assert orc.f16_bits(2.0 ** -25) == 0x0000
    assert orc.f16_bits(65520.0) == 0x7C00
    assert orc.f16_bits(-65504.0) == 0xFBFF


def test_bf16_against_torch(orc):
    rng = np.random.default_rng(2)
    vals = (rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000)).astype(np.float32)
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_bits(float(v)) for v in vals], np.uint16)
    np.testing.assert_array_equal(got, want)
    for b in range(0, 0x7F80, 131):
        assert orc.bf16_value(b) == float(torch.tensor([b], dtype=torch.int16).view(torch.bfloat16).float())


def _e4m3_formula(c: int) -> float:
    """OCP 8-bit floating point (E4M3, bias 7, no infinities)."""
    s = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 7
    if e == 0xF and m == 7:
        return math.nan
    if e == 0:
        return s * 2.0 ** -6 * (m / 8.0)
    return s * 2.0 ** (e - 7) * (1.0 + m / 8.0)


def test_e4m3_decode_all_codes(orc):
    for c in range(256):
        a, b = orc.e4m3_value(c), _e4m3_formula(c)
        assert (math.isnan(a) and math.isnan(b)) or a == b, c
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_against_torch(orc):
    rng = np.random.default_rng(3)
    vals = (rng.standard_normal(20000) * 10.0 ** rng.uniform(-3.5, 2.6, 20000)).astype(np.float32)
    vals = np.clip(vals, -448.0, 448.0)
    # every midpoint between neighbouring finite codes (ties) as well
    fin = sorted({_e4m3_formula(c) for c in range(0x7F) if not math.isnan(_e4m3_formula(c))})
    mids = np.array([(a + b) / 2 for a, b in zip(fin[:-1], fin[1:])], np.float32)
    vals = np.concatenate([vals, mids, -mids])
    want = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_code(float(v)) for v in vals], np.uint8)
    np.testing.assert_array_equal(got, want)


def test_e4m3_saturates(orc):
    assert orc.e4m3_code(448.0) == 0x7E
    assert orc.e4m3_code(470.0) == 0x7E
    assert orc.e4m3_code(1.0e6) == 0x7E
    assert orc.e4m3_code(-1.0e6) == 0xFE


E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # OCP FP4 (E2M1) magnitudes, codes 0..7


def test_e2m1_decode(orc):
    for c in range(16):
        want = (-1.0 if c & 8 else 1.0) * E2M1_MAGS[c & 7]
        assert orc.e2m1_value(c) == want


def test_e2m1_ties_and_saturation(orc):
    # ties go to the even code (mantissa bit 0)
    table = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0, 7.0: 6.0, 100.0: 6.0}
    for v, want in table.items():
        assert orc.e2m1_value(orc.e2m1_code(v)) == want, v
        assert orc.e2m1_value(orc.e2m1_code(-v)) == -want, v


def test_e2m1_brute_force(orc):
    rng = np.random.default_rng(4)
    for v in rng.uniform(-8, 8, 3000):
        a = abs(v)
        d = [abs(a - m) for m in E2M1_MAGS]
        best = min(d)
        cands = [c for c in range(8) if d[c] == best]
        c = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        got = orc.e2m1_code(float(v))
        assert got & 7 == c and (got >> 3) == (1 if v < 0 else 0), v
