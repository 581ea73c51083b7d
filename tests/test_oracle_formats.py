"""Pins for oracle.formats: element codecs checked against independent
implementations (ml_dtypes, torch casts, exact rational brute force) and
against the one number the pages fix (q_max = 6 for FP4, SVDQuant summary
page, section 3 "Quantization preliminary")."""

import math
import struct
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F


def test_e2m1_decode_matches_ml_dtypes_and_qmax():
    codes = np.arange(16, dtype=np.uint8)
    ours = F.e2m1_decode(codes)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(ours, ref)
    assert np.array_equal(np.signbit(ours), np.signbit(ref))
    # q_max = 6 for 4-bit floating point (page, section 3)
    assert np.max(ours) == 6.0 and np.min(ours) == -6.0


def test_e4m3_decode_matches_two_libraries():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    ref1 = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ref2 = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for ref in (ref1, ref2):
        nan = np.isnan(ref)
        assert np.array_equal(nan, np.isnan(ours))
        np.testing.assert_array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0
    assert F.e4m3_decode(np.uint8(1)) == 2.0**-9  # smallest subnormal


def _random_f32(n, lo_exp, hi_exp, seed):
    g = np.random.default_rng(seed)
    mant = g.uniform(1.0, 2.0, n)
    exp = g.integers(lo_exp, hi_exp, n)
    sign = np.where(g.random(n) < 0.5, -1.0, 1.0)
    return (sign * np.ldexp(mant, exp)).astype(np.float32)


def _midpoints(grid):
    mids = (grid[:-1] + grid[1:]) / 2
    return np.concatenate([mids, -mids]).astype(np.float32)


def _nudge(x):
    x = np.asarray(x, np.float32)
    return np.concatenate([x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(-np.inf))])


def test_e2m1_encode_matches_ml_dtypes_in_range():
    grid = F.e2m1_decode(np.arange(8, dtype=np.uint8))
    vals = np.concatenate([_random_f32(20000, -4, 3, 1), _nudge(_midpoints(grid)), _nudge(grid),
                           np.float32([0.0, -0.0, 0.1, -0.1, 0.25, -0.25])])
    vals = vals[np.abs(vals) <= 6.0]
    ours = F.e2m1_encode(vals)
    ref = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    np.testing.assert_array_equal(ours, ref)


def test_e2m1_ties_and_saturation_table():
    # round half to even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    x = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 100.0, 1e30])
    want = np.float64([0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, 6.0])
    np.testing.assert_array_equal(F.e2m1_decode(F.e2m1_encode(x)), want)
    np.testing.assert_array_equal(F.e2m1_decode(F.e2m1_encode(-x)), -want)
    assert F.e2m1_encode(np.float32(-0.1)) == 0x8  # negative zero kept


def test_e4m3_encode_matches_ml_dtypes_in_range():
    grid = F.e4m3_decode(np.arange(127, dtype=np.uint8))
    vals = np.concatenate([_random_f32(50000, -14, 9, 2), _nudge(_midpoints(grid)), _nudge(grid)])
    vals = vals[np.abs(vals) <= 448.0]
    ours = F.e4m3_encode(vals)
    ref = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_saturates_and_roundtrips():
    assert F.e4m3_encode(np.float32(449.0)) == 0x7E
    assert F.e4m3_encode(np.float32(1e9)) == 0x7E
    assert F.e4m3_encode(np.float32(-1e9)) == 0xFE
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F.e4m3_decode(codes).astype(np.float32)
    np.testing.assert_array_equal(F.e4m3_encode(vals), codes)
    c2 = np.arange(16, dtype=np.uint8)
    np.testing.assert_array_equal(F.e2m1_encode(F.e2m1_decode(c2).astype(np.float32)), c2)


def test_bf16_matches_ml_dtypes_and_torch():
    g = np.random.default_rng(3)
    bits = g.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32)
    # force many exact ties (low half == 0x8000)
    bits[:50000] = (bits[:50000] & 0xFFFF0000) | 0x8000
    x = bits.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 3.0e38)]
    ours = F.bf16_bits(x)
    ref1 = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    ref2 = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref1)
    np.testing.assert_array_equal(ours, ref2)


def _bf16_exact(x):
    """Nearest 8-significant-bit value to a Python float, ties to even (frexp form)."""
    if x == 0.0:
        return x
    m, e = math.frexp(x)  # x = m 2^e, 0.5 <= |m| < 1
    return math.ldexp(round(m * 256.0), e - 8)  # round(): half to even, exact here


def test_bf16_from_f64_direct_rounding():
    from oracle.svdquant import bf16_from_f64

    g = np.random.default_rng(4)
    x = g.standard_normal(20000) * 10.0 ** g.integers(-6, 6, 20000)
    # double-rounding traps: a hair above a bf16 midpoint
    traps = np.array([1.0 + 2.0**-8 + 2.0**-30, -(1.0 + 2.0**-8 + 2.0**-40), 3.0 * (1 + 2.0**-9 + 2.0**-35)])
    x = np.concatenate([x, traps])
    ours = bf16_from_f64(x)
    ref = np.array([_bf16_exact(float(v)) for v in x])
    np.testing.assert_array_equal(ours, ref)
    assert ours[-3] == 1.0 + 2.0**-7  # rounding through float32 would give 1.0


def test_pack_roundtrip_and_nibble_order():
    c = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    p = F.pack_e2m1(c)
    assert p.tolist() == [[0x21, 0x43, 0x0F]]
    np.testing.assert_array_equal(F.unpack_e2m1(p), c)


# exact rational reference grids, used by the brute-force tests elsewhere too
def e2m1_table():
    t = []
    for code in range(8):
        e, m = code >> 1, code & 1
        v = Fraction(m, 2) if e == 0 else Fraction(2) ** (e - 1) * (1 + Fraction(m, 2))
        t.append((v, code))
    return t


def e4m3_table():
    t = []
    for code in range(127):
        e, m = code >> 3, code & 7
        v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else Fraction(2) ** (e - 7) * (1 + Fraction(m, 8))
        t.append((v, code))
    return t


def test_rational_tables_agree_with_decoders():
    for table, dec in ((e2m1_table(), F.e2m1_decode), (e4m3_table(), F.e4m3_decode)):
        for v, code in table:
            assert Fraction(float(dec(np.uint8(code)))) == v


def test_f32_rounding_is_ieee():
    x = np.array([1.0 + 2.0**-24, 1.0 + 3 * 2.0**-24, 0.1])
    for v, r in zip(x, F.f32(x)):
        assert float(r) == struct.unpack("<f", struct.pack("<f", float(v)))[0]


@pytest.mark.parametrize("v", [0.0, -0.0])
def test_zero_sign(v):
    code = F.e2m1_encode(np.float32(v))
    assert code == (0x8 if math.copysign(1.0, v) < 0 else 0)
