"""Element formats of the NVFP4 quantizer, written from their definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

* E2M1 (4-bit float): sign, 2 exponent bits (bias 1), 1 mantissa bit, no
  inf/NaN.  Largest magnitude 6 = the q_max the SVDQuant summary page gives for
  4-bit floating point (section 3, "Quantization preliminary").
* E4M3 (8-bit float, "fn" flavour): sign, 4 exponent bits (bias 7), 3
  mantissa bits, no inf, S.1111.111 is NaN, largest magnitude 448.  Used as the
  per-16-element block scale (always non-negative, so it doubles as UE4M3).
* bfloat16: the compute dtype of the 16-bit branch ("compute_dtype:
  bfloat16" in the Nunchaku-Lite quantization_config, Diffusers page).

Encoders round to nearest with ties to the even code and saturate to the
largest finite magnitude ("satfinite"); the sign of the input is kept, so a
negative value that rounds to zero gives negative zero (E2M1 code 0x8).  These
are readings: the pages fix only q_max = 6.  Decisions are taken on float32
inputs (the precision of the kernels), evaluated exactly in float64.
"""

import numpy as np

# --------------------------------------------------------------------------
# decoders: value of every code, straight from the bit fields
# --------------------------------------------------------------------------


def e2m1_decode(code):
    """Value of 4-bit E2M1 codes (uint8 array, low nibble used) as float64."""
    c = np.asarray(code, dtype=np.uint8) & 0xF
    sign = (c >> 3) & 1
    exp = ((c >> 1) & 3).astype(np.int64)
    man = (c & 1).astype(np.float64)
    normal = np.ldexp(1.0 + man / 2.0, (exp - 1).astype(np.int32))
    subnormal = man / 2.0  # exponent field 0: 2^(1-bias) * 0.m = m/2
    mag = np.where(exp == 0, subnormal, normal)
    return np.where(sign == 1, -mag, mag)


def e4m3_decode(code):
    """Value of 8-bit E4M3 codes as float64 (NaN for S.1111.111)."""
    c = np.asarray(code, dtype=np.uint8)
    sign = (c >> 7) & 1
    exp = ((c >> 3) & 0xF).astype(np.int64)
    man = (c & 7).astype(np.float64)
    normal = np.ldexp(1.0 + man / 8.0, (exp - 7).astype(np.int32))
    subnormal = np.ldexp(man / 8.0, -6)  # 2^(1-bias) * 0.m
    mag = np.where(exp == 0, subnormal, normal)
    mag = np.where((exp == 15) & (c & 7 == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


# non-negative finite grids, index == code magnitude bits (monotone in value)
_E2M1_GRID = e2m1_decode(np.arange(8, dtype=np.uint8))
_E4M3_GRID = e4m3_decode(np.arange(127, dtype=np.uint8))  # 0x7F is NaN


def _encode_nearest_even(v, grid, sign_bit):
    """Round-to-nearest, ties-to-even-code, saturating encoder on ``grid``.

    ``v`` holds float32 values (or float64 values exactly representable in
    float32); distances are formed in float64, which is exact wherever a tie
    can occur (the input then lies within a factor of two of both neighbours).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    n = grid.shape[0]
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, n - 1)
    lo = np.clip(hi - 1, 0, n - 1)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a <= grid[0], 0, mag)
    mag = np.where(a >= grid[-1], n - 1, mag)  # satfinite
    neg = np.signbit(v)
    return (mag | np.where(neg, sign_bit, 0)).astype(np.uint8)


def e2m1_encode(v):
    """E2M1 code (uint8, 0..15) of float32 values: RNE, satfinite, signed zero."""
    return _encode_nearest_even(v, _E2M1_GRID, 0x8)


def e4m3_encode(v):
    """E4M3 code (uint8) of float32 values: RNE, satfinite (|v| >= 448 -> 448)."""
    return _encode_nearest_even(v, _E4M3_GRID, 0x80)


# --------------------------------------------------------------------------
# float32 / bfloat16 rounding
# --------------------------------------------------------------------------


def f32(x):
    """Round to float32 (IEEE round-to-nearest-even), returned as float32."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16(x):
    """Round float32 values to bfloat16 (RNE); returned as float32 holding them.

    Finite inputs only.  The float32 bit pattern is rounded at bit 16 with
    ties to even, which is the definition of RNE for a format that keeps the
    top 16 bits of binary32.
    """
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x32.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(x32.shape)


def bf16_bits(x):
    """The 16-bit patterns (uint16) of bf16(x)."""
    return (bf16(x).view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits):
    """float32 values of bf16 bit patterns (uint16)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# nibble packing of E2M1 codes (two per byte, element 2i in the low nibble)
# --------------------------------------------------------------------------


def pack_e2m1(codes):
    """Pack [..., K] 4-bit codes into [..., K/2] bytes; element 2i -> low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed):
    """Inverse of ``pack_e2m1``."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
