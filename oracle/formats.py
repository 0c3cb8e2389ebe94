"""Element formats used by the MoE layer, decoded and encoded exactly in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages name the formats (FP8 E4M3 weights and activations, UE8M0 block
scales, MXFP4 = E2M1 weights: DeepGEMM PR #445 "Environment"; DeepGEMM PR #386
title "native UE8M0"; TensorRT-LLM PR #16346 "Description") but do not define
them.  The definitions below are the OCP 8-bit floating point / Microscaling
format definitions:

  E4M3 (fn):  1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
              S.1111.111 is NaN; largest finite 448; exponent field 0 is
              subnormal with value m/8 * 2^-6.
  E2M1:       1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes
              {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no NaN / inf.
  UE8M0:      8-bit unsigned exponent, value 2^(b-127); b = 255 is NaN.
  BF16:       the upper 16 bits of an IEEE-754 binary32 (1 sign, 8 exponent
              bits with bias 127, 7 mantissa bits); same range as binary32.

Parity: pinned by exhaustive enumeration against torch's float8_e4m3fn /
float8_e8m0fnu / float4_e2m1fn_x2 dtypes (library routines used only in the
tests) and against the format constants above.
"""
import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def decode_e4m3(codes):
    """E4M3 byte codes -> float64 values (NaN for 0x7F / 0xFF)."""
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    exp = (b >> 3) & 0xF
    man = b & 0x7
    normal = (1.0 + man / 8.0) * np.exp2(exp - 7.0)
    sub = (man / 8.0) * np.exp2(-6.0)
    mag = np.where(exp == 0, sub, normal)
    mag = np.where((exp == 15) & (man == 7), np.nan, mag)
    return sign * mag


def _e4m3_positive_table():
    codes = np.arange(0, 0x7F, dtype=np.uint8)          # 0x00 .. 0x7E, all finite
    return codes, decode_e4m3(codes)


def encode_e4m3_rne_satfinite(values):
    """float64 -> E4M3 byte codes, round to nearest, ties to even mantissa, and
    saturation of finite out-of-range magnitudes to +-448.  The sign of a value
    that rounds to zero is kept (-0 -> 0x80).  NaN -> 0x7F."""
    v = np.asarray(values, dtype=np.float64)
    codes, mags = _e4m3_positive_table()               # mags ascending with code
    a = np.abs(v)
    a_sat = np.minimum(a, E4M3_MAX)
    hi = np.searchsorted(mags, a_sat, side="left")      # first mag >= a
    hi = np.clip(hi, 0, len(mags) - 1)
    lo = np.clip(hi - 1, 0, len(mags) - 1)
    d_lo = a_sat - mags[lo]
    d_hi = mags[hi] - a_sat
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    c = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    c = np.where(np.signbit(v), c | 0x80, c).astype(np.uint8)
    c = np.where(np.isnan(v), np.uint8(0x7F), c).astype(np.uint8)
    return c


_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def decode_e2m1(nibbles):
    """E2M1 4-bit codes (values 0..15) -> float64."""
    n = np.asarray(nibbles).astype(np.int64) & 0xF
    mag = _E2M1_MAG[n & 0x7]
    return np.where(n & 0x8, -mag, mag)


def unpack_e2m1_pairs(packed):
    """Bytes holding two E2M1 codes each -> codes, element 2i from the low
    nibble and element 2i+1 from the high nibble (last axis doubles)."""
    p = np.asarray(packed, dtype=np.uint8)
    lo = p & 0xF
    hi = p >> 4
    out = np.stack([lo, hi], axis=-1)
    return out.reshape(p.shape[:-1] + (p.shape[-1] * 2,))


def decode_ue8m0(codes):
    """UE8M0 scale bytes -> float64 2^(b-127); 255 -> NaN."""
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    val = np.exp2(b - 127.0)
    return np.where(b == 255, np.nan, val)


BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def decode_bf16(bits):
    """BF16 bit patterns (uint16) -> float64: the pattern is the upper half of a
    binary32, so widening it by 16 zero bits gives the exact value."""
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def encode_bf16_rne(values):
    """float64 -> BF16 bit patterns (uint16), rounding the exact value to the
    nearest BF16 number with ties to the even mantissa; magnitudes that round
    past the largest finite value give infinity; NaN gives 0x7FC0.

    Rounding step: for |v| in [2^E, 2^(E+1)) the BF16 spacing is 2^(E-7), and
    2^-133 below the smallest normal 2^-126 (8 significant bits, 7 stored)."""
    v = np.asarray(values, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        _, ex = np.frexp(a)                       # a = m * 2^ex, m in [0.5, 1)
        E = np.maximum(ex.astype(np.int64) - 1, -126)
        q = np.ldexp(1.0, (E - 7).astype(np.int64))
        r = np.rint(a / q) * q                    # rint: round half to even
    r = np.where(a == 0, 0.0, r)
    r = np.where(r > BF16_MAX, np.inf, r)
    r = np.where(np.isinf(a), np.inf, r)
    out = (np.copysign(r, v).astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return np.where(np.isnan(v), np.uint16(0x7FC0), out).astype(np.uint16)
