"""Pins for the oracle's element codecs (CPU only).

The codecs are checked against torch's float8 dtypes (a library implementation,
used here and nowhere in the oracle) over every code, and against a generic
minifloat decoder written from the bit-field definition and itself validated on
torch's E4M3 / E5M2 before it is applied to E2M1.
"""
import math

import numpy as np
import pytest
import torch

from oracle.formats import (decode_e2m1, decode_e4m3, decode_ue8m0,
                            encode_e4m3_rne_satfinite, unpack_e2m1_pairs)


def _minifloat(code, ebits, mbits, bias, nan_all_ones=False, has_inf=False):
    """Generic sign/exponent/mantissa decoder from the bit-field definition."""
    s = (code >> (ebits + mbits)) & 1
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    emax = (1 << ebits) - 1
    if has_inf and e == emax:
        v = math.inf if m == 0 else math.nan
    elif nan_all_ones and e == emax and m == (1 << mbits) - 1:
        v = math.nan
    elif e == 0:
        v = m / (1 << mbits) * 2.0 ** (1 - bias)
    else:
        v = (1 + m / (1 << mbits)) * 2.0 ** (e - bias)
    return -v if s else v


def test_minifloat_decoder_matches_torch_fp8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref43 = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref52 = codes.view(torch.float8_e5m2).to(torch.float64).numpy()
    mine43 = np.array([_minifloat(c, 4, 3, 7, nan_all_ones=True) for c in range(256)])
    mine52 = np.array([_minifloat(c, 5, 2, 15, has_inf=True) for c in range(256)])
    np.testing.assert_array_equal(mine43, ref43)
    np.testing.assert_array_equal(mine52, ref52)


def test_decode_e4m3_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = decode_e4m3(codes)
    np.testing.assert_array_equal(got, ref)          # NaNs in the same places
    assert got[0x7E] == 448.0 and got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9


def test_decode_e2m1_all_codes_vs_generic_minifloat():
    got = decode_e2m1(np.arange(16))
    ref = np.array([_minifloat(c, 2, 1, 1) for c in range(16)])
    np.testing.assert_array_equal(got, ref)
    assert got.max() == 6.0 and got[0] == 0.0


def test_unpack_e2m1_low_nibble_first():
    packed = np.array([[0x21, 0xF7]], dtype=np.uint8)
    np.testing.assert_array_equal(unpack_e2m1_pairs(packed), [[1, 2, 7, 15]])


def test_decode_ue8m0_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal(decode_ue8m0(codes), ref)


def test_encode_e4m3_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(encode_e4m3_rne_satfinite(decode_e4m3(codes)), codes)


def test_encode_e4m3_vs_torch_rne_in_range():
    rng = np.random.default_rng(0)
    # f32-representable values over the whole range, incl. subnormals and exact
    # midpoints between neighbouring codes (tie cases)
    finite = decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = (finite[:-1] + finite[1:]) / 2
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
        mids, -mids, rng.uniform(448, 463.9, 200)]).astype(np.float32)
    vals = vals[np.abs(vals) < 464.0]     # torch maps |v| >= 464 to NaN, not 448
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = encode_e4m3_rne_satfinite(vals.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_encode_e4m3_saturates_and_keeps_sign():
    got = encode_e4m3_rne_satfinite(np.array([1e6, -1e6, 464.0, -0.0, -1e-12, np.nan]))
    np.testing.assert_array_equal(got, [0x7E, 0xFE, 0x7E, 0x80, 0x80, 0x7F])
