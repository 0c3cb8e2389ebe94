"""Pins for the oracle's BF16 variant: the codecs against torch's bfloat16 and an
exhaustive nearest-value search, the layer against its element-by-element tier
and against integer-exact sums."""
import math

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import layer as L


def _torch_bf16_bits(x32):
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def test_decode_every_pattern_matches_torch():
    b = np.arange(65536, dtype=np.uint16)
    ours = F.decode_bf16(b)
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def test_encode_matches_torch_on_binary32_inputs():
    rng = np.random.default_rng(7)
    parts = [
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(5000) * 10.0 ** rng.uniform(-40, 38, 5000)).astype(np.float32),
    ]
    # Exact ties and their neighbours: low 16 bits 0x8000, 0x7FFF, 0x8001, with
    # even and odd kept mantissas, at several exponents.
    hi = rng.integers(0, 0x7F7F, 4000, dtype=np.uint32) << np.uint32(16)
    for low in (0x8000, 0x7FFF, 0x8001, 0x0000):
        parts.append((hi | np.uint32(low)).view(np.float32))
    # Subnormal binary32 inputs and magnitudes beyond the largest BF16 value.
    parts.append((rng.integers(1, 1 << 23, 4000, dtype=np.uint32)).view(np.float32))
    parts.append(np.float32(F.BF16_MAX) * (1 + rng.uniform(0, 0.0039, 1000)).astype(np.float32))
    parts.append(np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38],
                          dtype=np.float32))
    x32 = np.concatenate(parts)
    x32 = x32[np.isfinite(x32) | np.isinf(x32)]
    x32 = np.concatenate([x32, -x32])
    ours = F.encode_bf16_rne(x32.astype(np.float64))
    ref = _torch_bf16_bits(x32)
    assert np.array_equal(ours, ref)


def test_encode_nan():
    assert F.encode_bf16_rne(np.array([np.nan]))[0] == 0x7FC0


def test_encode_float64_is_one_rounding_of_the_exact_value():
    """Values that are not binary32 numbers (a cast to float32 first would round
    twice): the result must be the nearest finite BF16 value by exhaustive
    search, ties to the even pattern."""
    fin = np.arange(0, 0x7F80, dtype=np.uint16)          # non-negative finite patterns
    vals = F.decode_bf16(fin)
    rng = np.random.default_rng(11)
    x = np.abs(rng.standard_normal(300)) * 10.0 ** rng.uniform(-30, 30, 300)
    # Just above / below a midpoint by less than a binary32 ulp.
    mids = (vals[100:400:3] + vals[101:401:3]) / 2
    x = np.concatenate([x, mids * (1 + 2.0 ** -40), mids * (1 - 2.0 ** -40), mids])
    for v in x:
        d = np.abs(vals - v)
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else best[fin[best] % 2 == 0][0]
        assert F.encode_bf16_rne(np.array([v]))[0] == fin[code], v


def test_scalar_and_vector_rounding_agree():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(3000) * 10.0 ** rng.uniform(-38, 38, 3000)
    # Exact midpoints between consecutive finite BF16 values (normal and
    # subnormal, both signs, odd and even lower neighbours): the ties.
    b = np.concatenate([rng.integers(0x0001, 0x7F7F, 2000), np.arange(0x0000, 0x0100)])
    lo = F.decode_bf16(b.astype(np.uint16))
    hi = F.decode_bf16((b + 1).astype(np.uint16))
    ties = (lo + hi) / 2
    x = np.concatenate([x, ties, -ties])
    vec = F.decode_bf16(F.encode_bf16_rne(x))
    sca = np.array([L._rne_bf16_scalar(float(v)) for v in x])
    assert np.array_equal(vec, sca)


def _bits(values):
    return F.encode_bf16_rne(np.asarray(values, dtype=np.float64))


def test_layer_bf16_matches_element_by_element_tier():
    rng = np.random.default_rng(3)
    T, H, I, E, k = 3, 128, 64, 3, 2
    x = _bits(rng.standard_normal((T, H)))
    w1 = _bits(rng.standard_normal((E, 2 * I, H)) * 0.05)
    w2 = _bits(rng.standard_normal((E, H, I)) * 0.05)
    idx = np.array([[0, 2], [2, -1], [1, 0]])
    tw = rng.uniform(0.1, 1.0, (T, k))
    for kw in ({}, {"alpha": 1.702, "up_bias": 1.0, "limit": 7.0}):
        a = L.layer_bf16(x, idx, tw, w1, w2, **kw)
        b = L.layer_bf16_bruteforce(x, idx, tw, w1, w2, **kw)
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_layer_bf16_gemm_is_integer_exact():
    """Codes with small power-of-two values make every product and sum exact:
    FC1 equals an int64 matmul of the scaled integers."""
    rng = np.random.default_rng(9)
    T, H, I, E, k = 4, 256, 128, 2, 1
    xi = rng.integers(-4, 5, (T, H))
    wi = rng.integers(-4, 5, (E, 2 * I, H))
    x = _bits(xi * 0.25)
    w1 = _bits(wi * 0.5)
    w2 = _bits(np.zeros((E, H, I)))
    idx = rng.integers(0, E, (T, k))
    _, inter = L.layer_bf16(x, idx, np.ones((T, k)), w1, w2, keep=True)
    for e, h in inter["h"].items():
        tokens = inter["perm"][inter["offsets"][e]:inter["offsets"][e + 1]] // k
        exact = (xi[tokens] @ wi[e].T) * 0.125
        assert np.array_equal(h, exact.astype(np.float64))


def test_activation_is_rounded_to_bf16_before_fc2():
    """One token, one expert, checked by hand: a = silu(g) * u is rounded to
    BF16 before it multiplies W2 (an identity row here)."""
    T, H, I, E, k = 1, 2, 1, 1, 1
    x = _bits([[1.0, 0.0]])
    g, u = 1.0, 1.0 + 2.0 ** -7 + 2.0 ** -9        # u itself rounds when stored
    w1 = _bits([[[g, 0.0], [u, 0.0]]])
    w2 = _bits([[[1.0], [0.0]]])
    out, inter = L.layer_bf16(x, np.array([[0]]), np.array([[1.0]]), w1, w2, keep=True)
    ue = F.decode_bf16(w1[0, 1, 0])                 # u as stored in BF16
    a = 1.0 / (1.0 + math.exp(-1.0)) * ue
    assert out[0, 0] == L._rne_bf16_scalar(a)
    assert out[0, 1] == 0.0
