"""Pins for the oracle's routing, activation, requantisation, GEMMs and layer.

None of these re-runs the oracle's own formula: routing is checked against a
sort-based brute force and invariants, the activation against torch's SiLU and
closed forms, the requant against exact power-of-two boundary cases, the GEMMs
against integer arithmetic, and the layer against the element-by-element
brute-force tier on tiny shapes plus per-token independence.
"""
import math

import numpy as np
import pytest
import torch

from oracle import layer as L
from oracle.formats import decode_e4m3, encode_e4m3_rne_satfinite
from workloads.synth import Workload, make_inputs, to_numpy


# ------------------------------------------------------------------ routing
def _route_by_sort(flat, E):
    pairs = sorted((int(e), s) for s, e in enumerate(flat) if 0 <= e < E)
    return [s for _, s in pairs]


@pytest.mark.parametrize("T,k,E,kind", [(1, 1, 1, "u"), (7, 3, 5, "u"), (64, 8, 32, "zipf"),
                                        (50, 4, 64, "one"), (33, 2, 16, "bad")])
def test_route_matches_sort_and_invariants(T, k, E, kind):
    rng = np.random.default_rng(T * 100 + E)
    if kind == "u":
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    elif kind == "zipf":
        p = np.arange(1, E + 1) ** -1.2
        p[-E // 8:] = 0
        idx = np.stack([rng.choice(E, k, replace=False, p=p / p.sum()) for _ in range(T)])
    elif kind == "one":
        idx = np.full((T, k), 3)
    else:
        idx = rng.integers(-2, E + 2, size=(T, k))
    counts, offsets, perm, inv = L.route(idx, E)
    flat = idx.reshape(-1)
    ref = _route_by_sort(flat, E)
    nvalid = len(ref)
    np.testing.assert_array_equal(perm[:nvalid], ref)
    assert (perm[nvalid:] == -1).all()
    assert counts.sum() == nvalid == offsets[-1]
    if kind != "bad":
        assert nvalid == T * k
    # bijection between valid slots and positions
    for p in range(nvalid):
        assert inv[perm[p]] == p
    assert ((inv == -1) == ((flat < 0) | (flat >= E))).all()
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()


# --------------------------------------------------------------- activation
def test_swiglu_identity_reduces_to_silu_times_up():
    rng = np.random.default_rng(1)
    g, u = rng.standard_normal(1000) * 8, rng.standard_normal(1000) * 8
    silu = torch.nn.functional.silu(torch.from_numpy(g)).numpy()
    # equal up to the rounding order of the two sigmoid formulations
    np.testing.assert_allclose(L.swiglu(g, u, 1.0, 0.0, math.inf), silu * u, rtol=1e-14, atol=0)


def test_swiglu_clamp_closed_forms():
    lim, al, be = 7.0, 1.702, 1.0
    s = 1.0 / (1.0 + math.exp(-al * lim))
    # gate above limit -> gate = limit; up beyond +-limit -> +-limit; bias after clamp
    got = L.swiglu(np.array([9.0, 9.0, 100.0, -3.0]), np.array([20.0, -20.0, 0.5, 7.0]), al, be, lim)
    sm3 = 1.0 / (1.0 + math.exp(-al * -3.0))
    want = [7.0 * s * 8.0, 7.0 * s * -6.0, 7.0 * s * 1.5, -3.0 * sm3 * 8.0]
    np.testing.assert_allclose(got, want, rtol=1e-15)
    # the gate is only clamped from above: very negative gates pass unclamped
    assert L.swiglu(np.array([-50.0]), np.array([1.0]), 1.0, 0.0, 7.0)[0] == pytest.approx(
        -50.0 / (1.0 + math.exp(50.0)) * 1.0, rel=1e-15)


# ------------------------------------------------------------------ requant
@pytest.mark.parametrize("n", [-20, -3, 0, 1, 5])
def test_requant_scale_power_of_two_boundaries(n):
    blk = np.zeros((3, 128))
    top = 448.0 * 2.0 ** n
    blk[0, 5] = top                         # exactly 448*2^n -> exponent n
    blk[1, 7] = -np.nextafter(top, np.inf)  # one ulp above -> n+1
    blk[2, 9] = np.nextafter(448.0 * 2.0 ** (n - 1), np.inf)   # just above half -> n
    codes, sf = L.requant_1x128(blk)
    assert list(sf[:, 0].astype(int) - 127) == [n, n + 1, n]
    assert codes[0, 5] == 0x7E and codes[1, 7] == 0xF6   # 448 = S.1111.110; -224 = 1.1110.110
    assert decode_e4m3(np.array([codes[1, 7]], dtype=np.uint8))[0] == -224.0


def test_requant_zero_block_and_floor():
    codes, sf = L.requant_1x128(np.zeros((1, 256)))
    assert (codes == 0).all()
    # floor 1e-4: smallest n with 1e-4 <= 448 * 2^n is -22
    assert (sf.astype(int) - 127 == -22).all() and 1e-4 <= 448 * 2.0 ** -22 and 1e-4 > 448 * 2.0 ** -23


def test_requant_reconstructs_within_half_ulp():
    rng = np.random.default_rng(3)
    a = rng.standard_normal((4, 384)) * 3
    codes, sf = L.requant_1x128(a)
    deq = decode_e4m3(codes) * np.repeat(2.0 ** (sf.astype(float) - 127), 128, axis=1)
    # E4M3 has 3 mantissa bits: relative error <= 2^-4 for normals; subnormal abs err
    # <= 2^-10 * scale
    scale = np.repeat(2.0 ** (sf.astype(float) - 127), 128, axis=1)
    assert (np.abs(deq - a) <= np.maximum(np.abs(a) * 2.0 ** -4, 2.0 ** -10 * scale)).all()


# -------------------------------------------------------------------- GEMMs
def test_dequant_gemm_integer_exact_with_block_scales():
    """Codes in {+-1, +-0.5} with distinct power-of-two scales: the f64 product
    equals a blockwise integer sum computed with int64 arithmetic."""
    rng = np.random.default_rng(5)
    R, C = 256, 384
    cx = rng.choice([0x38, 0xB8, 0x30, 0xB0], size=(4, C)).astype(np.uint8)   # 1,-1,.5,-.5
    cw = rng.choice([0x38, 0xB8, 0x30, 0xB0], size=(R, C)).astype(np.uint8)
    sx = rng.integers(120, 134, size=(4, C // 128)).astype(np.uint8)
    sw = rng.integers(120, 134, size=(R // 128, C // 128)).astype(np.uint8)
    got = L.dequant_act(cx, sx) @ L.dequant_w_fp8(cw, sw).T
    ix = (decode_e4m3(cx) * 2).astype(np.int64)     # exact integers
    iw = (decode_e4m3(cw) * 2).astype(np.int64)
    want = np.zeros((4, R))
    for kb in range(C // 128):
        part = ix[:, kb * 128:(kb + 1) * 128] @ iw[:, kb * 128:(kb + 1) * 128].T
        for r in range(R):
            want[:, r] += part[:, r] * 2.0 ** (sx[:, kb].astype(float) - 127
                                              + float(sw[r // 128, kb]) - 127 - 2)
    np.testing.assert_array_equal(got, want)


def test_dequant_fp4_scale_per_1x32():
    packed = np.full((2, 64), 0x22, dtype=np.uint8)         # every element = 1.0
    sc = np.array([[127, 128, 126, 130], [127] * 4], dtype=np.uint8)
    w = L.dequant_w_fp4(packed, sc)
    assert w.shape == (2, 128)
    np.testing.assert_array_equal(w[0], np.repeat([1.0, 2.0, 0.5, 8.0], 32))


# -------------------------------------------------------------------- layer
def _tiny(w_dtype="e4m3", act="swiglu", T=4, H=256, I=256, E=3, k=2, seed=0):
    kw = dict(alpha=1.702, up_bias=1.0, limit=7.0) if act == "swiglu_oai" else {}
    wl = Workload("t", T, H, I, E, k, w_dtype=w_dtype, act=act, cfg_id=90 + seed, **kw)
    return wl, to_numpy(make_inputs(wl, seed=seed))


def _args(d, wl):
    return (d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"], d["w1_scales"],
            d["w2"], d["w2_scales"])


@pytest.mark.parametrize("w_dtype,act", [("e4m3", "swiglu"), ("e4m3", "swiglu_oai"),
                                         ("e2m1", "swiglu")])
def test_layer_matches_bruteforce_tier(w_dtype, act):
    wl, d = _tiny(w_dtype, act, T=3, H=128 if w_dtype == "e4m3" else 128, I=128)
    kw = dict(w_dtype=w_dtype, alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit)
    fast = L.layer(*_args(d, wl), **kw)
    slow = L.layer_bruteforce(*_args(d, wl), **kw)
    np.testing.assert_allclose(fast, slow, rtol=1e-9, atol=1e-12 * np.abs(slow).max())


def test_layer_per_token_independence():
    wl, d = _tiny(T=9, H=256, I=256, E=4, k=2, seed=2)
    full = L.layer(*_args(d, wl))
    sub = [1, 4, 8]
    ds = dict(d)
    for key in ("x", "x_scales", "topk_idx", "topk_w"):
        ds[key] = d[key][sub]
    part = L.layer(*_args(ds, wl))
    np.testing.assert_array_equal(part, full[sub])


def test_layer_single_expert_hand_example():
    """T=1, k=1, H=I=128: x = 1 everywhere, gate rows all 0.5/128, up rows 1;
    so g = 0.5, u = 128, a = 0.5*sigmoid(0.5)*128 for every column; with W2 = 1
    every output column is 128 * a_q, a_q the E4M3 rounding of a at the chosen
    scale; the weight 0.75 multiplies the result."""
    H = I = 128
    x = np.full((1, H), 0x38, np.uint8)                    # 1.0
    xs = np.full((1, 1), 127, np.uint8)
    w1 = np.zeros((1, 2 * I, H), np.uint8)
    w1[0, :I] = 0x38                                       # 1.0 * 2^-8 via scale
    w1[0, I:] = 0x38
    w1s = np.array([[[127 - 8], [127]]], np.uint8)         # gate block scale 2^-8
    w2 = np.full((1, H, I), 0x38, np.uint8)
    w2s = np.full((1, 1, 1), 127, np.uint8)
    out = L.layer(x, xs, np.zeros((1, 1), np.int32), np.array([[0.75]]), w1, w1s, w2, w2s)
    g, u = 128 * 2.0 ** -8, 128.0
    a = g / (1 + math.exp(-g)) * u
    n = math.ceil(math.log2(a / 448))                      # a ~ 39.9 -> n = -3
    aq = decode_e4m3(encode_e4m3_rne_satfinite(np.array([a / 2 ** n])))[0] * 2 ** n
    np.testing.assert_array_equal(out, np.full((1, H), 0.75 * 128 * aq))
    assert n == -3 and abs(aq - a) < 1.0


def test_layer_two_slot_combine_hand_example():
    """T=2, E=3, k=2, H=I=128, x = 1: expert e has gate codes 1.0 at block scale
    2^(e-8) (so g_e = 2^(e-1)), up codes 1.0 (u = 128) and W2 = 1, so each
    expert's output column is 128 * q(a_e) with a_e = g_e * sigmoid(g_e) * 128.
    Token 0 goes to experts (2, 0) with weights (0.25, 0.75), token 1 to (1, 2)
    with (0.5, 0.5): the combine must pair each slot's weight with its own
    expert's rows, in token order."""
    H = I = 128
    E = 3
    x = np.full((2, H), 0x38, np.uint8)
    xs = np.full((2, 1), 127, np.uint8)
    w1 = np.full((E, 2 * I, H), 0x38, np.uint8)
    w1s = np.array([[[127 - 8 + e], [127]] for e in range(E)], np.uint8)
    w2 = np.full((E, H, I), 0x38, np.uint8)
    w2s = np.full((E, 1, 1), 127, np.uint8)
    idx = np.array([[2, 0], [1, 2]], np.int32)
    w = np.array([[0.25, 0.75], [0.5, 0.5]])
    out = L.layer(x, xs, idx, w, w1, w1s, w2, w2s)

    def y(e):
        g = 2.0 ** (e - 1)
        a = g / (1 + math.exp(-g)) * 128
        n = math.ceil(math.log2(a / 448))
        return 128 * decode_e4m3(encode_e4m3_rne_satfinite(np.array([a / 2 ** n])))[0] * 2 ** n

    expect = np.array([[0.25 * y(2) + 0.75 * y(0)] * H, [0.5 * y(1) + 0.5 * y(2)] * H])
    np.testing.assert_allclose(out, expect, rtol=1e-15)
    assert len({y(0), y(1), y(2)}) == 3


def test_bruteforce_e4m3_rounding_agrees_with_the_encoder_on_ties():
    """The brute-force tier's scalar E4M3 rounding (a scan of every code) against
    the vectorised encoder on every midpoint between consecutive finite E4M3
    values, both signs, the values themselves and out-of-range magnitudes."""
    mags = decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = (mags[:-1] + mags[1:]) / 2
    vals = np.concatenate([mids, -mids, mags, -mags, [449.0, 464.0, 1e6, -500.0]])
    vec = decode_e4m3(encode_e4m3_rne_satfinite(vals))
    sca = np.array([L._rne_e4m3_scalar(float(v)) for v in vals])
    np.testing.assert_array_equal(sca, vec)
