"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare."""
import numpy as np
import torch

import moe_expert_ffn_permute_b200 as moe
from moe_expert_ffn_permute_b200.build import build
from workloads.synth import Workload, make_inputs, to_numpy
from oracle import layer as L

CALC_DIFF_MAX = 1e-4       # DeepGEMM-style calc_diff bound
REL_ERR_MAX = 2e-2         # per-element |err| <= 2e-2 * max|ref|


def ensure_built():
    build()
    moe.lib()


def calc_diff(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = (x * x + y * y).sum()
    if den == 0:
        return 0.0
    return 1.0 - 2.0 * (x * y).sum() / den


def assert_parity(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    d = calc_diff(gpu, ref)
    err = np.abs(gpu - ref).max()
    scale = np.abs(ref).max()
    assert d <= CALC_DIFF_MAX, f"{what}: calc_diff {d:.3e} > {CALC_DIFF_MAX}"
    assert err <= REL_ERR_MAX * scale, f"{what}: max|err| {err:.3e} > {REL_ERR_MAX}*{scale:.3e}"
    return d, err / max(scale, 1e-300)


def layer_for(wl, debug=False):
    return moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                        alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, debug=debug)


def run_gpu(wl, d, debug=False):
    lay = layer_for(wl, debug)
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                      d["w1_scales"], d["w2"], d["w2_scales"])
    torch.cuda.synchronize()
    return out, lay


def oracle_args(dn):
    return (dn["x"], dn["x_scales"], dn["topk_idx"], dn["topk_w"], dn["w1"], dn["w1_scales"],
            dn["w2"], dn["w2_scales"])


def oracle_kw(wl):
    return dict(w_dtype=wl.w_dtype, alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit)


def oracle_layer(wl, dn, keep=False):
    """The oracle for the workload's weight format (numpy inputs)."""
    if wl.w_dtype == "bf16":
        return L.layer_bf16(dn["x"], dn["topk_idx"], dn["topk_w"], dn["w1"], dn["w2"],
                            alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, keep=keep)
    return L.layer(*oracle_args(dn), **oracle_kw(wl), keep=keep)


def oracle_tokens(wl, dn, tokens, keep=False):
    """Oracle output for a subset of tokens (rows of the full-layer output:
    every token's output depends only on its own inputs)."""
    sub = dict(dn)
    for key in ("x", "x_scales", "topk_idx", "topk_w"):
        if dn[key] is not None:
            sub[key] = dn[key][tokens]
    return oracle_layer(wl, sub, keep=keep)


def inputs(wl, device="cuda", seed=None):
    return make_inputs(wl, device=device, seed=seed)


def bench_layer(wl, d, swap=None):
    """The layer in the launch configuration bench.py times: FP8 / BF16 weights
    prepacked into tiles, MXFP4 codes into tiles and scales into chunks, automatic tile
    orientation (unless `swap` forces one).  Returns (layer, weights dict)."""
    tiled = True                     # FP8 / BF16 tiles, MXFP4 code tiles
    chunked = wl.w_dtype == "e2m1"
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                       alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit,
                       tiled_weights=tiled, chunked_scales=chunked, swap_ab=swap)
    w = {k: d[k] for k in ("w1", "w1_scales", "w2", "w2_scales")}
    if tiled:
        w["w1"], w["w2"] = lay.prepack(d["w1"], d["w2"])
    if chunked:
        w["w1_scales"], w["w2_scales"] = lay.prepack_scales(d["w1_scales"], d["w2_scales"])
    return lay, w


def bench_forward(lay, w, d, out=None):
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], w["w1"],
                      w["w1_scales"], w["w2"], w["w2_scales"], out=out)
    torch.cuda.synchronize()
    return out
