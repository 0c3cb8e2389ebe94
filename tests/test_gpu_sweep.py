"""Whole-layer parity across the MXFP4 token sweep (T = 128 ... 32768, H=7168,
I=3072, E=48, top-6) and the other full-size workloads, in the launch
configuration the benchmark times (prepacked weights or scale chunks,
automatic tile orientation); bitwise determinism at the token counts whose
digests the pages compare (832, 1792, 8192, 32768) and across masked /
unmasked runs; and the layer's degenerate cases: every slot masked, and the
largest expert count a plan accepts (E = 256)."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from oracle import layer as L
from workloads.synth import MXFP4_TOKEN_SWEEP, WORKLOADS, Workload, to_numpy

from gpu_helpers import (assert_parity, bench_forward, bench_layer, ensure_built, inputs,
                         oracle_args, oracle_kw, oracle_tokens)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _sampled_parity(wl, ntok, seed):
    d = inputs(wl)
    lay, w = bench_layer(wl, d)
    out = bench_forward(lay, w, d)
    assert lay.check() == 0
    rnd = np.random.default_rng(seed).choice(wl.T, size=min(ntok, wl.T), replace=False)
    tokens = np.array(sorted(set(rnd.tolist()) | {0, wl.T - 1}))
    ref = oracle_tokens(wl, to_numpy(d), tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, wl.name)


@pytest.mark.parametrize("T", MXFP4_TOKEN_SWEEP)
def test_mxfp4_token_sweep_sampled_parity(T):
    """Every token count of the MXFP4 sweep; the sampled tokens include the
    first and the last token (a ragged last tile of some expert)."""
    wl = WORKLOADS["mxfp4"].with_tokens(T)
    _sampled_parity(wl, 4, T)


@pytest.mark.parametrize("name", ["decode", "prefill", "oai", "bf16"])
def test_other_workloads_bench_configuration_sampled_parity(name):
    _sampled_parity(WORKLOADS[name], 6, 11)


@pytest.mark.parametrize("T", [832, 1792, 8192, 32768])
def test_bitwise_repeatable_at_digest_token_counts(T):
    """Two runs of the layer (separate plans and workspaces) give the same
    bytes at the token counts the pages' digest checks use."""
    wl = WORKLOADS["mxfp4"].with_tokens(T)
    d = inputs(wl)
    lay, w = bench_layer(wl, d)
    a = bench_forward(lay, w, d).clone()
    del lay
    lay2, w2 = bench_layer(wl, d)
    b = bench_forward(lay2, w2, d)
    assert lay2.check() == 0
    assert torch.equal(a, b)


@pytest.mark.parametrize("swap", [1, 2], ids=["token-rows", "token-major"])
@pytest.mark.parametrize("T", [832, 8192])
def test_masked_unmasked_pairs_bitwise(T, swap):
    """A run in which a quarter of the slots are masked (-1) gives, for every
    token none of whose slots is masked, the same bytes as the unmasked run
    (with a fixed tile orientation: which tiles the other tokens form does not
    change a token's result)."""
    wl = WORKLOADS["mxfp4"].with_tokens(T)
    d = inputs(wl)
    lay, w = bench_layer(wl, d, swap=swap)
    full = bench_forward(lay, w, d).clone()
    g = torch.Generator(device="cuda").manual_seed(T)
    mask = torch.rand(wl.T, wl.k, generator=g, device="cuda") < 0.25
    dm = dict(d)
    dm["topk_idx"] = torch.where(mask, torch.full_like(d["topk_idx"], -1), d["topk_idx"])
    masked = bench_forward(lay, w, dm)
    assert lay.check() == 0
    keep = ~mask.any(dim=1)
    assert int(keep.sum()) > 0
    assert torch.equal(masked[keep], full[keep])


@pytest.mark.parametrize("T,k", [(300, 4), (2048, 4)], ids=["fused-front", "separate-front"])
def test_every_slot_masked(T, k):
    """All slots masked: no GEMM tile exists, the output is all zeros, no
    device error is recorded, and the step calls give the same bytes."""
    wl = Workload("all-masked", T, 1024, 512, 8, k, cfg_id=40)
    d = inputs(wl)
    d["topk_idx"].fill_(-1)
    lay, w = bench_layer(wl, d)
    out = torch.full((wl.T, wl.H), 3.0, dtype=torch.bfloat16, device="cuda")
    bench_forward(lay, w, d, out=out)
    assert lay.check() == 0
    assert not out.any()
    sep = torch.full_like(out, 5.0)
    moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
    moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
    moe.moe_fc1(lay.plan, w["w1"], w["w1_scales"], lay.workspace)
    moe.moe_fc2(lay.plan, w["w2"], w["w2_scales"], lay.workspace)
    moe.moe_combine(lay.plan, d["topk_w"], sep, lay.workspace)
    torch.cuda.synchronize()
    assert torch.equal(sep, out)
    counts = lay.workspace[lay.view().counts - lay.workspace.data_ptr():][:4 * wl.E]
    assert not counts.view(torch.int32).any()


@pytest.mark.parametrize("w_dtype", ["e4m3", "e2m1"])
@pytest.mark.parametrize("T", [300, 700], ids=["fused-front", "separate-front"])
def test_largest_expert_count(T, w_dtype):
    """E = 256 experts, top-8: most experts get a handful of tokens (ragged
    tiles everywhere); whole-layer parity with the oracle."""
    wl = Workload("e256", T, 512, 256, 256, 8, w_dtype=w_dtype, cfg_id=41)
    d = inputs(wl)
    lay, w = bench_layer(wl, d)
    out = bench_forward(lay, w, d)
    assert lay.check() == 0
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, wl.name)
