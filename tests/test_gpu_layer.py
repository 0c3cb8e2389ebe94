"""Whole-layer parity of the CUDA path (through the C ABI) against the oracle,
plus the FC1 epilogue's requantisation checked byte for byte."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from workloads.synth import WORKLOADS, Workload, make_activations, to_numpy
from oracle import layer as L

from gpu_helpers import (assert_parity, ensure_built, inputs, layer_for, oracle_args,
                         oracle_kw, oracle_tokens, run_gpu)

pytestmark = pytest.mark.gpu

RAGGED = Workload("ragged", 300, 1024, 512, 8, 4, cfg_id=20)
RAGGED_FP4 = Workload("ragged-fp4", 300, 1024, 512, 8, 4, w_dtype="e2m1", cfg_id=21)
RAGGED_OAI = Workload("ragged-oai", 200, 512, 384, 6, 3, act="swiglu_oai", alpha=1.702,
                      up_bias=1.0, limit=7.0, cfg_id=22)
SINGLE = Workload("single", 1, 512, 128, 1, 1, cfg_id=23)


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _ws_bytes(lay, ptr, nbytes):
    off = ptr - lay.workspace.data_ptr()
    return lay.workspace[off:off + nbytes]


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"], RAGGED, RAGGED_FP4, RAGGED_OAI, SINGLE],
                         ids=lambda w: w.name)
def test_layer_parity_small(wl):
    d = inputs(wl)
    out, lay = run_gpu(wl, d)
    assert lay.check() == 0
    dn = to_numpy(d)
    ref = L.layer(*oracle_args(dn), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, wl.name)


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"], RAGGED, RAGGED_FP4, RAGGED_OAI],
                         ids=lambda w: w.name)
def test_fc1_requant_bytes_exact_and_activation_close(wl):
    """The FP8 codes and UE8M0 bytes the FC1 epilogue writes equal the oracle's
    quantiser applied to the epilogue's own fp32 activation; that activation
    agrees with the oracle's float64 one."""
    d = inputs(wl)
    out, lay = run_gpu(wl, d, debug=True)
    v = lay.view()
    rows = v.rows
    act_t = torch.empty(rows, wl.I, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act(lay.plan, lay.workspace, act_t)
    act = act_t.cpu().numpy()
    a32 = _ws_bytes(lay, v.act_f32, rows * wl.I * 4).view(torch.float32).view(rows, wl.I)
    a32 = a32.cpu().numpy()
    sf = torch.empty(rows, wl.I // 128, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act_scales(lay.plan, lay.workspace, sf)
    sf = sf.cpu().numpy()
    pad = _ws_bytes(lay, v.pad_offsets, 4 * (wl.E + 1)).view(torch.int32).cpu().numpy()
    dn = to_numpy(d)
    _, inter = L.layer(*oracle_args(dn), **oracle_kw(wl), keep=True)
    for e, a_ref in inter["a"].items():
        n = a_ref.shape[0]
        rows_e = slice(pad[e], pad[e] + n)
        q_ref, s_ref = L.requant_1x128(a32[rows_e].astype(np.float64))
        np.testing.assert_array_equal(act[rows_e], q_ref, err_msg=f"codes, expert {e}")
        np.testing.assert_array_equal(sf[rows_e], s_ref, err_msg=f"scales, expert {e}")
        assert_parity(a32[rows_e], a_ref, f"activation expert {e}")


def test_layer_is_bitwise_repeatable():
    wl = RAGGED
    d = inputs(wl)
    a, _ = run_gpu(wl, d)
    b, _ = run_gpu(wl, d)
    assert torch.equal(a, b)


def test_out_of_range_ids_contribute_nothing():
    wl = RAGGED
    d = inputs(wl)
    d["topk_idx"][5, 2] = -3
    d["topk_idx"][100, 0] = wl.E + 7
    out, lay = run_gpu(wl, d)
    assert lay.check() == 6
    dn = to_numpy(d)
    ref = L.layer(*oracle_args(dn), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, "bad ids")


def test_masked_slots_contribute_nothing_and_are_not_errors():
    wl = RAGGED
    d = inputs(wl)
    mask = torch.rand(wl.T, wl.k, device="cuda") < 0.25
    d["topk_idx"][mask] = -1
    out, lay = run_gpu(wl, d)
    assert lay.check() == 0
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, "masked")


def test_step_calls_equal_forward():
    wl = RAGGED_OAI
    d = inputs(wl)
    full, lay = run_gpu(wl, d)
    out = torch.empty_like(full)
    moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
    moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
    moe.moe_fc1(lay.plan, d["w1"], d["w1_scales"], lay.workspace)
    moe.moe_fc2(lay.plan, d["w2"], d["w2_scales"], lay.workspace)
    moe.moe_combine(lay.plan, d["topk_w"], out, lay.workspace)
    torch.cuda.synchronize()
    assert torch.equal(out, full)


def test_fused_gemm_step_equals_separate_gemms():
    """FC1 and FC2 in one persistent launch (dynamic scheduler, per-m-tile
    dependency counters) give the same bytes as two separate launches."""
    for wl in (RAGGED, RAGGED_FP4):
        d = inputs(wl)
        _, lay = run_gpu(wl, d)
        v = lay.view()
        n = wl.T * wl.k * wl.H * 2
        off = v.y - lay.workspace.data_ptr()
        moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
        moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
        moe.moe_fc1(lay.plan, d["w1"], d["w1_scales"], lay.workspace)
        moe.moe_fc2(lay.plan, d["w2"], d["w2_scales"], lay.workspace)
        torch.cuda.synchronize()
        y_sep = lay.workspace[off:off + n].clone()
        lay.workspace[off:off + n].zero_()
        moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
        moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
        moe.moe_fc1_fc2(lay.plan, d["w1"], d["w1_scales"], d["w2"], d["w2_scales"],
                        lay.workspace)
        torch.cuda.synchronize()
        assert torch.equal(lay.workspace[off:off + n], y_sep), wl.name


def test_hostio_equals_device_forward():
    wl = RAGGED
    d = inputs(wl)
    full, lay = run_gpu(wl, d)
    host = {k: v.cpu().pin_memory() for k, v in d.items() if k in ("x", "x_scales", "topk_idx",
                                                                   "topk_w")}
    out_h = torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_hostio(lay.plan, host["x"], host["x_scales"], host["topk_idx"],
                           host["topk_w"], d["w1"], d["w1_scales"], d["w2"], d["w2_scales"],
                           out_h, lay.workspace)
    torch.cuda.synchronize()
    assert torch.equal(out_h, full.cpu())


@pytest.mark.parametrize("name,T,ntok", [("decode", None, 48), ("prefill", None, 12),
                                         ("oai", None, 64), ("mxfp4", 128, 12),
                                         ("mxfp4", 8192, 6)])
def test_layer_parity_full_size_sampled(name, T, ntok):
    """Full-size workloads in the launch configuration the bench uses; the
    oracle computes a seeded sample of tokens (each token's output depends only
    on its own inputs)."""
    wl = WORKLOADS[name] if T is None else WORKLOADS[name].with_tokens(T)
    d = inputs(wl)
    out, lay = run_gpu(wl, d)
    assert lay.check() == 0
    rng = np.random.default_rng(wl.T)
    tokens = np.sort(rng.choice(wl.T, size=min(ntok, wl.T), replace=False))
    dn = {k: v.cpu().numpy() for k, v in d.items()}
    ref = oracle_tokens(wl, dn, tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, wl.name)


def test_cuda_graph_replay_is_bitwise_identical():
    """moe_forward captured once in a CUDA graph and replayed: every replay
    recomputes routing and resets the GEMM scheduler's counters in-graph, so
    each replay equals the eager result bit for bit (also after the inputs'
    routing changes in place between replays)."""
    wl = RAGGED
    d = inputs(wl)
    eager, lay = run_gpu(wl, d)
    out = torch.empty_like(eager)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_forward(lay.plan, d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                        d["w1_scales"], d["w2"], d["w2_scales"], out, lay.workspace,
                        torch.cuda.current_stream())
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    # new routing in the same buffers: the replay follows it
    d2 = inputs(wl, seed=777)
    d["topk_idx"].copy_(d2["topk_idx"])
    d["topk_w"].copy_(d2["topk_w"])
    g.replay()
    torch.cuda.synchronize()
    ref2, _ = run_gpu(wl, d)
    assert torch.equal(out, ref2)


def _run_tiled(wl, d):
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                       alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, tiled_weights=True)
    w1t, w2t = lay.prepack(d["w1"], d["w2"])
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], w1t, d["w1_scales"],
                      w2t, d["w2_scales"])
    torch.cuda.synchronize()
    return out, lay


def _tiles_reference(w, K):
    """Tiled layout written out from its definition (torch indexing)."""
    rows = w.numel() // K
    m = w.reshape(rows, K).view(rows // 128, 128, K // 128, 8, 16)   # [rb, r, kb, c16, byte]
    r = torch.arange(128, device=w.device).view(128, 1)
    c16 = torch.arange(8, device=w.device).view(1, 8)
    dest_c16 = (c16 ^ (r % 8))                                        # [r, c16]
    out = torch.empty(rows // 128, K // 128, 128, 8, 16, dtype=torch.uint8, device=w.device)
    src = m.permute(0, 2, 1, 3, 4)                                    # [rb, kb, r, c16, byte]
    idx = dest_c16.view(1, 1, 128, 8, 1).expand_as(src)
    out.scatter_(3, idx, src)
    return out.reshape(-1)


def test_prepack_matches_layout_definition():
    wl = RAGGED
    d = inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, tiled_weights=True)
    w1t, w2t = lay.prepack(d["w1"], d["w2"])
    torch.cuda.synchronize()
    assert torch.equal(w1t.reshape(-1), _tiles_reference(d["w1"], wl.H))
    assert torch.equal(w2t.reshape(-1), _tiles_reference(d["w2"], wl.I))


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"], RAGGED, RAGGED_OAI], ids=lambda w: w.name)
def test_tiled_weights_bitwise_equal_row_major(wl):
    d = inputs(wl)
    ref, _ = run_gpu(wl, d)
    out, lay = _run_tiled(wl, d)
    assert lay.check() == 0
    assert torch.equal(out, ref)


@pytest.mark.parametrize("name,ntok", [("decode", 32), ("prefill", 8)])
def test_tiled_weights_full_size_parity(name, ntok):
    wl = WORKLOADS[name]
    d = inputs(wl)
    out, lay = _run_tiled(wl, d)
    assert lay.check() == 0
    rng = np.random.default_rng(wl.T + 1)
    tokens = np.sort(rng.choice(wl.T, size=ntok, replace=False))
    dn = {k: v.cpu().numpy() for k, v in d.items()}
    ref = oracle_tokens(wl, dn, tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, wl.name + "-tiled")


def _run_mode(wl, d, pairs, debug=False):
    # The pair kernel computes token-row tiles; its single-CTA reference does too.
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                       alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, tiled_weights=True,
                       cta_pairs=pairs, swap_ab=1, debug=debug)
    w1t, w2t = lay.prepack(d["w1"], d["w2"])
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], w1t, d["w1_scales"],
                      w2t, d["w2_scales"])
    torch.cuda.synchronize()
    return out, lay


@pytest.mark.parametrize("wl", [WORKLOADS["tiny"], RAGGED, RAGGED_OAI, SINGLE],
                         ids=lambda w: w.name)
def test_cta_pair_gemm_bitwise_equal_single_cta(wl):
    """The 2-SM GEMM (CTA pairs, 256-row tiles) gives the same bytes as the
    single-CTA GEMM, including experts with an odd number of 128-row tiles
    (the pair's second CTA then has no rows)."""
    d = inputs(wl)
    ref, _ = _run_mode(wl, d, pairs=1)
    out, lay = _run_mode(wl, d, pairs=2)
    assert lay.check() == 0
    assert torch.equal(out, ref)


def test_cta_pair_gemm_requant_bytes_exact():
    wl = RAGGED
    d = inputs(wl)
    out, lay = _run_mode(wl, d, pairs=2, debug=True)
    v = lay.view()
    rows = v.rows
    act_t = torch.empty(rows, wl.I, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act(lay.plan, lay.workspace, act_t)
    a32 = _ws_bytes(lay, v.act_f32, rows * wl.I * 4).view(torch.float32).view(rows, wl.I)
    sf = torch.empty(rows, wl.I // 128, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act_scales(lay.plan, lay.workspace, sf)
    counts = _ws_bytes(lay, v.counts, 4 * wl.E).view(torch.int32).cpu().numpy()
    pad = _ws_bytes(lay, v.pad_offsets, 4 * (wl.E + 1)).view(torch.int32).cpu().numpy()
    act, a32, sf = act_t.cpu().numpy(), a32.cpu().numpy(), sf.cpu().numpy()
    for e in range(wl.E):
        r = slice(pad[e], pad[e] + counts[e])
        q_ref, s_ref = L.requant_1x128(a32[r].astype(np.float64))
        np.testing.assert_array_equal(act[r], q_ref)
        np.testing.assert_array_equal(sf[r], s_ref)


def test_cta_pair_gemm_full_size_prefill_parity():
    wl = WORKLOADS["prefill"]
    d = inputs(wl)
    out, lay = _run_mode(wl, d, pairs=2)
    assert moe.moe_plan_cta_pairs_active(lay.plan)
    assert lay.check() == 0
    rng = np.random.default_rng(5)
    tokens = np.sort(rng.choice(wl.T, size=8, replace=False))
    dn = {k: v.cpu().numpy() for k, v in d.items()}
    ref = oracle_tokens(wl, dn, tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, "prefill-pairs")


def _whole_workspace_after(lay, d, fused):
    """Fill the workspace with a fixed byte pattern, run the layer either as
    moe_forward (routing and gather fused at small slot counts) or as the
    separate step calls, and return the entire workspace."""
    lay.workspace.fill_(0x5A)
    moe.moe_clear_device_error(lay.plan, lay.workspace)
    out = torch.zeros(d["x"].shape[0], lay.H, dtype=torch.bfloat16, device="cuda")
    if fused == "forward":
        moe.moe_forward(lay.plan, d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                        d["w1_scales"], d["w2"], d["w2_scales"], out, lay.workspace)
    elif fused == "steps":
        moe.moe_route_gather(lay.plan, d["topk_idx"], d["x"], d["x_scales"], lay.workspace)
        moe.moe_fc1_fc2(lay.plan, d["w1"], d["w1_scales"], d["w2"], d["w2_scales"],
                        lay.workspace)
        moe.moe_combine(lay.plan, d["topk_w"], out, lay.workspace)
    else:
        moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
        moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
        moe.moe_fc1_fc2(lay.plan, d["w1"], d["w1_scales"], d["w2"], d["w2_scales"],
                        lay.workspace)
        moe.moe_combine(lay.plan, d["topk_w"], out, lay.workspace)
    torch.cuda.synchronize()
    return lay.workspace.clone(), out


@pytest.mark.parametrize("case", ["ragged", "masked", "bad-ids", "decode", "boundary-4096"])
def test_fused_route_gather_writes_the_same_bytes(case):
    """At slot counts up to 4096 moe_forward routes and gathers in one launch;
    every workspace byte (routing arrays, padding map, gathered tiles and
    scale chunks, GEMM counters, error word) and the output equal those of the
    separate launches."""
    if case == "decode":
        wl = WORKLOADS["decode"]
    elif case == "boundary-4096":
        wl = Workload("boundary", 512, 1024, 256, 16, 8, cfg_id=24)   # S = 4096
    else:
        wl = RAGGED
    d = inputs(wl)
    if case == "masked":
        d["topk_idx"][torch.rand(wl.T, wl.k, device="cuda") < 0.25] = -1
    if case == "bad-ids":
        d["topk_idx"][5, 2] = -3
        d["topk_idx"][100, 0] = wl.E + 7
    lay = layer_for(wl, False)
    assert moe.moe_forward_launch_count(lay.plan) == 3
    ws_sep, out_sep = _whole_workspace_after(lay, d, fused=None)
    for how in ("forward", "steps"):     # moe_forward, and moe_route_gather + later steps
        ws_fused, out_fused = _whole_workspace_after(lay, d, fused=how)
        assert torch.equal(out_fused, out_sep), how
        diff = (ws_fused != ws_sep).nonzero().flatten()
        if wl.T * wl.k > 2048:
            # The separate path then routes with two blocks whose histogram
            # scratch (between the padded offsets and perm) the fused launch
            # does not need: only bytes there may differ.
            base, v = lay.workspace.data_ptr(), lay.view()
            assert diff.numel() <= 2 * wl.E * 4, how
            if diff.numel():
                assert int(diff.min()) >= v.pad_offsets - base, how
                assert int(diff.max()) < v.perm - base, how
        else:
            assert diff.numel() == 0, how
        assert lay.check() == (6 if case == "bad-ids" else 0)



SWAP_CASES = [RAGGED, RAGGED_FP4, RAGGED_OAI, WORKLOADS["tiny"], SINGLE]


def _layer_swap(wl, swap, debug=False, tiled=False):
    return moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                        alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, debug=debug,
                        tiled_weights=tiled, swap_ab=swap)


@pytest.mark.parametrize("wl", SWAP_CASES, ids=lambda w: w.name)
def test_token_major_tiles_match_oracle(wl):
    """Swap-AB GEMM tiles (weights as A, tokens as B) forced on: parity with the
    oracle, including experts with more than 64 and more than 128 rows."""
    d = inputs(wl)
    lay = _layer_swap(wl, 2)
    assert moe.moe_plan_swap_ab_active(lay.plan) == 1
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                      d["w1_scales"], d["w2"], d["w2_scales"])
    torch.cuda.synchronize()
    assert lay.check() == 0
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, f"swap {wl.name}")


@pytest.mark.parametrize("wl", [RAGGED, RAGGED_FP4], ids=lambda w: w.name)
def test_token_major_requant_bytes_exact(wl):
    """With swap-AB tiles the FC1 epilogue reduces each token's amax across
    lanes; its FP8 codes and scales equal the oracle quantiser applied to the
    GPU's own fp32 activation, byte for byte."""
    d = inputs(wl)
    lay = _layer_swap(wl, 2, debug=True)
    lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"], d["w1_scales"],
                d["w2"], d["w2_scales"])
    torch.cuda.synchronize()
    v = lay.view()
    rows = v.rows
    act_t = torch.empty(rows, wl.I, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act(lay.plan, lay.workspace, act_t)
    a32 = _ws_bytes(lay, v.act_f32, rows * wl.I * 4).view(torch.float32).view(rows, wl.I)
    sf = torch.empty(rows, wl.I // 128, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act_scales(lay.plan, lay.workspace, sf)
    counts = _ws_bytes(lay, v.counts, 4 * wl.E).view(torch.int32).cpu().numpy()
    pad = _ws_bytes(lay, v.pad_offsets, 4 * (wl.E + 1)).view(torch.int32).cpu().numpy()
    act, a32, sf = act_t.cpu().numpy(), a32.cpu().numpy(), sf.cpu().numpy()
    for e in range(wl.E):
        r = slice(pad[e], pad[e] + counts[e])
        q_ref, s_ref = L.requant_1x128(a32[r].astype(np.float64))
        np.testing.assert_array_equal(act[r], q_ref, err_msg=f"codes, expert {e}")
        np.testing.assert_array_equal(sf[r], s_ref, err_msg=f"scales, expert {e}")


def test_token_major_fused_equals_separate_and_tiled_equals_row_major():
    wl = RAGGED
    d = inputs(wl)
    outs = []
    for tiled in (False, True):
        lay = _layer_swap(wl, 2, tiled=tiled)
        w1, w2 = lay.prepack(d["w1"], d["w2"]) if tiled else (d["w1"], d["w2"])
        outs.append(lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], w1,
                                d["w1_scales"], w2, d["w2_scales"]))
        torch.cuda.synchronize()
        if not tiled:
            v = lay.view()
            n = wl.T * wl.k * wl.H * 2
            off = v.y - lay.workspace.data_ptr()
            y_fused = lay.workspace[off:off + n].clone()
            moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
            moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
            moe.moe_fc1(lay.plan, w1, d["w1_scales"], lay.workspace)
            moe.moe_fc2(lay.plan, w2, d["w2_scales"], lay.workspace)
            torch.cuda.synchronize()
            assert torch.equal(lay.workspace[off:off + n], y_fused)
    assert torch.equal(outs[0], outs[1])


def test_token_major_decode_full_size():
    """The decode layer (T=128, E=32, k=8) in automatic mode: token-major tiles
    wherever an expert's tile holds at most 96 tokens."""
    wl = WORKLOADS["decode"]
    d = inputs(wl)
    lay = _layer_swap(wl, None, tiled=True)
    assert moe.moe_plan_swap_ab_active(lay.plan) == 2
    w1, w2 = lay.prepack(d["w1"], d["w2"])
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], w1, d["w1_scales"],
                      w2, d["w2_scales"])
    torch.cuda.synchronize()
    assert lay.check() == 0
    tokens = np.sort(np.random.default_rng(4).choice(wl.T, size=8, replace=False))
    ref = oracle_tokens(wl, to_numpy(d), tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, "decode swap")



@pytest.mark.parametrize("swap", [1, 2], ids=["token-rows", "swap-ab"])
def test_tokens_without_routed_slots_get_zero_rows(swap):
    """A token whose slots are all masked or invalid gets a zero row (no FC2
    row reaches it); moe_forward equals the step calls byte for byte and the
    oracle within tolerance, with either tile orientation."""
    wl = RAGGED
    d = inputs(wl)
    d["topk_idx"][3, :] = -1
    d["topk_idx"][10, :] = wl.E + 5
    d["topk_idx"][11, 1:] = -1
    lay = _layer_swap(wl, swap)
    out = torch.full((wl.T, wl.H), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(lay.plan, d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                    d["w1_scales"], d["w2"], d["w2_scales"], out, lay.workspace)
    torch.cuda.synchronize()
    assert lay.check() == 6
    assert not out[3].any() and not out[10].any()
    sep = torch.full_like(out, 7.0)
    moe.moe_route_gather(lay.plan, d["topk_idx"], d["x"], d["x_scales"], lay.workspace)
    moe.moe_fc1_fc2(lay.plan, d["w1"], d["w1_scales"], d["w2"], d["w2_scales"], lay.workspace)
    moe.moe_combine(lay.plan, d["topk_w"], sep, lay.workspace)
    torch.cuda.synchronize()
    assert torch.equal(out, sep)
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, "zero rows")


def test_fp4_scale_chunk_layout_matches_its_definition():
    """moe_prepack_weight_scales: chunk (b, kb) at (b * K/128 + kb) * 512 holds
    row r of block b's four k-block scale bytes at (r % 32) * 16 + (r / 32) * 4."""
    wl = RAGGED_FP4
    d = inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype="e2m1", chunked_scales=True)
    c1, c2 = lay.prepack_scales(d["w1_scales"], d["w2_scales"])
    torch.cuda.synchronize()
    for src, got, K in ((d["w1_scales"], c1, wl.H), (d["w2_scales"], c2, wl.I)):
        s = src.reshape(-1, K // 32).cpu().numpy()          # [rows, K/32]
        rows, kbn = s.shape[0], K // 128
        ref = np.zeros(rows * K // 32, dtype=np.uint8)
        for row in range(rows):
            b, r = divmod(row, 128)
            for kb in range(kbn):
                o = (b * kbn + kb) * 512 + (r % 32) * 16 + (r // 32) * 4
                ref[o:o + 4] = s[row, 4 * kb:4 * kb + 4]
        np.testing.assert_array_equal(got.reshape(-1).cpu().numpy(), ref)


@pytest.mark.parametrize("swap", [1, 2], ids=["token-rows", "swap-ab"])
def test_fp4_chunked_scales_and_tiled_codes_give_the_same_bytes(swap):
    """MXFP4 weights row-major, with chunked scales, and with tiled codes and
    chunked scales: the same output bytes in either tile orientation."""
    wl = RAGGED_FP4
    d = inputs(wl)
    outs = []
    for chunked, tiled in ((False, False), (True, False), (True, True)):
        lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype="e2m1", swap_ab=swap,
                           chunked_scales=chunked, tiled_weights=tiled)
        s1, s2 = (lay.prepack_scales(d["w1_scales"], d["w2_scales"]) if chunked
                  else (d["w1_scales"], d["w2_scales"]))
        w1, w2 = lay.prepack(d["w1"], d["w2"]) if tiled else (d["w1"], d["w2"])
        outs.append(lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], w1, s1, w2,
                                s2))
        torch.cuda.synchronize()
        assert lay.check() == 0
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[0], outs[2])


def test_fp4_code_tiles_match_their_definition():
    """moe_prepack_weights on MXFP4 codes: tile (b, kb) at (b * KB/64 + kb) * 8192
    holds bytes 64kb..64kb+63 of row 128b + r at r * 64 (KB = K/2 bytes a row)."""
    wl = RAGGED_FP4
    d = inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype="e2m1", chunked_scales=True,
                       tiled_weights=True)
    t1, t2 = lay.prepack(d["w1"], d["w2"])
    torch.cuda.synchronize()
    for src, got, K in ((d["w1"], t1, wl.H), (d["w2"], t2, wl.I)):
        kbytes = K // 2
        rows = src.numel() // kbytes
        ref = (src.reshape(rows // 128, 128, kbytes // 64, 64)   # [b, r, kb, byte]
               .permute(0, 2, 1, 3).contiguous().reshape(-1))
        assert torch.equal(got.reshape(-1), ref)


def test_fp4_chunked_scales_full_size_128_tokens():
    wl = WORKLOADS["mxfp4"]
    d = inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype="e2m1", chunked_scales=True)
    s1, s2 = lay.prepack_scales(d["w1_scales"], d["w2_scales"])
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"], s1, d["w2"], s2)
    torch.cuda.synchronize()
    assert lay.check() == 0
    tokens = np.sort(np.random.default_rng(6).choice(wl.T, size=6, replace=False))
    ref = oracle_tokens(wl, to_numpy(d), tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, "mxfp4 chunked scales")


def test_token_rows_are_independent_of_the_batch():
    """With token-row tiles a token's output does not depend on the other tokens
    of the batch: the layer on a subset of tokens gives those tokens' rows of
    the full run byte for byte."""
    wl = RAGGED
    d = inputs(wl)
    full = _layer_swap(wl, 1)
    out_full = full.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                            d["w1_scales"], d["w2"], d["w2_scales"])
    tokens = torch.arange(5, wl.T, 7, device="cuda")
    sub = Workload("ragged-subset", int(tokens.numel()), wl.H, wl.I, wl.E, wl.k, cfg_id=20)
    part = _layer_swap(sub, 1)
    out_part = part.forward(d["x"][tokens].contiguous(), d["x_scales"][tokens].contiguous(),
                            d["topk_idx"][tokens].contiguous(), d["topk_w"][tokens].contiguous(),
                            d["w1"], d["w1_scales"], d["w2"], d["w2_scales"])
    torch.cuda.synchronize()
    assert full.check() == 0 and part.check() == 0
    assert torch.equal(out_part, out_full[tokens])


@pytest.mark.parametrize("wl", [RAGGED, WORKLOADS["bf16"]], ids=lambda w: w.name)
def test_hostio_batches_equal_device_forwards(wl):
    """Three consecutive batches through the pipelined host-buffer entry (the
    copies of one batch overlap the neighbours' layers, two staging sets):
    every batch's output equals moe_forward on the same inputs, byte for byte,
    also when the call is repeated and when all batches share one output
    buffer (the last batch's output lands last)."""
    base = inputs(wl)
    batches = [make_activations(wl, device="cuda", seed=900 + i) for i in range(3)]
    lay = layer_for(wl)
    ref = []
    for d in batches:
        out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], base["w1"],
                          base["w1_scales"], base["w2"], base["w2_scales"])
        torch.cuda.synchronize()
        ref.append(out.cpu())
    keys = ("x", "x_scales", "topk_idx", "topk_w")
    host = [{k: (None if d[k] is None else d[k].cpu().pin_memory()) for k in keys}
            for d in batches]
    for repeat in range(2):
        outs = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory() for _ in batches]
        moe.moe_forward_hostio_batches(
            lay.plan, [h["x"] for h in host],
            None if host[0]["x_scales"] is None else [h["x_scales"] for h in host],
            [h["topk_idx"] for h in host], [h["topk_w"] for h in host], base["w1"],
            base["w1_scales"], base["w2"], base["w2_scales"], outs, lay.workspace)
        torch.cuda.current_stream().synchronize()
        for i in range(3):
            assert torch.equal(outs[i], ref[i]), (repeat, i)
    shared = torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_hostio_batches(
        lay.plan, [h["x"] for h in host],
        None if host[0]["x_scales"] is None else [h["x_scales"] for h in host],
        [h["topk_idx"] for h in host], [h["topk_w"] for h in host], base["w1"],
        base["w1_scales"], base["w2"], base["w2_scales"], [shared] * 3, lay.workspace)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(shared, ref[2])
    assert lay.check() == 0


WIDE_SPLIT = Workload("wide-split", 600, 1024, 512, 8, 4, cfg_id=25)   # ~300 rows per expert
RAGGED_BF16 = Workload("ragged-bf16", 300, 1024, 512, 8, 4, w_dtype="bf16", cfg_id=26)


def _layer_wide(wl, wide, debug=False, tiled=False, swap=None):
    return moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                        alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, debug=debug,
                        tiled_weights=tiled, chunked_scales=tiled and wl.w_dtype == "e2m1",
                        swap_ab=swap, wide_tiles=wide)


def _forward(lay, d, w1=None, w2=None, s1=None, s2=None):
    out = lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"],
                      d["w1"] if w1 is None else w1, d["w1_scales"] if s1 is None else s1,
                      d["w2"] if w2 is None else w2, d["w2_scales"] if s2 is None else s2)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("wl", [RAGGED, RAGGED_FP4, RAGGED_OAI, RAGGED_BF16, WIDE_SPLIT,
                                WORKLOADS["tiny"], SINGLE], ids=lambda w: w.name)
def test_wide_tiles_match_oracle(wl):
    """Wide token-major tiles forced on: pairs of m-tiles with 129..240 rows
    become one tile of N up to 240 tokens, larger pairs two tiles, lone
    m-tiles one; whole-layer parity with the oracle for every weight format."""
    d = inputs(wl)
    lay = _layer_wide(wl, 2)
    assert moe.moe_plan_wide_tiles_active(lay.plan)
    out = _forward(lay, d)
    assert lay.check() == 0
    dn = to_numpy(d)
    if wl.w_dtype == "bf16":
        ref = L.layer_bf16(dn["x"], dn["topk_idx"], dn["topk_w"], dn["w1"], dn["w2"],
                           alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit)
    else:
        ref = L.layer(*oracle_args(dn), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, f"wide {wl.name}")


@pytest.mark.parametrize("w_dtype", ["e4m3", "e2m1"])
def test_wide_tile_boundaries_240_and_241_rows(w_dtype):
    """An expert with exactly 240 tokens (the widest tile: accumulators fill
    TMEM columns 0..479) and one with 241 (split into 128 + 113 rows)."""
    wl = Workload("wide-edge", 481, 1024, 512, 2, 1, w_dtype=w_dtype, cfg_id=27)
    d = inputs(wl)
    d["topk_idx"][:241, 0] = 0
    d["topk_idx"][241:, 0] = 1
    d["topk_w"].fill_(1.0)
    lay = _layer_wide(wl, 2)
    out = _forward(lay, d)
    assert lay.check() == 0
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, "wide 240/241")
    # the same tokens with token-row tiles only agree within rounding
    ref_rows = _forward(_layer_wide(wl, 1, swap=1), d)
    assert_parity(out.float().cpu().numpy(), ref_rows.float().cpu().numpy(), "wide vs rows")


@pytest.mark.parametrize("wl", [RAGGED, RAGGED_FP4, WIDE_SPLIT], ids=lambda w: w.name)
def test_wide_requant_bytes_exact(wl):
    """With wide tiles the FC1 epilogue's two rounds of tokens write FP8 codes
    and scales equal to the oracle quantiser on the GPU's own fp32 activation."""
    d = inputs(wl)
    lay = _layer_wide(wl, 2, debug=True)
    _forward(lay, d)
    v = lay.view()
    rows = v.rows
    act_t = torch.empty(rows, wl.I, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act(lay.plan, lay.workspace, act_t)
    a32 = _ws_bytes(lay, v.act_f32, rows * wl.I * 4).view(torch.float32).view(rows, wl.I)
    sf = torch.empty(rows, wl.I // 128, dtype=torch.uint8, device="cuda")
    moe.moe_copy_act_scales(lay.plan, lay.workspace, sf)
    counts = _ws_bytes(lay, v.counts, 4 * wl.E).view(torch.int32).cpu().numpy()
    pad = _ws_bytes(lay, v.pad_offsets, 4 * (wl.E + 1)).view(torch.int32).cpu().numpy()
    act, a32, sf = act_t.cpu().numpy(), a32.cpu().numpy(), sf.cpu().numpy()
    assert counts.max() > 128
    for e in range(wl.E):
        r = slice(pad[e], pad[e] + counts[e])
        q_ref, s_ref = L.requant_1x128(a32[r].astype(np.float64))
        np.testing.assert_array_equal(act[r], q_ref, err_msg=f"codes, expert {e}")
        np.testing.assert_array_equal(sf[r], s_ref, err_msg=f"scales, expert {e}")


@pytest.mark.parametrize("wl", [RAGGED, RAGGED_FP4, WIDE_SPLIT], ids=lambda w: w.name)
def test_wide_fused_equals_separate_tiled_equals_row_major_and_repeatable(wl):
    d = inputs(wl)
    lay = _layer_wide(wl, 2)
    full = _forward(lay, d)
    again = _forward(lay, d)
    assert torch.equal(full, again)
    v = lay.view()
    n = wl.T * wl.k * wl.H * 2
    off = v.y - lay.workspace.data_ptr()
    y_fused = lay.workspace[off:off + n].clone()
    moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
    moe.moe_gather(lay.plan, d["x"], d["x_scales"], lay.workspace)
    moe.moe_fc1(lay.plan, d["w1"], d["w1_scales"], lay.workspace)
    moe.moe_fc2(lay.plan, d["w2"], d["w2_scales"], lay.workspace)
    torch.cuda.synchronize()
    assert torch.equal(lay.workspace[off:off + n], y_fused)
    tl = _layer_wide(wl, 2, tiled=True)
    w1, w2 = tl.prepack(d["w1"], d["w2"])
    s1, s2 = ((tl.prepack_scales(d["w1_scales"], d["w2_scales"])) if wl.w_dtype == "e2m1"
              else (d["w1_scales"], d["w2_scales"]))
    assert torch.equal(_forward(tl, d, w1, w2, s1, s2), full)


def test_wide_tiles_auto_at_the_mid_size_workloads():
    for T in (1024, 1536):
        wl = WORKLOADS["mxfp4"].with_tokens(T)
        lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype)
        assert moe.moe_plan_wide_tiles_active(lay.plan), wl.name
    for name in ("decode", "prefill", "oai"):
        wl = WORKLOADS[name]
        lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                           alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit)
        assert not moe.moe_plan_wide_tiles_active(lay.plan), name
