"""The BF16 variant through the C ABI against the oracle's layer_bf16: ragged
parity, the bf16 FC1 activation byte for byte, the layouts and launch forms
tied together bitwise, and the full-size decode-shaped layer on sampled tokens."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from workloads.synth import WORKLOADS, Workload, to_numpy
from oracle import formats as F

from gpu_helpers import assert_parity, ensure_built, inputs, oracle_layer, oracle_tokens

pytestmark = pytest.mark.gpu

RAGGED_BF16 = Workload("ragged-bf16", 300, 1024, 512, 8, 4, w_dtype="bf16", cfg_id=30)
OAI_BF16 = Workload("oai-bf16", 200, 512, 384, 6, 3, w_dtype="bf16", act="swiglu_oai",
                    alpha=1.702, up_bias=1.0, limit=7.0, cfg_id=31)
SINGLE_BF16 = Workload("single-bf16", 1, 512, 128, 1, 1, w_dtype="bf16", cfg_id=32)


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _layer(wl, tiled=False, debug=False, swap=None):
    return moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype="bf16", act=wl.act,
                        alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, debug=debug,
                        tiled_weights=tiled, swap_ab=swap)


def _run(wl, d, tiled=False, debug=False, swap=None):
    lay = _layer(wl, tiled, debug, swap)
    w1, w2 = (lay.prepack(d["w1"], d["w2"]) if tiled else (d["w1"], d["w2"]))
    out = lay.forward(d["x"], None, d["topk_idx"], d["topk_w"], w1, None, w2, None)
    torch.cuda.synchronize()
    return out, lay


@pytest.mark.parametrize("swap", [1, 2], ids=["token-rows", "swap-ab"])
@pytest.mark.parametrize("wl", [RAGGED_BF16, OAI_BF16, SINGLE_BF16], ids=lambda w: w.name)
def test_layer_matches_oracle(wl, swap):
    d = inputs(wl)
    out, lay = _run(wl, d, swap=swap)
    assert lay.check() == 0
    ref = oracle_layer(wl, to_numpy(d))
    assert_parity(out.float().cpu().numpy(), ref, wl.name)


@pytest.mark.parametrize("swap", [1, 2], ids=["token-rows", "swap-ab"])
def test_activation_is_bf16_rne_of_the_fp32_activation(swap):
    """The FC1 epilogue's bf16 activation equals the oracle's round-to-nearest-
    even of the GPU's own fp32 activation (debug capture), bit for bit, on every
    routed row; and that fp32 activation matches the oracle's float64 one."""
    wl = RAGGED_BF16
    d = inputs(wl)
    out, lay = _run(wl, d, debug=True, swap=swap)
    v = lay.view()
    rows = v.rows
    act = torch.empty(rows, wl.I, dtype=torch.bfloat16, device="cuda")
    moe.moe_copy_act(lay.plan, lay.workspace, act)
    off = v.act_f32 - lay.workspace.data_ptr()
    a32 = lay.workspace[off:off + rows * wl.I * 4].view(torch.float32).view(rows, wl.I)
    off = v.pad_offsets - lay.workspace.data_ptr()
    pad = lay.workspace[off:off + 4 * (wl.E + 1)].view(torch.int32).cpu().numpy()
    act = act.view(torch.int16).cpu().numpy().view(np.uint16)
    a32 = a32.cpu().numpy()
    _, inter = oracle_layer(wl, to_numpy(d), keep=True)
    for e, a_ref in inter["a"].items():
        r = slice(pad[e], pad[e] + a_ref.shape[0])
        np.testing.assert_array_equal(act[r], F.encode_bf16_rne(a32[r].astype(np.float64)),
                                      err_msg=f"expert {e}")
        assert_parity(a32[r], a_ref, f"activation expert {e}")


def test_tiled_weights_give_the_same_bytes():
    wl = RAGGED_BF16
    d = inputs(wl)
    a, _ = _run(wl, d, tiled=False)
    b, lay = _run(wl, d, tiled=True)
    assert lay.check() == 0
    assert torch.equal(a, b)


def test_fused_gemm_equals_separate_launches():
    wl = RAGGED_BF16
    d = inputs(wl)
    _, lay = _run(wl, d)
    v = lay.view()
    n = wl.T * wl.k * wl.H * 2
    off = v.y - lay.workspace.data_ptr()
    moe.moe_route_gather(lay.plan, d["topk_idx"], d["x"], None, lay.workspace)
    moe.moe_fc1(lay.plan, d["w1"], None, lay.workspace)
    moe.moe_fc2(lay.plan, d["w2"], None, lay.workspace)
    torch.cuda.synchronize()
    y_sep = lay.workspace[off:off + n].clone()
    lay.workspace[off:off + n].zero_()
    moe.moe_route(lay.plan, d["topk_idx"], lay.workspace)
    moe.moe_gather(lay.plan, d["x"], None, lay.workspace)
    moe.moe_fc1_fc2(lay.plan, d["w1"], None, d["w2"], None, lay.workspace)
    torch.cuda.synchronize()
    assert lay.check() == 0
    assert torch.equal(lay.workspace[off:off + n], y_sep)


def test_hostio_equals_device_forward():
    wl = RAGGED_BF16
    d = inputs(wl)
    dev_out, lay = _run(wl, d)
    host = {k: d[k].cpu().pin_memory() for k in ("x", "topk_idx", "topk_w")}
    out_h = torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_hostio(lay.plan, host["x"], None, host["topk_idx"], host["topk_w"],
                           d["w1"], None, d["w2"], None, out_h, lay.workspace)
    torch.cuda.synchronize()
    assert torch.equal(out_h, dev_out.cpu())


def test_masked_and_bad_ids():
    wl = RAGGED_BF16
    d = inputs(wl)
    d["topk_idx"][torch.rand(wl.T, wl.k, device="cuda") < 0.2] = -1
    d["topk_idx"][7, 1] = wl.E + 3
    out, lay = _run(wl, d)
    assert lay.check() == 6
    ref = oracle_layer(wl, to_numpy(d))
    assert_parity(out.float().cpu().numpy(), ref, "bf16 masked / bad ids")


@pytest.mark.parametrize("tiled", [True, False], ids=["tiled", "row-major"])
def test_full_size_decode_shape_sampled_parity(tiled):
    """The decode layer's shape (T=128, H=7168, I=2048, E=32, k=8, skewed
    routing) with BF16 weights, in the launch configuration the benchmark times."""
    wl = WORKLOADS["bf16"]
    d = inputs(wl)
    out, lay = _run(wl, d, tiled=tiled)
    assert lay.check() == 0
    tokens = np.sort(np.random.default_rng(2).choice(wl.T, size=6, replace=False))
    ref = oracle_tokens(wl, to_numpy(d), tokens)
    assert_parity(out.float().cpu().numpy()[tokens], ref, f"bf16 decode {tiled}")
