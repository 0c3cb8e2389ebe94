"""The Python convenience layer's tensor checks (``check_layer_args``, called by
``MoELayer.forward`` before the C ABI, which sees only pointers): every input
the generators produce for each weight format passes, including prepacked
weights and chunked scales (same shapes), and a wrong shape, dtype, device,
layout or a missing tensor is refused with MOE_ERR_INVALID_ARG."""
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from workloads.synth import Workload, make_inputs

CPU = torch.device("cpu")
CASES = [Workload("ragged", 300, 1024, 512, 8, 4, cfg_id=10),
         Workload("ragged-fp4", 200, 1024, 512, 6, 3, w_dtype="e2m1", cfg_id=11),
         Workload("ragged-bf16", 300, 1024, 512, 8, 4, w_dtype="bf16", cfg_id=30),
         Workload("single", 1, 512, 128, 1, 1, cfg_id=12)]


def _args(wl, d, **over):
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16)
    a = dict(x=d["x"], x_scales=d["x_scales"], topk_idx=d["topk_idx"], topk_w=d["topk_w"],
             w1=d["w1"], w1_scales=d["w1_scales"], w2=d["w2"], w2_scales=d["w2_scales"], out=out)
    a.update(over)
    return a


def _check(wl, **a):
    moe.check_layer_args(wl.T, wl.H, wl.I, wl.E, wl.k, wl.w_dtype, CPU, **a)


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_generated_inputs_pass(wl):
    d = make_inputs(wl)
    _check(wl, **_args(wl, d))
    # Prepacked weights / chunked scales are buffers of the same shape.
    _check(wl, **_args(wl, d, w1=torch.empty_like(d["w1"]), w2=torch.empty_like(d["w2"])))
    # Raw addresses are passed through unchecked.
    _check(wl, **_args(wl, d, w1=12345 * 256))


@pytest.mark.parametrize("wl", CASES[:3], ids=lambda w: w.name)
def test_bad_tensors_are_refused(wl):
    d = make_inputs(wl)
    bad = [dict(x=d["x"][:-1]),                                  # too few rows
           dict(topk_idx=d["topk_idx"].long()),                  # int64 ids
           dict(topk_w=d["topk_w"].double()),
           dict(w2=d["w2"][:, :, :-16]),                         # short rows
           dict(out=torch.empty(wl.T, wl.H, dtype=torch.float32)),
           dict(x=d["x"].t().contiguous().t()),                  # not contiguous
           dict(topk_idx=None)]
    if wl.w_dtype != "bf16":
        bad += [dict(x_scales=None), dict(w1_scales=d["w1_scales"][:-1])]
    for over in bad:
        with pytest.raises(moe.MoEError) as ei:
            _check(wl, **_args(wl, d, **over))
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG, over
    with pytest.raises(moe.MoEError):
        moe.check_layer_args(wl.T, wl.H, wl.I, wl.E, wl.k, wl.w_dtype, torch.device("meta"),
                             **_args(wl, d))


def test_bf16_layers_ignore_scale_arguments():
    wl = CASES[2]
    d = make_inputs(wl)
    _check(wl, **_args(wl, d, x_scales=torch.empty(1), w1_scales=None))


@pytest.mark.parametrize("w_dtype", ["e4m3", "e2m1", "bf16"])
def test_layer_forward_checks_before_the_call(monkeypatch, w_dtype):
    """MoELayer.forward runs the checks and only then calls moe_forward (the
    library calls that need a GPU are replaced by recorders here)."""
    calls = []
    monkeypatch.setattr(moe, "moe_clear_device_error", lambda *a, **k: None)
    monkeypatch.setattr(moe, "moe_forward", lambda *a, **k: calls.append(a))
    wl = Workload("t", 40, 512, 256, 4, 2, w_dtype=w_dtype, cfg_id=3)
    d = make_inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=w_dtype, device="cpu")
    args = [d[n] for n in ("x", "x_scales", "topk_idx", "topk_w", "w1", "w1_scales", "w2",
                           "w2_scales")]
    out = lay.forward(*args)
    assert out.shape == (wl.T, wl.H) and out.dtype == torch.bfloat16 and len(calls) == 1
    args[0] = args[0][:-1]
    with pytest.raises(moe.MoEError):
        lay.forward(*args)
    assert len(calls) == 1


def test_route_static_refuses_bad_tensors_before_the_call():
    """moe_route_static's binding checks dtype, contiguity, size and device of
    its five tensors before the C call (which would otherwise write past a
    short buffer); every refusal happens on the host."""
    import torch
    T, k, E = 16, 2, 8
    S = T * k
    good = dict(topk_idx=torch.zeros(S, dtype=torch.int32), counts=torch.zeros(E, dtype=torch.int32),
                offsets=torch.zeros(E + 1, dtype=torch.int32), perm=torch.zeros(S, dtype=torch.int32),
                inv=torch.zeros(S, dtype=torch.int32))
    order = ("topk_idx", "counts", "offsets", "perm", "inv")

    def call(**kw):
        a = dict(good, **kw)
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_route_static(a["topk_idx"], T, k, E, *(a[n] for n in order[1:]))
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG
        return str(ei.value)

    assert "int32" in call(counts=torch.zeros(E, dtype=torch.int64))
    assert "needs 9" in call(offsets=torch.zeros(E, dtype=torch.int32))
    assert "needs 32" in call(perm=torch.zeros(S - 1, dtype=torch.int32))
    assert "contiguous" in call(inv=torch.zeros(S, 2, dtype=torch.int32)[:, 0])
    assert "required" in call(topk_idx=None)
    assert "CUDA device" in call()                     # right shapes, but host tensors
