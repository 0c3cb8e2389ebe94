"""The C-ABI library: it loads, exports every entry point include/moe.h
declares, and validates arguments on the host before launching anything
(these calls never reach the GPU, so they run on CPU-only machines)."""
import ctypes
import math
import os
import re

import pytest

import moe_expert_ffn_permute_b200 as moe
from moe_expert_ffn_permute_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    build()
    return moe.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_entry_points():
    names = _declared()
    for n in ("moe_plan", "moe_forward", "moe_route", "moe_gather", "moe_fc1_fc2", "moe_fc1", "moe_fc2", "moe_combine",
              "moe_workspace_bytes", "moe_check_device_error", "moe_plan_destroy",
              "moe_status_str"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) <= set(moe._SIGS)


def test_plan_validation():
    ok = moe.moe_plan(64, 512, 256, 8, 2)
    assert moe.moe_workspace_bytes(ok) > 0
    moe.moe_plan_destroy(ok)
    bad = [dict(T=0, H=512, I=256, E=8, k=2), dict(T=4, H=500, I=256, E=8, k=2),
           dict(T=4, H=512, I=200, E=8, k=2), dict(T=4, H=512, I=256, E=2, k=3),
           dict(T=4, H=512, I=256, E=300, k=2), dict(T=4, H=384, I=256, E=8, k=2)]
    codes = []
    for b in bad:
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_plan(b["T"], b["H"], b["I"], b["E"], b["k"])
        codes.append(ei.value.status)
    assert codes == [1, 2, 2, 1, 2, 2]
    with pytest.raises(moe.MoEError):
        moe.moe_plan(4, 512, 256, 8, 2, act="swiglu_oai", alpha=1.0, up_bias=0.0, limit=-1.0)
    with pytest.raises(moe.MoEError):
        moe.moe_plan(4, 512, 256, 8, 2, act="swiglu_oai", alpha=math.nan)


def test_workspace_grows_with_debug_capture():
    p = moe.moe_plan(64, 512, 256, 8, 2)
    a = moe.moe_workspace_bytes(p)
    moe.moe_plan_set_debug(p, True)
    b = moe.moe_workspace_bytes(p)
    assert b > a
    moe.moe_plan_destroy(p)


def test_forward_rejects_bad_pointers_before_launch():
    p = moe.moe_plan(64, 512, 256, 8, 2)
    good = 1 << 20                        # aligned fake addresses: never dereferenced
    args = [good] * 9
    with pytest.raises(moe.MoEError) as ei:             # null workspace
        moe.moe_forward(p, *args, None, stream=0)
    assert ei.value.status == 1
    with pytest.raises(moe.MoEError) as ei:             # misaligned workspace
        moe.moe_forward(p, *args, good + 8, stream=0)
    assert ei.value.status == 3
    with pytest.raises(moe.MoEError) as ei:             # null x
        moe.moe_forward(p, None, *args[1:], good, stream=0)
    assert ei.value.status == 1
    with pytest.raises(moe.MoEError) as ei:             # misaligned w1
        moe.moe_forward(p, good, good, good, good, good + 4, good, good, good, good, good,
                        stream=0)
    assert ei.value.status == 3
    moe.moe_plan_destroy(p)


def test_fp4_weights_need_32_byte_alignment():
    p = moe.moe_plan(8, 512, 256, 8, 2, w_dtype="e2m1")
    g = 1 << 20
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_fc2(p, g + 16, g, g, stream=0)
    assert ei.value.status == 3
    moe.moe_plan_destroy(p)


def test_status_strings():
    assert moe.moe_status_str(0) == "MOE_OK"
    assert moe.moe_status_str(5) == "MOE_ERR_DEVICE_TIMEOUT"


def test_tiled_weights_only_for_fp8():
    p = moe.moe_plan(8, 512, 256, 8, 2, w_dtype="e2m1")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_plan_set_weight_layout(p, True)
    assert ei.value.status == 2
    moe.moe_plan_destroy(p)
    q = moe.moe_plan(8, 512, 256, 8, 2)
    moe.moe_plan_set_weight_layout(q, True)
    moe.moe_plan_destroy(q)


def test_cta_pair_mode_selection_and_launch_count():
    """The 2-SM GEMM runs only when asked for with tiled FP8 weights; it adds
    the weight-scale expansion launch to the forward sequence."""
    p = moe.moe_plan(8192, 7168, 2048, 32, 8)
    base = moe.moe_forward_launch_count(p)
    with pytest.raises(moe.MoEError) as ei:          # row-major weights: no pairs
        moe.moe_plan_set_cta_pairs(p, 2)
    assert ei.value.status == 2
    assert not moe.moe_plan_cta_pairs_active(p)
    moe.moe_plan_set_weight_layout(p, True)
    for mode, active in ((0, False), (1, False), (2, True), (0, False)):
        moe.moe_plan_set_cta_pairs(p, mode)
        assert moe.moe_plan_cta_pairs_active(p) == active
        assert moe.moe_forward_launch_count(p) == base + (1 if active else 0)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_plan_set_cta_pairs(p, 3)
    assert ei.value.status == 1
    moe.moe_plan_destroy(p)
    q = moe.moe_plan(64, 512, 256, 8, 2, w_dtype="e2m1")
    with pytest.raises(moe.MoEError):
        moe.moe_plan_set_cta_pairs(q, 2)
    assert not moe.moe_plan_cta_pairs_active(q)
    moe.moe_plan_destroy(q)
    assert not moe.moe_plan_cta_pairs_active(None)


def test_bf16_plans_take_no_scales_and_tiled_weights():
    g = 1 << 20                          # aligned fake addresses: never dereferenced
    p = moe.moe_plan(64, 512, 256, 8, 2, w_dtype="bf16")
    q = moe.moe_plan(64, 512, 256, 8, 2)
    # Without scales a BF16 plan gets as far as the alignment check of x (no
    # launch happens); an FP8 plan stops at the missing x_scales.
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward(p, g + 4, None, g, g, g, None, g, None, g, g, stream=0)
    assert ei.value.status == 3
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward(q, g + 4, None, g, g, g, g, g, g, g, g, stream=0)
    assert ei.value.status == 1
    with pytest.raises(moe.MoEError) as ei:          # no activation scales to copy
        moe.moe_copy_act_scales(p, g, g, stream=0)
    assert ei.value.status == 2
    moe.moe_plan_set_weight_layout(p, True)           # tiled BF16 weights are fine
    with pytest.raises(moe.MoEError) as ei:          # the 2-SM kernel is FP8 only
        moe.moe_plan_set_cta_pairs(p, 2)
    assert ei.value.status == 2
    # 2-byte activations: the workspace is larger than the FP8 plan's.
    assert moe.moe_workspace_bytes(p) > moe.moe_workspace_bytes(q)
    moe.moe_plan_destroy(p)
    moe.moe_plan_destroy(q)


def test_swap_ab_selection():
    """Token-major tiles: tile by tile in automatic mode (any weight format),
    forced on or off by the mode, never with CTA pairs."""
    p = moe.moe_plan(128, 7168, 2048, 32, 8)
    assert moe.moe_plan_swap_ab_active(p) == 2
    moe.moe_plan_set_swap_ab(p, 1)
    assert moe.moe_plan_swap_ab_active(p) == 0
    moe.moe_plan_set_weight_layout(p, True)
    moe.moe_plan_set_swap_ab(p, 2)
    assert moe.moe_plan_swap_ab_active(p) == 1
    moe.moe_plan_set_cta_pairs(p, 2)                    # pairs take precedence
    assert moe.moe_plan_swap_ab_active(p) == 0
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_plan_set_swap_ab(p, 3)
    assert ei.value.status == 1
    moe.moe_plan_destroy(p)
    b = moe.moe_plan(128, 512, 256, 8, 2, w_dtype="bf16")
    assert moe.moe_plan_swap_ab_active(b) == 2
    moe.moe_plan_set_swap_ab(b, 2)
    assert moe.moe_plan_swap_ab_active(b) == 1
    moe.moe_plan_destroy(b)


def test_debug_flags():
    p = moe.moe_plan(64, 512, 256, 8, 2)
    a = moe.moe_workspace_bytes(p)
    moe.moe_plan_set_debug(p, 2)                 # failure-path hook only: no capture buffer
    assert moe.moe_workspace_bytes(p) == a
    moe.moe_plan_set_debug(p, 3)
    assert moe.moe_workspace_bytes(p) > a
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_plan_set_debug(p, 4)
    assert ei.value.status == 1
    moe.moe_plan_destroy(p)



def test_fp4_chunked_scale_layout_rules():
    g = 1 << 20
    p = moe.moe_plan(64, 512, 256, 8, 2, w_dtype="e2m1")
    q = moe.moe_plan(64, 512, 256, 8, 2)
    moe.moe_plan_set_weight_layout(p, 2)
    with pytest.raises(moe.MoEError) as ei:          # chunked scales: MXFP4 only
        moe.moe_plan_set_weight_layout(q, 2)
    assert ei.value.status == 2
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_prepack_weight_scales(q, g, g, g, g, stream=0)
    assert ei.value.status == 2
    with pytest.raises(moe.MoEError) as ei:          # chunk copies need 16-byte alignment
        moe.moe_prepack_weight_scales(p, g, g, g + 4, g, stream=0)
    assert ei.value.status == 3
    with pytest.raises(moe.MoEError) as ei:          # and so do the kernels' reads of them
        moe.moe_fc2(p, g, g + 4, g, stream=0)
    assert ei.value.status == 3
    moe.moe_plan_destroy(p)
    moe.moe_plan_destroy(q)


def test_debug_capture_moves_no_other_buffer():
    """Switching the fp32 debug capture on grows the workspace at its end only:
    every other buffer keeps its offset (a workspace sized before the switch is
    still valid for all of them)."""
    fake = 1 << 30                                     # any 256-B aligned address
    for w_dtype in ("e4m3", "e2m1", "bf16"):
        p = moe.moe_plan(300, 1024, 512, 8, 4, w_dtype=w_dtype)
        before = moe.moe_workspace_bytes(p)
        v0 = moe.moe_workspace_view(p, fake)
        moe.moe_plan_set_debug(p, 1)
        after = moe.moe_workspace_bytes(p)
        v1 = moe.moe_workspace_view(p, fake)
        names = ("counts", "offsets", "perm", "inv", "pad_offsets", "act", "y", "error_word")
        for name in names:
            assert getattr(v0, name) == getattr(v1, name), (w_dtype, name)
        assert v0.act_f32 is None and v1.act_f32 is not None
        assert v1.act_f32 - fake >= before - 256          # placed after everything else
        assert after - before >= v1.rows * 512 * 4
        moe.moe_plan_set_debug(p, 0)
        assert moe.moe_workspace_bytes(p) == before
        moe.moe_plan_destroy(p)


def test_hostio_batches_validates_before_enqueuing(L):
    """The batched host-buffer entry refuses a bad batch count or a missing
    array / entry before it touches CUDA (it creates its copy streams only
    after validation)."""
    p = moe.moe_plan(64, 512, 256, 8, 2)
    ws, w = 1 << 30, 1 << 20                               # aligned stand-ins, never read
    arr = lambda n, v=1 << 12: (ctypes.c_void_p * n)(*([v] * n))
    good = dict(x=arr(2), xs=arr(2), idx=arr(2), tw=arr(2), out=arr(2))

    def call(n, **kw):
        a = dict(good, **kw)
        return L.moe_forward_hostio_batches(p, n, a["x"], a["xs"], a["idx"], a["tw"], w, w, w, w,
                                            a["out"], ws, None)
    assert call(0) == 1
    assert call(-3) == 1
    assert call(2, x=None) == 1
    assert call(2, xs=None) == 1                            # FP8 plans need x scales
    assert call(2, out=arr(2, 0)) == 1                      # a NULL entry
    assert call(2, idx=(ctypes.c_void_p * 2)(1 << 12, None)) == 1
    assert L.moe_forward_hostio_batches(p, 2, good["x"], good["xs"], good["idx"], good["tw"],
                                        w + 1, w, w, w, good["out"], ws, None) == 3
    moe.moe_plan_destroy(p)


def test_weight_layout_values_per_format():
    """Tiled MXFP4 codes (layout 3) need an MXFP4 plan; FP8 / BF16 take the
    pre-swizzled tiles (1); chunked scales alone (2) are MXFP4 only."""
    expect = {"e4m3": {0: 0, 1: 0, 2: 2, 3: 2}, "bf16": {0: 0, 1: 0, 2: 2, 3: 2},
              "e2m1": {0: 0, 1: 2, 2: 0, 3: 0}}
    for w_dtype, codes in expect.items():
        p = moe.moe_plan(64, 512, 256, 8, 2, w_dtype=w_dtype)
        for layout, status in codes.items():
            got = moe.lib().moe_plan_set_weight_layout(p, layout)
            assert got == status, (w_dtype, layout, got)
        assert moe.lib().moe_plan_set_weight_layout(p, 4) == 1
        moe.moe_plan_destroy(p)


def test_wide_tile_selection():
    """Wide token-major tiles: automatic for MXFP4 weights with 96 < T*k/E <= 224
    slots per expert, forced on or off by mode, never without token-major
    tiles."""
    def active(T, k, E, w_dtype="e2m1", **modes):
        p = moe.moe_plan(T, 1024, 512, E, k, w_dtype=w_dtype)
        if "swap" in modes:
            moe.moe_plan_set_swap_ab(p, modes["swap"])
        if "wide" in modes:
            moe.moe_plan_set_wide_tiles(p, modes["wide"])
        a = moe.moe_plan_wide_tiles_active(p)
        moe.moe_plan_destroy(p)
        return a
    assert active(1024, 6, 48)                 # 128 slots per expert
    assert active(1536, 6, 48)                 # 192
    assert not active(1024, 6, 48, "e4m3")     # FP8 and BF16 weights: never automatically
    assert not active(2048, 4, 64, "e4m3")
    assert not active(512, 8, 32, "bf16")
    assert not active(128, 6, 48)              # 16: decode size
    assert not active(8192, 6, 48)             # 1024: prefill size
    assert active(97, 4, 4)                    # 97 slots per expert
    assert not active(96, 4, 4)                # 96
    assert active(224, 4, 4)                   # 224
    assert not active(225, 4, 4)               # 225
    assert active(128, 8, 32, "e4m3", wide=2)
    assert not active(1024, 6, 48, wide=1)
    assert not active(1024, 6, 48, swap=1)     # needs token-major tiles
    assert not active(1024, 6, 48, swap=1, wide=2)
    with pytest.raises(moe.MoEError):
        p = moe.moe_plan(64, 512, 256, 8, 2)
        try:
            moe.moe_plan_set_wide_tiles(p, 3)
        finally:
            moe.moe_plan_destroy(p)
