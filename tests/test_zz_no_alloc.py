"""The allocation-free routing entry point (moe_route_static).

Callers that cannot allocate device memory where they route (for example a
runtime whose pooled allocator owns the whole device budget) use
moe_route_static, whose scratch lives in the library's static device memory.
Its results must equal those of the workspace-based moe_route, call after call
(the static scratch is shared and keeps the previous call's contents).  This
file is collected last so that a stop-at-first-failure run has already run
every other test.
"""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe

from gpu_helpers import ensure_built

pytestmark = pytest.mark.gpu


def _workspace_route(idx, T, k, E):
    plan = moe.moe_plan(T, 512, 128, E, k)
    ws = torch.empty(moe.moe_workspace_bytes(plan), dtype=torch.uint8, device="cuda")
    moe.moe_route(plan, idx, ws)
    v = moe.moe_workspace_view(plan, ws)
    S = T * k
    out = {}
    for name, n in (("counts", E), ("offsets", E + 1), ("perm", S), ("inv", S)):
        off = getattr(v, name) - ws.data_ptr()
        out[name] = ws[off:off + 4 * n].view(torch.int32).clone()
    torch.cuda.synchronize()
    moe.moe_plan_destroy(plan)
    return out


def _static_route(idx, T, k, E):
    S = T * k
    out = {"counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
           "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
           "perm": torch.full((S,), -7, dtype=torch.int32, device="cuda"),
           "inv": torch.full((S,), -7, dtype=torch.int32, device="cuda")}
    moe.moe_route_static(idx, T, k, E, out["counts"], out["offsets"], out["perm"], out["inv"])
    torch.cuda.synchronize()
    return out


def test_static_route_equals_workspace_route_on_consecutive_calls():
    ensure_built()
    rng = np.random.default_rng(123)
    cases = [(8192, 8, 32), (128, 8, 32)]           # many blocks, then one block
    for T, k, E in cases:
        idx_np = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
        idx_np[T // 2, 0] = E + 3                    # one unrouted slot
        idx = torch.from_numpy(idx_np).cuda()
        ref = _workspace_route(idx, T, k, E)
        got = _static_route(idx, T, k, E)
        for key in ref:
            assert torch.equal(got[key], ref[key]), (T, key)


def test_static_route_rejects_sizes_beyond_its_scratch():
    ensure_built()
    T, k, E = moe.ROUTE_STATIC_MAX_SLOTS // 8 + 1, 8, 32
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route_static(idx, T, k, E, idx, idx, idx, idx)
    assert ei.value.status == 2          # MOE_ERR_UNSUPPORTED, nothing enqueued


def test_static_route_drops_a_bad_id_without_a_status():
    """An expert id outside [0, E) (other than -1) leaves its slot unrouted
    (inv = -1, not counted) and, as documented, is not reported: the call
    returns MOE_OK because this entry point has no error word to read back."""
    ensure_built()
    T, k, E = 64, 4, 16
    idx = torch.randint(0, E, (T, k), dtype=torch.int32, device="cuda")
    idx[3, 1] = E + 3
    idx[9, 0] = -1
    got = _static_route(idx, T, k, E)
    assert int(got["inv"][3 * k + 1]) == -1 and int(got["inv"][9 * k]) == -1
    assert int(got["counts"].sum()) == T * k - 2
