"""Routing (histogram, exclusive scan, stable scatter) on the GPU, bit-exact
against the oracle's routing."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from oracle import layer as L

from gpu_helpers import ensure_built

pytestmark = pytest.mark.gpu


def _route_gpu(T, k, E, idx):
    ensure_built()
    plan = moe.moe_plan(T, 512, 128, E, k)
    ws = torch.empty(moe.moe_workspace_bytes(plan), dtype=torch.uint8, device="cuda")
    moe.moe_clear_device_error(plan, ws)
    d_idx = torch.from_numpy(idx.astype(np.int32)).cuda()
    moe.moe_route(plan, d_idx, ws)
    v = moe.moe_workspace_view(plan, ws)
    S = T * k

    torch.cuda.synchronize()
    out = {}
    for name, n in (("counts", E), ("offsets", E + 1), ("perm", S), ("inv", S)):
        ptr = getattr(v, name)
        buf = torch.empty(n, dtype=torch.int32, device="cuda")
        off = ptr - ws.data_ptr()
        buf.copy_(ws[off:off + 4 * n].view(torch.int32))
        out[name] = buf.cpu().numpy()
    status = moe.moe_check_device_error(plan, ws)
    moe.moe_plan_destroy(plan)
    return out, status


def _cases():
    rng = np.random.default_rng(7)
    cases = []
    for T, k, E in [(1, 1, 1), (1, 8, 32), (64, 2, 8), (128, 8, 32), (2048, 4, 64),
                    (8192, 8, 32), (32768, 6, 48), (3000, 8, 256)]:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]) if T <= 4096 else \
            np.argsort(rng.random((T, E)), axis=1)[:, :k]
        cases.append((f"uniform-T{T}-k{k}-E{E}", T, k, E, idx))
    p = np.arange(1, 33) ** -1.2
    p[-4:] = 0
    idx = np.stack([rng.choice(32, 8, replace=False, p=p / p.sum()) for _ in range(128)])
    cases.append(("zipf-empty-experts", 128, 8, 32, idx))
    cases.append(("all-one-expert", 500, 1, 16, np.full((500, 1), 5)))
    return cases


@pytest.mark.parametrize("name,T,k,E,idx", _cases(), ids=[c[0] for c in _cases()])
def test_route_bit_exact(name, T, k, E, idx):
    got, status = _route_gpu(T, k, E, idx)
    counts, offsets, perm, inv = L.route(idx, E)
    np.testing.assert_array_equal(got["counts"], counts)
    np.testing.assert_array_equal(got["offsets"], offsets)
    np.testing.assert_array_equal(got["perm"], perm)
    np.testing.assert_array_equal(got["inv"], inv)
    assert status == 0


def test_route_out_of_range_ids_are_skipped_and_reported():
    rng = np.random.default_rng(11)
    T, k, E = 777, 4, 16
    idx = rng.integers(0, E, size=(T, k))
    idx[3, 1] = -1
    idx[500, 0] = E
    idx[776, 3] = 1 << 20
    got, status = _route_gpu(T, k, E, idx)
    counts, offsets, perm, inv = L.route(idx, E)
    np.testing.assert_array_equal(got["perm"], perm)
    np.testing.assert_array_equal(got["inv"], inv)
    np.testing.assert_array_equal(got["counts"], counts)
    assert status == 6      # MOE_ERR_BAD_ROUTING


def test_route_is_repeatable():
    rng = np.random.default_rng(3)
    idx = np.argsort(rng.random((8192, 32)), axis=1)[:, :8]
    a, _ = _route_gpu(8192, 8, 32, idx)
    b, _ = _route_gpu(8192, 8, 32, idx)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])


def test_route_masked_slots_are_not_errors():
    rng = np.random.default_rng(19)
    T, k, E = 513, 4, 16
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    idx[rng.random((T, k)) < 0.2] = -1          # masked slots
    got, status = _route_gpu(T, k, E, idx)
    counts, offsets, perm, inv = L.route(idx, E)
    np.testing.assert_array_equal(got["perm"], perm)
    np.testing.assert_array_equal(got["inv"], inv)
    assert status == 0
