"""Failure detection on the GPU without a fault: the fused FC1+FC2 launch's
FC2 dependency wait is made unreachable (debug flag bit 1), the bounded wait
runs out, the kernel returns with MOE_ERR_DEVICE_TIMEOUT in the workspace's
error word -- no trap, no hang -- and the context stays usable.  Plus a
scheduler stress run: many tiny experts, the task-slot ring reused thousands of
times, every replay bitwise equal."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from workloads.synth import Workload, to_numpy
from oracle import layer as L

from gpu_helpers import assert_parity, ensure_built, inputs, oracle_args, oracle_kw

pytestmark = pytest.mark.gpu

RAGGED = Workload("ragged", 300, 1024, 512, 8, 4, cfg_id=20)
TINY_EXPERTS = Workload("tiny-experts", 48, 512, 256, 64, 2, routing="zipf", cfg_id=40)


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _forward(lay, d, out=None):
    return lay.forward(d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"],
                       d["w1_scales"], d["w2"], d["w2_scales"], out)


@pytest.mark.timeout(120)
@pytest.mark.parametrize("swap", [1, 2], ids=["token-rows", "swap-ab"])
def test_bounded_wait_runs_out_and_reports_timeout(swap):
    wl = RAGGED
    d = inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, swap_ab=swap)
    moe.moe_plan_set_debug(lay.plan, 2)
    _forward(lay, d)
    torch.cuda.synchronize()
    assert lay.check() == 5            # MOE_ERR_DEVICE_TIMEOUT
    # The context is usable: the same plan without the hook gives the layer.
    moe.moe_plan_set_debug(lay.plan, 0)
    moe.moe_clear_device_error(lay.plan, lay.workspace)
    out = _forward(lay, d)
    torch.cuda.synchronize()
    assert lay.check() == 0
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(out.float().cpu().numpy(), ref, "after timeout")


def test_scheduler_slot_ring_stress():
    """64 experts, 96 slots (most experts get 0-3 tokens): thousands of tiny
    tasks cycle through the 4-slot task ring; 300 graph replays must all give
    the first replay's bytes."""
    wl = TINY_EXPERTS
    d = inputs(wl)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device="cuda")
    _forward(lay, d, out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _forward(lay, d, out)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    first = out.clone()
    for _ in range(300):
        g.replay()
    torch.cuda.synchronize()
    assert lay.check() == 0
    assert torch.equal(out, first)
    ref = L.layer(*oracle_args(to_numpy(d)), **oracle_kw(wl))
    assert_parity(first.float().cpu().numpy(), ref, "tiny experts")
    del g
