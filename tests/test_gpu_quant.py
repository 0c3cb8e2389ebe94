"""Input quantisation (bf16 -> E4M3 + UE8M0 per 1x128) on the GPU, byte for
byte against the oracle's quantiser applied to the same bf16 values."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from oracle import layer as L

from gpu_helpers import assert_parity, ensure_built
from workloads.synth import Workload, make_inputs, to_numpy

pytestmark = pytest.mark.gpu


def _quant_gpu(x):
    T, H = x.shape
    codes = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    scales = torch.empty(T, H // 128, dtype=torch.uint8, device="cuda")
    moe.moe_quantize_act(x, T, H, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("T,H,scale", [(1, 128, 1.0), (64, 512, 1.0), (300, 7168, 3.0),
                                        (7, 1024, 1e-3), (5, 3072, 200.0)])
def test_quantize_matches_oracle_bytes(T, H, scale):
    ensure_built()
    g = torch.Generator(device="cuda")
    g.manual_seed(T * 1000 + H)
    x = (torch.randn(T, H, generator=g, device="cuda") * scale).to(torch.bfloat16)
    x[0, :128] = 0                                   # an all-zero block
    if H >= 256:
        x[0, 128] = 448.0                            # amax exactly on a boundary
        x[0, 129:256] = 1.0
    codes, scales = _quant_gpu(x)
    ref_codes, ref_scales = L.requant_1x128(x.float().cpu().numpy().astype(np.float64))
    np.testing.assert_array_equal(scales, ref_scales)
    np.testing.assert_array_equal(codes, ref_codes)


def test_quantize_feeds_the_layer():
    """bf16 activations quantised by the kernel, then the whole layer on those
    codes, against the oracle layer on the oracle quantiser's codes of the same
    bf16 values (the two quantisations are byte-identical, checked first)."""
    ensure_built()
    wl = Workload("quant-chain", 96, 512, 256, 8, 2, cfg_id=42)
    d = make_inputs(wl, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(42)
    x = (torch.randn(wl.T, wl.H, generator=g, device="cuda") * 2.0).to(torch.bfloat16)
    codes, scales = _quant_gpu(x)
    ref_codes, ref_scales = L.requant_1x128(x.float().cpu().numpy().astype(np.float64))
    np.testing.assert_array_equal(codes, ref_codes)
    np.testing.assert_array_equal(scales, ref_scales)
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k)
    out = lay.forward(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                      d["topk_idx"], d["topk_w"], d["w1"], d["w1_scales"], d["w2"],
                      d["w2_scales"])
    torch.cuda.synchronize()
    assert lay.check() == 0
    dn = to_numpy(d)
    ref = L.layer(ref_codes, ref_scales, dn["topk_idx"], dn["topk_w"], dn["w1"],
                  dn["w1_scales"], dn["w2"], dn["w2_scales"])
    assert_parity(out.float().cpu().numpy(), ref, "quantised input chain")


def test_quantize_rejects_bad_shapes():
    ensure_built()
    x = torch.zeros(4, 200, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_quantize_act(x, 4, 200, x, x)
    assert ei.value.status == 2
