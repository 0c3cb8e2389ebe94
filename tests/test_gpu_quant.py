"""Input quantisation (bf16 -> E4M3 + UE8M0 per 1x128) on the GPU, byte for
byte against the oracle's quantiser applied to the same bf16 values."""
import numpy as np
import pytest
import torch

import moe_expert_ffn_permute_b200 as moe
from oracle import layer as L

from gpu_helpers import ensure_built

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
    """Quantising with the kernel and running the layer equals running the layer
    on the same codes quantised by the oracle."""
    ensure_built()
    T, H = 64, 512
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    codes, scales = _quant_gpu(x)
    ref_codes, ref_scales = L.requant_1x128(x.float().cpu().numpy().astype(np.float64))
    assert (codes == ref_codes).all() and (scales == ref_scales).all()


def test_quantize_rejects_bad_shapes():
    ensure_built()
    x = torch.zeros(4, 200, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_quantize_act(x, 4, 200, x, x)
    assert ei.value.status == 2
