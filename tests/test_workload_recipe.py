"""The input recipe (workloads/synth.py) quantises x and the weights with the
same power-of-two block rule the oracle's requantiser states.  The recipe is
not part of either side, but a drift in it would silently change every
workload; these pins tie its quantisers to the oracle (E4M3, 1x128 and
128x128 blocks) and to the E2M1 definition (nearest representable value,
ties to the even code) on values that include the rule's edge cases."""
import numpy as np
import torch

from oracle import layer as L
from oracle.formats import (decode_e2m1, decode_ue8m0, encode_e4m3_rne_satfinite,
                            unpack_e2m1_pairs)
from workloads import synth


def _bf16_values(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16).float()


def _with_edge_blocks(v):
    """Blocks whose amax sits exactly on 448 * 2^n, just above it, a tiny-amax
    block (below the 1e-4 floor) and an all-zero block."""
    v = v.clone()
    v[0, 0:128] = 0.0                                   # zero block
    v[1, 0:128] = 1e-6                                  # below the amax floor
    v[1, 5] = -3e-6
    v[2, 0:128] = 0.5
    v[2, 7] = 448.0                                     # amax exactly 448 * 2^0
    v[3, 0:128] = -0.25
    v[3, 9] = -448.0 * 2.0 ** -6                        # exactly 448 * 2^-6
    v[4, 0:128] = 1.0
    v[4, 100] = float(torch.tensor(448.0).to(torch.bfloat16).float() * 1.0078125)  # just above
    v[5, 0:128] = 3.0
    v[5, 3] = 448.0 * 2.0 ** 5                           # 448 * 2^5
    return v


def test_x_quantiser_equals_oracle_requant_1x128():
    v = _with_edge_blocks(_bf16_values(64, 1024, 1))
    v = v.to(torch.bfloat16).float()                     # the recipe quantises bf16 values
    q, s = synth._quant_e4m3_blocks(v, 1, 128)
    q_ref, s_ref = L.requant_1x128(v.numpy().astype(np.float64))
    np.testing.assert_array_equal(s.numpy(), s_ref)
    np.testing.assert_array_equal(q.numpy(), q_ref)


def test_x_quantiser_over_wide_magnitudes():
    for seed, scale in ((2, 1e-3), (3, 250.0), (4, 3e4)):
        v = _bf16_values(16, 512, seed, scale)
        q, s = synth._quant_e4m3_blocks(v, 1, 128)
        q_ref, s_ref = L.requant_1x128(v.numpy().astype(np.float64))
        np.testing.assert_array_equal(s.numpy(), s_ref)
        np.testing.assert_array_equal(q.numpy(), q_ref)


def test_weight_quantiser_128x128_equals_oracle_rule_per_block():
    """A 128x128 block's scale byte is n + 127 with n the oracle's exponent for
    the block's amax, and its codes are the oracle's RNE-satfinite E4M3
    encoding of the block divided by 2^n."""
    v = _bf16_values(256, 384, 5, 0.02)
    v[0:128, 0:128] *= 1e3                               # blocks of very different size
    v[128, 300] = 448.0 * 2.0 ** -3                      # exact boundary in one block
    q, s = synth._quant_e4m3_blocks(v, 128, 128)
    vn = v.numpy().astype(np.float64)
    for rb in range(2):
        for cb in range(3):
            blk = vn[128 * rb:128 * rb + 128, 128 * cb:128 * cb + 128]
            n = L.ue8m0_exponent_for(np.abs(blk).max())
            assert int(s[rb, cb]) == n + 127
            np.testing.assert_array_equal(
                q[128 * rb:128 * rb + 128, 128 * cb:128 * cb + 128].numpy(),
                encode_e4m3_rne_satfinite(blk / 2.0 ** n))


def test_e2m1_quantiser_is_nearest_with_ties_to_even():
    v = _bf16_values(8, 256, 6, 0.02)
    v[0, 0:32] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4)  # exact ties
    v[1, 0:32] = torch.linspace(-6.0, 6.0, 32)
    packed, s = synth._quant_e2m1_rows(v)
    codes = unpack_e2m1_pairs(packed.numpy())
    vals = decode_e2m1(codes)
    scale = decode_ue8m0(s.numpy())                      # [R, C/32]
    x = v.numpy().astype(np.float64) / np.repeat(scale, 32, axis=1)
    grid = decode_e2m1(np.arange(16))
    for r in range(x.shape[0]):
        blk_amax = np.abs(v.numpy()[r].reshape(-1, 32)).max(axis=1).astype(np.float64)
        n = np.log2(scale[r])
        # the scale: smallest power of two with max(amax, 1e-4) <= 6 * 2^n
        a = np.maximum(blk_amax, 1e-4)
        assert np.all(a <= 6.0 * 2.0 ** n) and np.all(a > 6.0 * 2.0 ** (n - 1))
        for c in range(x.shape[1]):
            d = np.abs(grid - x[r, c])
            best = [b for b in np.flatnonzero(d == d.min())
                    if grid[b] == 0.0 or np.sign(grid[b]) == np.sign(x[r, c])]
            mags = sorted(set(abs(grid[b]) for b in best))
            if len(mags) > 1:                            # a tie: the even magnitude code wins
                want = [m for m in mags if list(grid[:8]).index(m) % 2 == 0]
                assert len(want) == 1
                assert abs(vals[r, c]) == want[0], (r, c, x[r, c], vals[r, c])
            else:
                assert abs(vals[r, c]) == mags[0], (r, c, x[r, c], vals[r, c])
            if vals[r, c] != 0.0:
                assert np.sign(vals[r, c]) == np.sign(x[r, c])
