"""Seeded synthetic inputs for the MoE expert layer (the workloads' stand-ins).

This module only draws and packs inputs; it performs no step of the layer
itself.  Both the CUDA path's tests/bench and the CPU oracle consume what it
returns.  Every array comes from a torch.Generator seeded with 1000 + config id,
on the device the caller names (CPU for the small cases; CUDA for the
multi-gigabyte weight sets, where CPU generation would take minutes).

Recipe (per workload):
  * x: f32 N(0, 1) -> bf16 (round to nearest even) -> E4M3 codes with one UE8M0
    scale per 1x128 block, the scale being the smallest power of two 2^n with
    block amax <= 448 * 2^n.
  * W1 [E, 2I, H], W2 [E, H, I]: f32 N(0, 0.02) -> E4M3 with one UE8M0 scale per
    128x128 block (same rule), or, for MXFP4, E2M1 codes packed two per byte (low
    nibble first) with one UE8M0 scale per 1x32 block (rule with 6 in place of 448).
  * routing: logits f32 N(0, 1) [T, E] -> softmax -> top-k (logit descending, ties
    to the lower expert id) -> the chosen probabilities renormalised to sum 1.
  * skewed ("zipf") routing: expert ranks 1..E drawn with probability proportional
    to r^-1.2, except that the last E/8 ranks get probability 0 so that some
    experts receive no token; ranks map to expert ids through a seeded
    permutation; each token draws k distinct experts one after another without
    replacement; weights are a softmax of N(0, 1) logits over the k chosen.
"""
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    w_dtype: str = "e4m3"          # "e4m3", "e2m1" or "bf16" (then x is bf16 too)
    routing: str = "gaussian"      # "gaussian" or "zipf"
    act: str = "swiglu"            # "swiglu" or "swiglu_oai"
    alpha: float = 1.0
    up_bias: float = 0.0
    limit: float = float("inf")
    cfg_id: int = 0

    @property
    def S(self):
        return self.T * self.k

    def with_tokens(self, T):
        d = dict(self.__dict__)
        d["T"] = T
        d["name"] = f"{self.name.split('@')[0]}@T={T}"
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 512, 256, 8, 2, cfg_id=0),
    "decode": Workload("decode", 128, 7168, 2048, 32, 8, routing="zipf", cfg_id=1),
    "prefill": Workload("prefill", 8192, 7168, 2048, 32, 8, cfg_id=2),
    "oai": Workload("oai", 2048, 3072, 1536, 64, 4, act="swiglu_oai",
                    alpha=1.702, up_bias=1.0, limit=7.0, cfg_id=3),
    "mxfp4": Workload("mxfp4", 128, 7168, 3072, 48, 6, w_dtype="e2m1", cfg_id=4),
    # The BF16 variant at the decode layer's shape and routing.
    "bf16": Workload("bf16", 128, 7168, 2048, 32, 8, w_dtype="bf16", routing="zipf", cfg_id=5),
}
MXFP4_TOKEN_SWEEP = (128, 512, 1024, 2048, 4096, 8192, 16384, 32768)

_E2M1_MAGS = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=torch.float32)


def _pow2_exponent(amax, fmax):
    """Smallest integer n with amax <= fmax * 2^n, elementwise (exact compare)."""
    a = torch.clamp(amax.to(torch.float64), min=1e-4)
    n = torch.ceil(torch.log2(a / fmax))
    n = torch.where(a > fmax * torch.exp2(n), n + 1, n)
    n = torch.where(a <= fmax * torch.exp2(n - 1), n - 1, n)
    return n


def _quant_e4m3_blocks(v, br, bc):
    """v [R, C] f32 -> (E4M3 codes u8 [R, C], UE8M0 bytes [R/br, C/bc])."""
    R, C = v.shape
    blk = v.reshape(R // br, br, C // bc, bc)
    amax = blk.abs().amax(dim=(1, 3))
    n = _pow2_exponent(amax, 448.0)
    scale = torch.exp2(-n).to(torch.float32)[:, None, :, None]
    q = (blk * scale).reshape(R, C).to(torch.float8_e4m3fn).view(torch.uint8)
    return q, (n + 127).to(torch.uint8)


def _quant_e2m1_rows(v):
    """v [R, C] f32 -> (E2M1 codes packed [R, C/2] u8, UE8M0 bytes [R, C/32])."""
    R, C = v.shape
    blk = v.reshape(R, C // 32, 32)
    n = _pow2_exponent(blk.abs().amax(dim=2), 6.0)
    s = (blk * torch.exp2(-n).to(torch.float32)[:, :, None]).reshape(R, C)
    mags = _E2M1_MAGS.to(v.device)
    a = s.abs().clamp(max=6.0)
    hi = torch.searchsorted(mags, a.contiguous()).clamp(max=7)
    lo = (hi - 1).clamp(min=0)
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = torch.where(pick_hi, hi, lo).to(torch.uint8)
    code = torch.where(torch.signbit(s), code | 8, code)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).to(torch.uint8)
    return packed, (n + 127).to(torch.uint8)


def _routing(wl, gen, device):
    T, E, k = wl.T, wl.E, wl.k
    if wl.routing == "gaussian":
        logits = torch.randn(T, E, generator=gen, device=device, dtype=torch.float32)
        probs = torch.softmax(logits, dim=1)
        order = torch.sort(-logits, dim=1, stable=True).indices[:, :k]
        w = torch.gather(probs, 1, order)
        w = w / w.sum(dim=1, keepdim=True)
        return order.to(torch.int32), w.to(torch.float32)
    if wl.routing == "zipf":
        ranks = torch.arange(1, E + 1, dtype=torch.float64, device=device)
        p = ranks ** -1.2
        p[E - E // 8:] = 0.0
        p = (p / p.sum()).to(torch.float32)
        rank_to_expert = torch.randperm(E, generator=gen, device=device)
        draws = torch.multinomial(p.expand(T, E).contiguous(), k, replacement=False,
                                  generator=gen)
        idx = rank_to_expert[draws]
        logits = torch.randn(T, k, generator=gen, device=device, dtype=torch.float32)
        w = torch.softmax(logits, dim=1)
        return idx.to(torch.int32), w.to(torch.float32)
    raise ValueError(wl.routing)


def make_weights(wl, device="cpu", seed=None):
    """W1/W2 codes and scales for a workload (shared by a token sweep)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 + wl.cfg_id if seed is None else seed)
    E, H, I = wl.E, wl.H, wl.I
    out = {}
    for name, (R, C) in (("w1", (2 * I, H)), ("w2", (H, I))):
        codes, scales = [], []
        for _ in range(E):
            v = torch.randn(R, C, generator=gen, device=device, dtype=torch.float32) * 0.02
            if wl.w_dtype == "e4m3":
                q, s = _quant_e4m3_blocks(v, 128, 128)
            elif wl.w_dtype == "e2m1":
                q, s = _quant_e2m1_rows(v)
            else:
                q, s = v.to(torch.bfloat16), None
            codes.append(q)
            scales.append(s)
        out[name] = torch.stack(codes)
        out[name + "_scales"] = None if scales[0] is None else torch.stack(scales)
    return out


def make_activations(wl, device="cpu", seed=None):
    """x codes/scales and routing for a workload."""
    gen = torch.Generator(device=device)
    gen.manual_seed((1000 + wl.cfg_id) * 7919 + wl.T if seed is None else seed)
    x = torch.randn(wl.T, wl.H, generator=gen, device=device, dtype=torch.float32)
    x = x.to(torch.bfloat16)
    if wl.w_dtype == "bf16":
        xq, xs = x, None
    else:
        xq, xs = _quant_e4m3_blocks(x.to(torch.float32), 1, 128)
    idx, w = _routing(wl, gen, device)
    return {"x": xq, "x_scales": xs, "topk_idx": idx, "topk_w": w}


def make_inputs(wl, device="cpu", seed=None):
    d = make_weights(wl, device, seed)
    d.update(make_activations(wl, device, None if seed is None else seed + 1))
    return d


def to_numpy(d):
    """Tensors -> numpy (bf16 as its uint16 bit patterns; None stays None)."""
    def conv(v):
        if v is None:
            return None
        if v.dtype == torch.bfloat16:
            return v.cpu().view(torch.int16).numpy().view("uint16")
        return v.cpu().numpy()
    return {k: conv(v) for k, v in d.items()}
