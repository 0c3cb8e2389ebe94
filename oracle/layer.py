"""Float64 CPU statement of the fused MoE expert layer: TEST INFRASTRUCTURE ONLY.

What the layer computes, for every token t with top-k experts topk_idx[t, j] and
weights topk_w[t, j] (j = 0..k-1):

  xh[t]    = E4M3(x[t]) * UE8M0(x_scales[t, c // 128])           1x128 blocks
  h        = xh[t] @ W1h[e].T        e = topk_idx[t, j]; W1h[e] is [2I, H]
  g, u     = h[:I], h[I:]            gate rows first, then up rows
  a        = min(g, L) * sigmoid(alpha * min(g, L)) * (clip(u, -L, L) + beta)
  q, sf    = requant(a)              E4M3 codes + UE8M0 per 1x128 block of a
  y[t, j]  = (E4M3(q) * UE8M0(sf)) @ W2h[e].T      W2h[e] is [H, I]
  out[t]   = sum_j topk_w[t, j] * y[t, j]

Sources, by page and section:
  * Grouping tokens by expert (histogram, exclusive scan, stable scatter) and the
    "direct combine" back to token order: DeepGEMM PR #386 "Optimize sm100
    version with token-aware BM240 tiling, native UE8M0, and direct combine",
    title and Description (tokens per rank, direct-combine path).
  * The activation: DeepGEMM PR #445 "fix(sm90): support parameterized SwiGLU in
    FP8 MegaMoE", Summary (gate clamped from above at limit, up clamped to
    [-limit, limit], gate * sigmoid(alpha * gate) * (up + up_bias)) and
    Compatibility (alpha = 1, up_bias = 0 is standard SwiGLU SiLU(gate) * up).
  * FP8 E4M3 weights/activations with block scales: DeepGEMM PR #445
    "Environment" (weight format FP8 E4M3); UE8M0 scales: DeepGEMM PR #386 title
    ("native UE8M0"); MXFP4 (E2M1) weights: the FP8/FP4 MegaMoE named in fw-ai
    DeepGEMM PR #16 "Overview".
  * The requantisation of the activation to FP8 with one UE8M0 scale per 1x128
    block, chosen from the block's amax: TensorRT-LLM PR #16346 "Description"
    (fused BF16 -> FP8 + 1x128 UE8M0 quantisation with an amax reduction).

Readings where the pages are silent (each listed in the design notes):
  * gate = rows [0, I) of W1[e], up = rows [I, 2I) (non-interleaved).
  * no clamp (L = +inf) for standard SwiGLU.
  * requant scale = the smallest power of two 2^n with max(amax, 1e-4) <= 448 * 2^n;
    codes = round-to-nearest-even, saturating, E4M3 of a / 2^n.
  * topk_w is applied after FC2, in the combine.
  * E2M1 packing: element 2i in the low nibble of byte i.
  * out-of-range expert ids are not routed: their slots are skipped.

Parity: every function here is pinned by tests that do not call it back with its
own formula (exhaustive codec tables, brute-force loops on tiny inputs,
integer-exact GEMMs, closed-form activation special cases, requant boundary
cases, routing invariants).  The whole-layer values have no worked example on
the pages; the layer is pinned through those parts and through an independent
element-by-element brute-force tier (``layer_bruteforce``).
"""
import math

import numpy as np

from .formats import (E4M3_MAX, decode_bf16, decode_e2m1, decode_e4m3, decode_ue8m0,
                      encode_bf16_rne, encode_e4m3_rne_satfinite, unpack_e2m1_pairs)

BLOCK = 128          # activation / FP8-weight scale block along K (and N for weights)
FP4_BLOCK = 32       # MXFP4 weight scale block along K
AMAX_FLOOR = 1e-4    # floor on the requant block amax (reading; the pages are silent)


# --------------------------------------------------------------------------- routing
def route(topk_idx, num_experts):
    """Group the T*k routing slots by expert.

    Slot s = t*k + j holds expert topk_idx[t, j].  Returns
      counts  [E]    number of slots routed to each expert
      offsets [E+1]  exclusive prefix sum of counts
      perm    [S]    position p -> slot s; positions offsets[e] .. offsets[e+1]-1
                     hold expert e's slots in ascending slot order (stable);
                     positions past offsets[E] are -1
      inv     [S]    slot s -> position p, -1 for a slot whose expert id is out
                     of range (not routed)
    """
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    S = flat.shape[0]
    valid = (flat >= 0) & (flat < num_experts)
    counts = np.zeros(num_experts, dtype=np.int64)
    for e in range(num_experts):
        counts[e] = np.count_nonzero(flat == e)
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.full(S, -1, dtype=np.int64)
    inv = np.full(S, -1, dtype=np.int64)
    for e in range(num_experts):
        slots = np.nonzero(flat == e)[0]           # ascending slot order
        pos = offsets[e] + np.arange(slots.shape[0])
        perm[pos] = slots
        inv[slots] = pos
    assert np.count_nonzero(valid) == offsets[-1]
    return counts, offsets, perm, inv


# ----------------------------------------------------------------------- dequantise
# The decoders evaluated once for every code; indexing these tables is the same
# function as calling them element by element.
_E4M3 = decode_e4m3(np.arange(256, dtype=np.uint8))
_UE8M0 = decode_ue8m0(np.arange(256, dtype=np.uint8))
_E2M1 = decode_e2m1(np.arange(16))


def dequant_act(codes, scales):
    """E4M3 codes [R, C] with one UE8M0 scale per 1x128 block [R, C/128] -> f64."""
    v = _E4M3[np.asarray(codes, dtype=np.uint8)]
    s = _UE8M0[np.asarray(scales, dtype=np.uint8)]
    return v * np.repeat(s, BLOCK, axis=1)


def dequant_w_fp8(codes, scales):
    """E4M3 weight codes [R, C] with UE8M0 scales per 128x128 block
    [R/128, C/128] -> f64."""
    v = _E4M3[np.asarray(codes, dtype=np.uint8)]
    s = _UE8M0[np.asarray(scales, dtype=np.uint8)]
    s = np.repeat(np.repeat(s, BLOCK, axis=0), BLOCK, axis=1)
    return v * s


def dequant_w_fp4(packed, scales):
    """E2M1 weights packed two per byte [R, C/2] with UE8M0 scales per 1x32 block
    [R, C/32] -> f64."""
    v = _E2M1[unpack_e2m1_pairs(packed)]
    s = _UE8M0[np.asarray(scales, dtype=np.uint8)]
    return v * np.repeat(s, FP4_BLOCK, axis=1)


def dequant_weight(codes, scales, w_dtype):
    if w_dtype == "e4m3":
        return dequant_w_fp8(codes, scales)
    if w_dtype == "e2m1":
        return dequant_w_fp4(codes, scales)
    raise ValueError(w_dtype)


# ------------------------------------------------------------------------ activation
def sigmoid(z):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def swiglu(g, u, alpha=1.0, up_bias=0.0, limit=math.inf):
    """Parameterised (OAI) SwiGLU; alpha=1, up_bias=0, limit=inf is SiLU(g)*u."""
    gc = np.minimum(g, limit)
    uc = np.clip(u, -limit, limit)
    return gc * sigmoid(alpha * gc) * (uc + up_bias)


# --------------------------------------------------------------------------- requant
def ue8m0_exponent_for(amax):
    """Smallest integer n with max(amax, 1e-4) <= 448 * 2^n (exact comparison)."""
    a = max(float(amax), AMAX_FLOOR)
    n = math.ceil(math.log2(a / E4M3_MAX))
    while a > E4M3_MAX * 2.0 ** n:          # repair log2 rounding, both ways
        n += 1
    while a <= E4M3_MAX * 2.0 ** (n - 1):
        n -= 1
    return n


def requant_1x128(a):
    """Activation [R, C] -> (E4M3 codes [R, C], UE8M0 scale bytes [R, C/128])."""
    a = np.asarray(a, dtype=np.float64)
    R, C = a.shape
    codes = np.zeros((R, C), dtype=np.uint8)
    sf = np.zeros((R, C // BLOCK), dtype=np.uint8)
    for r in range(R):
        for b in range(C // BLOCK):
            blk = a[r, b * BLOCK:(b + 1) * BLOCK]
            n = ue8m0_exponent_for(np.max(np.abs(blk)))
            if n + 127 > 254:
                # UE8M0 scales stop at 2^127 (byte 254; 255 is NaN).  Any binary32
                # activation fits (n <= 120); larger float64 blocks have no encoding.
                raise ValueError(f"block amax {np.max(np.abs(blk))!r} exceeds 448 * 2^127")
            sf[r, b] = n + 127
            codes[r, b * BLOCK:(b + 1) * BLOCK] = encode_e4m3_rne_satfinite(blk / 2.0 ** n)
    return codes, sf


# ----------------------------------------------------------------------------- layer
def layer(x, x_scales, topk_idx, topk_w, w1, w1_scales, w2, w2_scales,
          w_dtype="e4m3", alpha=1.0, up_bias=0.0, limit=math.inf, keep=False):
    """The whole layer in float64.  Shapes: x [T,H] u8, x_scales [T,H/128] u8,
    topk_idx [T,k] int, topk_w [T,k] float, w1 [E,2I,H] (e4m3) or [E,2I,H/2]
    (e2m1 packed), w1_scales [E,2I/128,H/128] (e4m3) or [E,2I,H/32] (e2m1),
    w2 / w2_scales likewise with [E,H,I].  Returns out [T,H] float64 (and the
    intermediates when keep=True)."""
    T, k = np.asarray(topk_idx).shape
    E = w1.shape[0]
    H = x.shape[1]
    I = w2.shape[2] * (2 if w_dtype == "e2m1" else 1)
    counts, offsets, perm, inv = route(topk_idx, E)
    xh = dequant_act(x, x_scales)
    S = T * k
    y = np.zeros((S, H), dtype=np.float64)
    inter = {"h": {}, "a": {}, "q": {}, "sf": {}}
    for e in range(E):
        slots = perm[offsets[e]:offsets[e + 1]]
        if slots.shape[0] == 0:
            continue
        tokens = slots // k
        W1 = dequant_weight(w1[e], w1_scales[e], w_dtype)      # [2I, H]
        h = xh[tokens] @ W1.T                                    # [n_e, 2I]
        a = swiglu(h[:, :I], h[:, I:], alpha, up_bias, limit)   # [n_e, I]
        q, sf = requant_1x128(a)
        ah = dequant_act(q, sf)
        W2 = dequant_weight(w2[e], w2_scales[e], w_dtype)       # [H, I]
        y[slots] = ah @ W2.T                                     # [n_e, H]
        if keep:
            inter["h"][e], inter["a"][e], inter["q"][e], inter["sf"][e] = h, a, q, sf
    w = np.asarray(topk_w, dtype=np.float64)
    out = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            if inv[t * k + j] >= 0:
                out[t] += w[t, j] * y[t * k + j]
    if keep:
        inter.update(counts=counts, offsets=offsets, perm=perm, inv=inv, y=y)
        return out, inter
    return out


def layer_bf16(x, topk_idx, topk_w, w1, w2, alpha=1.0, up_bias=0.0, limit=math.inf,
               keep=False):
    """The BF16 variant of the layer (fw-ai/DeepGEMM PR #16 "Overview": BF16 and
    FP8/FP4 Mega MoE share the scheduler) in float64: x [T,H], w1 [E,2I,H] and
    w2 [E,H,I] are BF16 bit patterns (uint16), no block scales.  Reading (the
    pages name the variant only): the activation a goes to FC2 as BF16 (round to
    nearest even) instead of FP8 + 1x128 scales; everything else as in layer()."""
    T, k = np.asarray(topk_idx).shape
    E = w1.shape[0]
    H = x.shape[1]
    I = w2.shape[2]
    counts, offsets, perm, inv = route(topk_idx, E)
    xh = decode_bf16(x)
    S = T * k
    y = np.zeros((S, H), dtype=np.float64)
    inter = {"h": {}, "a": {}, "ab": {}}
    for e in range(E):
        slots = perm[offsets[e]:offsets[e + 1]]
        if slots.shape[0] == 0:
            continue
        tokens = slots // k
        h = xh[tokens] @ decode_bf16(w1[e]).T                   # [n_e, 2I]
        a = swiglu(h[:, :I], h[:, I:], alpha, up_bias, limit)   # [n_e, I]
        ab = encode_bf16_rne(a)
        y[slots] = decode_bf16(ab) @ decode_bf16(w2[e]).T        # [n_e, H]
        if keep:
            inter["h"][e], inter["a"][e], inter["ab"][e] = h, a, ab
    w = np.asarray(topk_w, dtype=np.float64)
    out = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            if inv[t * k + j] >= 0:
                out[t] += w[t, j] * y[t * k + j]
    if keep:
        inter.update(counts=counts, offsets=offsets, perm=perm, inv=inv, y=y)
        return out, inter
    return out


# ------------------------------------------------------------- brute-force tier (tiny)
def _e4m3_scalar(b):
    s = -1.0 if b & 0x80 else 1.0
    e = (b >> 3) & 0xF
    m = b & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * m / 8.0 * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def _e2m1_scalar(n):
    mag = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0][n & 7]
    return -mag if n & 8 else mag


def _w_scalar(w, ws, e, r, c, w_dtype):
    if w_dtype == "e4m3":
        return _e4m3_scalar(int(w[e, r, c])) * 2.0 ** (int(ws[e, r // 128, c // 128]) - 127)
    byte = int(w[e, r, c // 2])
    nib = byte & 0xF if c % 2 == 0 else byte >> 4
    return _e2m1_scalar(nib) * 2.0 ** (int(ws[e, r, c // 32]) - 127)


def layer_bruteforce(x, x_scales, topk_idx, topk_w, w1, w1_scales, w2, w2_scales,
                     w_dtype="e4m3", alpha=1.0, up_bias=0.0, limit=math.inf):
    """Element-by-element pure-Python loops over (t, j): no routing, no matmul
    library, no vectorised codecs.  For tiny shapes only."""
    T, k = np.asarray(topk_idx).shape
    H = x.shape[1]
    I = w2.shape[2] * (2 if w_dtype == "e2m1" else 1)
    E = w1.shape[0]
    out = [[0.0] * H for _ in range(T)]
    for t in range(T):
        xh = [_e4m3_scalar(int(x[t, c])) * 2.0 ** (int(x_scales[t, c // 128]) - 127)
              for c in range(H)]
        for j in range(k):
            e = int(topk_idx[t, j])
            if e < 0 or e >= E:
                continue
            a = []
            for i in range(I):
                g = sum(xh[c] * _w_scalar(w1, w1_scales, e, i, c, w_dtype) for c in range(H))
                u = sum(xh[c] * _w_scalar(w1, w1_scales, e, I + i, c, w_dtype) for c in range(H))
                gc = min(g, limit)
                uc = max(-limit, min(u, limit))
                a.append(gc / (1.0 + math.exp(-alpha * gc)) * (uc + up_bias)
                         if -alpha * gc < 700 else 0.0)
            ah = []
            for b in range(I // 128):
                blk = a[b * 128:(b + 1) * 128]
                amax = max(max(abs(v) for v in blk), AMAX_FLOOR)
                n = 0
                while amax > 448.0 * 2.0 ** n:
                    n += 1
                while amax <= 448.0 * 2.0 ** (n - 1):
                    n -= 1
                for v in blk:
                    ah.append(_rne_e4m3_scalar(v / 2.0 ** n) * 2.0 ** n)
            for c in range(H):
                yc = sum(ah[i] * _w_scalar(w2, w2_scales, e, c, i, w_dtype) for i in range(I))
                out[t][c] += float(topk_w[t, j]) * yc
    return np.array(out)


def _rne_e4m3_scalar(v):
    """Nearest E4M3 value to v (ties to even mantissa), saturating at 448,
    by scanning every finite non-negative code."""
    a = min(abs(v), 448.0)
    best, best_code = None, None
    for code in range(0x7F):
        m = _e4m3_scalar(code)
        d = abs(m - a)
        if best is None or d < best or (d == best and code % 2 == 0):
            best, best_code = d, code
    r = _e4m3_scalar(best_code)
    return -r if v < 0 else r


def _bf16_scalar(bits):
    """BF16 pattern -> float via the binary32 bytes (struct, not numpy)."""
    import struct
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def _rne_bf16_scalar(v):
    """Nearest BF16 value to v, ties to even mantissa, past the top -> inf:
    Python's round() (half to even) on v scaled by the spacing at v."""
    if v == 0.0 or math.isinf(v) or math.isnan(v):
        return v
    m, ex = math.frexp(abs(v))            # |v| = m * 2^ex, m in [0.5, 1)
    e = max(ex - 1, -126)
    r = round(abs(v) / 2.0 ** (e - 7)) * 2.0 ** (e - 7)
    if r > (2.0 - 2.0 ** -7) * 2.0 ** 127:
        r = math.inf
    return -r if v < 0 else r


def layer_bf16_bruteforce(x, topk_idx, topk_w, w1, w2, alpha=1.0, up_bias=0.0,
                          limit=math.inf):
    """Element-by-element pure-Python statement of layer_bf16 (tiny shapes)."""
    T, k = np.asarray(topk_idx).shape
    H = x.shape[1]
    I = w2.shape[2]
    E = w1.shape[0]
    out = [[0.0] * H for _ in range(T)]
    for t in range(T):
        xh = [_bf16_scalar(x[t, c]) for c in range(H)]
        for j in range(k):
            e = int(topk_idx[t, j])
            if e < 0 or e >= E:
                continue
            ab = []
            for i in range(I):
                g = sum(xh[c] * _bf16_scalar(w1[e, i, c]) for c in range(H))
                u = sum(xh[c] * _bf16_scalar(w1[e, I + i, c]) for c in range(H))
                gc = min(g, limit)
                uc = max(-limit, min(u, limit))
                a = (gc / (1.0 + math.exp(-alpha * gc)) * (uc + up_bias)
                     if -alpha * gc < 700 else 0.0)
                ab.append(_rne_bf16_scalar(a))
            for c in range(H):
                yc = sum(ab[i] * _bf16_scalar(w2[e, c, i]) for i in range(I))
                out[t][c] += float(topk_w[t, j]) * yc
    return np.array(out)
