"""Python binding of the B200 fused MoE expert layer (libmoe_b200.so).

Argument marshalling only: every step of the layer runs in the CUDA library.
The functions carry the C ABI's names (include/moe.h) and accept either
integers (raw device/host addresses) or torch tensors (their data_ptr() is
passed).  Errors come back as MoEError carrying the moe_status code.

If the compiled library is missing this module raises ImportError when a
function is first called: there is no fallback implementation.
"""
import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_ALIGNMENT", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
                6: "MOE_ERR_BAD_ROUTING"}
W_DTYPES = {"e4m3": 0, "e2m1": 1, "bf16": 2}
ACT_KINDS = {"swiglu": 0, "swiglu_oai": 1}


class MoEError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class _Dtypes(ctypes.Structure):
    _fields_ = [("w_dtype", ctypes.c_int)]


class _Act(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("alpha", ctypes.c_float),
                ("up_bias", ctypes.c_float), ("limit", ctypes.c_float)]


class WorkspaceView(ctypes.Structure):
    _fields_ = [("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("inv", ctypes.c_void_p),
                ("pad_offsets", ctypes.c_void_p), ("act", ctypes.c_void_p),
                ("act_f32", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("error_word", ctypes.c_void_p), ("rows", ctypes.c_int64)]


_P = ctypes.c_void_p
_SIGS = {
    "moe_plan": (ctypes.c_int, [ctypes.c_int] * 5 + [_Dtypes, _Act, ctypes.POINTER(_P)]),
    "moe_plan_destroy": (None, [_P]),
    "moe_workspace_bytes": (ctypes.c_size_t, [_P]),
    "moe_forward": (ctypes.c_int, [_P] * 12),
    "moe_forward_hostio": (ctypes.c_int, [_P] * 12),
    "moe_forward_hostio_batches": (ctypes.c_int, [_P, ctypes.c_int] + [_P] * 11),
    "moe_route": (ctypes.c_int, [_P] * 4),
    "moe_route_gather": (ctypes.c_int, [_P] * 6),
    "moe_quantize_act": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P]),
    "moe_route_static": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int] + [_P] * 5),
    "moe_gather": (ctypes.c_int, [_P] * 5),
    "moe_fc1": (ctypes.c_int, [_P] * 5),
    "moe_fc2": (ctypes.c_int, [_P] * 5),
    "moe_fc1_fc2": (ctypes.c_int, [_P] * 7),
    "moe_combine": (ctypes.c_int, [_P] * 5),
    "moe_workspace_view": (ctypes.c_int, [_P, _P, ctypes.POINTER(WorkspaceView)]),
    "moe_copy_act_scales": (ctypes.c_int, [_P] * 4),
    "moe_plan_set_debug": (ctypes.c_int, [_P, ctypes.c_int]),
    "moe_plan_set_weight_layout": (ctypes.c_int, [_P, ctypes.c_int]),
    "moe_plan_set_cta_pairs": (ctypes.c_int, [_P, ctypes.c_int]),
    "moe_plan_cta_pairs_active": (ctypes.c_int, [_P]),
    "moe_plan_set_swap_ab": (ctypes.c_int, [_P, ctypes.c_int]),
    "moe_prepack_weight_scales": (ctypes.c_int, [_P] * 6),
    "moe_plan_swap_ab_active": (ctypes.c_int, [_P]),
    "moe_plan_set_wide_tiles": (ctypes.c_int, [_P, ctypes.c_int]),
    "moe_plan_wide_tiles_active": (ctypes.c_int, [_P]),
    "moe_prepack_weights": (ctypes.c_int, [_P] * 6),
    "moe_copy_act": (ctypes.c_int, [_P] * 4),
    "moe_clear_device_error": (ctypes.c_int, [_P] * 3),
    "moe_check_device_error": (ctypes.c_int, [_P] * 3),
    "moe_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_forward_launch_count": (ctypes.c_int, [_P]),
}

_lib = None


def lib():
    """The loaded CUDA library (ImportError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m moe_expert_ffn_permute_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(v):
    if v is None:
        return None
    if isinstance(v, int):
        return v
    if hasattr(v, "data_ptr"):
        return v.data_ptr()
    raise TypeError(f"expected an address or a tensor, got {type(v)}")


def _stream(s):
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:  # pragma: no cover
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status, what):
    if status != MOE_OK:
        raise MoEError(status, what)


def moe_plan(T, H, I, E, k, w_dtype="e4m3", act="swiglu", alpha=1.0, up_bias=0.0,
             limit=math.inf):
    """Build a plan (host object).  Returns an opaque handle."""
    h = _P()
    st = lib().moe_plan(T, H, I, E, k, _Dtypes(W_DTYPES[w_dtype]),
                        _Act(ACT_KINDS[act], alpha, up_bias, limit), ctypes.byref(h))
    _check(st, "moe_plan")
    return h.value


def moe_plan_destroy(plan):
    lib().moe_plan_destroy(plan)


def moe_workspace_bytes(plan):
    return lib().moe_workspace_bytes(plan)


def moe_plan_set_debug(plan, flags):
    """Bit 0 (or True): capture the fp32 FC1 activation; bit 1: the failure-path
    test hook (the fused launch's FC2 dependency wait runs out)."""
    _check(lib().moe_plan_set_debug(plan, int(flags)), "moe_plan_set_debug")


def moe_forward(plan, x, x_scales, topk_idx, topk_w, w1, w1_scales, w2, w2_scales, out,
                workspace, stream=None):
    _check(lib().moe_forward(plan, *map(_ptr, (x, x_scales, topk_idx, topk_w, w1, w1_scales,
                                               w2, w2_scales, out, workspace)),
                             _stream(stream)), "moe_forward")


def moe_forward_hostio(plan, x_host, x_scales_host, topk_idx_host, topk_w_host, w1, w1_scales,
                       w2, w2_scales, out_host, workspace, stream=None):
    _check(lib().moe_forward_hostio(plan, *map(_ptr, (x_host, x_scales_host, topk_idx_host,
                                                      topk_w_host, w1, w1_scales, w2, w2_scales,
                                                      out_host, workspace)),
                                    _stream(stream)), "moe_forward_hostio")


def _ptr_array(items):
    """A C array of addresses (void *[]) for a list of tensors / addresses;
    None if `items` is None."""
    if items is None:
        return None
    arr = (ctypes.c_void_p * len(items))(*[_ptr(v) for v in items])
    return ctypes.cast(arr, ctypes.c_void_p).value, arr


def moe_forward_hostio_batches(plan, x_host, x_scales_host, topk_idx_host, topk_w_host, w1,
                               w1_scales, w2, w2_scales, out_host, workspace, stream=None):
    """len(x_host) consecutive layers on host buffers (lists of pinned tensors or
    addresses, one entry per batch; x_scales_host None for BF16 plans), copies
    overlapped with the layers; outputs valid after the stream is synchronised."""
    n = len(x_host)
    for name, lst in (("x_scales_host", x_scales_host), ("topk_idx_host", topk_idx_host),
                      ("topk_w_host", topk_w_host), ("out_host", out_host)):
        if lst is not None and len(lst) != n:
            raise MoEError(MOE_ERR_INVALID_ARG,
                           f"moe_forward_hostio_batches: {name} has {len(lst)} entries, "
                           f"x_host has {n}")
    arrays = [_ptr_array(v) for v in (x_host, x_scales_host, topk_idx_host, topk_w_host)]
    outs = _ptr_array(out_host)
    keep = [a for a in arrays + [outs] if a is not None]   # alive until the call returns
    addr = [None if a is None else a[0] for a in arrays]
    _check(lib().moe_forward_hostio_batches(plan, n, addr[0], addr[1], addr[2], addr[3],
                                            *map(_ptr, (w1, w1_scales, w2, w2_scales)),
                                            None if outs is None else outs[0], _ptr(workspace),
                                            _stream(stream)), "moe_forward_hostio_batches")
    del keep


def moe_route(plan, topk_idx, workspace, stream=None):
    _check(lib().moe_route(plan, _ptr(topk_idx), _ptr(workspace), _stream(stream)), "moe_route")


def moe_quantize_act(x_bf16, T, H, x_codes, x_scales, stream=None):
    """bf16 [T,H] -> E4M3 codes [T,H] + UE8M0 scales [T,H/128] (device buffers)."""
    _check(lib().moe_quantize_act(_ptr(x_bf16), T, H, _ptr(x_codes), _ptr(x_scales),
                                  _stream(stream)), "moe_quantize_act")


def _expect_i32(name, t, numel):
    """A tensor argument of moe_route_static: contiguous int32 on a CUDA device
    with at least `numel` elements (the C ABI would otherwise write past its
    end or read host memory).  Raw addresses are passed through unchecked."""
    if t is None:
        raise MoEError(MOE_ERR_INVALID_ARG, f"moe_route_static: {name} is required")
    if isinstance(t, int):
        return
    import torch
    if t.dtype != torch.int32:
        raise MoEError(MOE_ERR_INVALID_ARG, f"moe_route_static: {name} must be int32, got {t.dtype}")
    if not t.is_contiguous():
        raise MoEError(MOE_ERR_INVALID_ARG, f"moe_route_static: {name} must be contiguous")
    if t.numel() < numel:
        raise MoEError(MOE_ERR_INVALID_ARG,
                       f"moe_route_static: {name} holds {t.numel()} elements, needs {numel}")


def moe_route_static(topk_idx, T, k, E, counts, offsets, perm, inv, stream=None):
    """Routing without a workspace: scratch lives in the library's static device
    memory (at most MOE_ROUTE_STATIC_MAX_SLOTS slots; calls must not overlap).
    Expert ids outside [0, E) other than -1 are dropped without an error status."""
    T, k, E = int(T), int(k), int(E)
    if T >= 1 and k >= 1 and E >= 1 and T * k <= ROUTE_STATIC_MAX_SLOTS and E <= 256:
        S = T * k
        args = (("topk_idx", topk_idx, S), ("counts", counts, E), ("offsets", offsets, E + 1),
                ("perm", perm, S), ("inv", inv, S))
        for name, t, n in args:
            _expect_i32(name, t, n)
        for name, t, _ in args:
            if not isinstance(t, int) and not t.is_cuda:
                raise MoEError(MOE_ERR_INVALID_ARG,
                               f"moe_route_static: {name} must be on a CUDA device")
    # Sizes out of range are refused by the library itself (nothing enqueued).
    _check(lib().moe_route_static(_ptr(topk_idx), T, k, E, *map(_ptr, (counts, offsets, perm,
                                                                         inv)),
                                  _stream(stream)), "moe_route_static")


ROUTE_STATIC_MAX_SLOTS = 1 << 20


def moe_gather(plan, x, x_scales, workspace, stream=None):
    _check(lib().moe_gather(plan, *map(_ptr, (x, x_scales, workspace)), _stream(stream)),
           "moe_gather")


def moe_route_gather(plan, topk_idx, x, x_scales, workspace, stream=None):
    """moe_route + moe_gather (one launch up to 4096 slots)."""
    _check(lib().moe_route_gather(plan, *map(_ptr, (topk_idx, x, x_scales, workspace)),
                                  _stream(stream)), "moe_route_gather")


def moe_fc1(plan, w1, w1_scales, workspace, stream=None):
    _check(lib().moe_fc1(plan, *map(_ptr, (w1, w1_scales, workspace)), _stream(stream)),
           "moe_fc1")


def moe_fc2(plan, w2, w2_scales, workspace, stream=None):
    _check(lib().moe_fc2(plan, *map(_ptr, (w2, w2_scales, workspace)), _stream(stream)),
           "moe_fc2")


def moe_fc1_fc2(plan, w1, w1_scales, w2, w2_scales, workspace, stream=None):
    _check(lib().moe_fc1_fc2(plan, *map(_ptr, (w1, w1_scales, w2, w2_scales, workspace)),
                             _stream(stream)), "moe_fc1_fc2")


def moe_combine(plan, topk_w, out, workspace, stream=None):
    _check(lib().moe_combine(plan, *map(_ptr, (topk_w, out, workspace)), _stream(stream)),
           "moe_combine")


def moe_workspace_view(plan, workspace):
    v = WorkspaceView()
    _check(lib().moe_workspace_view(plan, _ptr(workspace), ctypes.byref(v)), "moe_workspace_view")
    return v


def moe_copy_act_scales(plan, workspace, dst, stream=None):
    _check(lib().moe_copy_act_scales(plan, _ptr(workspace), _ptr(dst), _stream(stream)),
           "moe_copy_act_scales")


def moe_plan_set_weight_layout(plan, layout):
    """0 / False: row-major, 1 / True: tiled (FP8, BF16), 2: MXFP4 scales chunked,
    3: MXFP4 codes tiled and scales chunked."""
    _check(lib().moe_plan_set_weight_layout(plan, int(layout)), "moe_plan_set_weight_layout")


def moe_prepack_weight_scales(plan, w1_scales, w2_scales, w1s_chunked, w2s_chunked, stream=None):
    _check(lib().moe_prepack_weight_scales(plan, *map(_ptr, (w1_scales, w2_scales, w1s_chunked,
                                                              w2s_chunked)), _stream(stream)),
           "moe_prepack_weight_scales")


def moe_plan_set_cta_pairs(plan, mode):
    """0: automatic, 1: never, 2: always use the 2-SM GEMM."""
    _check(lib().moe_plan_set_cta_pairs(plan, int(mode)), "moe_plan_set_cta_pairs")


def moe_plan_cta_pairs_active(plan):
    return bool(lib().moe_plan_cta_pairs_active(plan))


def moe_plan_set_swap_ab(plan, mode):
    """0: automatic, 1: never, 2: always use token-major (swap-AB) GEMM tiles."""
    _check(lib().moe_plan_set_swap_ab(plan, int(mode)), "moe_plan_set_swap_ab")


def moe_plan_swap_ab_active(plan):
    """0: token-row tiles only, 1: token-major throughout, 2: tile by tile."""
    return int(lib().moe_plan_swap_ab_active(plan))


def moe_plan_set_wide_tiles(plan, mode):
    """0: automatic, 1: never, 2: always use wide token-major tiles (up to 240
    tokens of two m-tiles of one expert per tile)."""
    _check(lib().moe_plan_set_wide_tiles(plan, int(mode)), "moe_plan_set_wide_tiles")


def moe_plan_wide_tiles_active(plan):
    return bool(lib().moe_plan_wide_tiles_active(plan))


def moe_prepack_weights(plan, w1, w2, w1_tiled, w2_tiled, stream=None):
    _check(lib().moe_prepack_weights(plan, *map(_ptr, (w1, w2, w1_tiled, w2_tiled)),
                                     _stream(stream)), "moe_prepack_weights")


def moe_copy_act(plan, workspace, dst, stream=None):
    _check(lib().moe_copy_act(plan, _ptr(workspace), _ptr(dst), _stream(stream)), "moe_copy_act")


def moe_clear_device_error(plan, workspace, stream=None):
    _check(lib().moe_clear_device_error(plan, _ptr(workspace), _stream(stream)),
           "moe_clear_device_error")


def moe_check_device_error(plan, workspace, stream=None):
    """Synchronises the stream; returns the moe_status code (0 = no device error)."""
    return lib().moe_check_device_error(plan, _ptr(workspace), _stream(stream))


def moe_status_str(status):
    return lib().moe_status_str(status).decode()


def moe_forward_launch_count(plan):
    return lib().moe_forward_launch_count(plan)


def _expect(name, t, shape, dtype, device):
    import torch
    if t is None:
        raise MoEError(MOE_ERR_INVALID_ARG, f"{name} is required")
    if not isinstance(t, torch.Tensor):
        return                      # a raw address: the caller vouches for it
    if (tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous()
            or t.device != device):
        raise MoEError(MOE_ERR_INVALID_ARG,
                       f"{name}: expected a contiguous {dtype} tensor of shape {tuple(shape)} on "
                       f"{device}, got {t.dtype} {tuple(t.shape)} on {t.device}"
                       f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def check_layer_args(T, H, I, E, k, w_dtype, device, x, x_scales, topk_idx, topk_w, w1,
                     w1_scales, w2, w2_scales, out):
    """Shapes, dtypes, contiguity and device of moe_forward's tensors for a plan
    (T, H, I, E, k, w_dtype), as include/moe.h lays them out.  The C ABI sees
    only pointers, so a wrong-sized tensor would be read past its end; this
    check catches that before the call.  Tiled weights and chunked scales have
    the shapes of the row-major ones.  Raises MoEError(MOE_ERR_INVALID_ARG)."""
    import torch
    u8, bf16 = torch.uint8, torch.bfloat16
    if w_dtype == "bf16":
        _expect("x", x, (T, H), bf16, device)
        _expect("w1", w1, (E, 2 * I, H), bf16, device)
        _expect("w2", w2, (E, H, I), bf16, device)
    else:
        _expect("x", x, (T, H), u8, device)
        _expect("x_scales", x_scales, (T, H // 128), u8, device)
        if w_dtype == "e4m3":
            shapes = ((E, 2 * I, H), (E, 2 * I // 128, H // 128), (E, H, I), (E, H // 128, I // 128))
        else:
            shapes = ((E, 2 * I, H // 2), (E, 2 * I, H // 32), (E, H, I // 2), (E, H, I // 32))
        for name, t, shape in zip(("w1", "w1_scales", "w2", "w2_scales"),
                                  (w1, w1_scales, w2, w2_scales), shapes):
            _expect(name, t, shape, u8, device)
    _expect("topk_idx", topk_idx, (T, k), torch.int32, device)
    _expect("topk_w", topk_w, (T, k), torch.float32, device)
    _expect("out", out, (T, H), bf16, device)


class MoELayer:
    """Convenience owner of a plan and its torch-allocated workspace."""

    def __init__(self, T, H, I, E, k, w_dtype="e4m3", act="swiglu", alpha=1.0, up_bias=0.0,
                 limit=math.inf, device="cuda", debug=False, tiled_weights=False,
                 cta_pairs=None, swap_ab=None, chunked_scales=False, wide_tiles=None):
        import torch
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        self.w_dtype = w_dtype
        self.plan = moe_plan(T, H, I, E, k, w_dtype, act, alpha, up_bias, limit)
        if w_dtype == "e2m1" and tiled_weights:
            # MXFP4: tiled codes come with chunked scales (one layout value).
            if not chunked_scales:
                raise MoEError(MOE_ERR_INVALID_ARG, "tiled MXFP4 codes need chunked_scales=True")
            moe_plan_set_weight_layout(self.plan, 3)
        elif tiled_weights:
            moe_plan_set_weight_layout(self.plan, 1)
        elif chunked_scales:
            moe_plan_set_weight_layout(self.plan, 2)
        if cta_pairs is not None:
            moe_plan_set_cta_pairs(self.plan, cta_pairs)
        if swap_ab is not None:
            moe_plan_set_swap_ab(self.plan, swap_ab)
        if wide_tiles is not None:
            moe_plan_set_wide_tiles(self.plan, wide_tiles)
        if debug:
            moe_plan_set_debug(self.plan, True)
        nbytes = moe_workspace_bytes(self.plan)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        moe_clear_device_error(self.plan, self.workspace)

    def forward(self, x, x_scales, topk_idx, topk_w, w1, w1_scales, w2, w2_scales, out=None,
                stream=None):
        import torch
        if out is None:
            out = torch.empty(self.T, self.H, dtype=torch.bfloat16, device=self.workspace.device)
        check_layer_args(self.T, self.H, self.I, self.E, self.k, self.w_dtype,
                         self.workspace.device, x, x_scales, topk_idx, topk_w, w1, w1_scales,
                         w2, w2_scales, out)
        moe_forward(self.plan, x, x_scales, topk_idx, topk_w, w1, w1_scales, w2, w2_scales, out,
                    self.workspace, stream)
        return out

    def prepack(self, w1, w2):
        """Tiled copies of row-major weights (FP8 / BF16: 16 KB pre-swizzled
        tiles; MXFP4 codes: 8 KB tiles) for a plan with tiled_weights."""
        import torch
        w1t, w2t = torch.empty_like(w1), torch.empty_like(w2)
        moe_prepack_weights(self.plan, w1, w2, w1t, w2t)
        return w1t, w2t

    def prepack_scales(self, w1_scales, w2_scales):
        """Chunked copies of MXFP4 weight scales for a plan with chunked_scales."""
        import torch
        a, b = torch.empty_like(w1_scales), torch.empty_like(w2_scales)
        moe_prepack_weight_scales(self.plan, w1_scales, w2_scales, a, b)
        return a, b

    def view(self):
        return moe_workspace_view(self.plan, self.workspace)

    def check(self, stream=None):
        return moe_check_device_error(self.plan, self.workspace, stream)

    def __del__(self):
        try:
            if getattr(self, "plan", None):
                moe_plan_destroy(self.plan)
                self.plan = None
        except Exception:
            pass
