"""Python binding of the B200 routed-expert MoE layer (libmoe_b200.so).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (bf16 as torch.bfloat16);
calls are enqueued on torch's current CUDA stream.  The C ABI and its
conventions are documented in include/moe.h.

There is no fallback: if the shared library is missing or the device is not
an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

__all__ = [
    "MoEError", "lib", "TILES_AUTO", "TILES_SMALL", "TILES_LARGE", "TILES_PAIR", "TILES_PERSISTENT",
    "ROUTER_AUTO", "ROUTER_FMA", "ROUTER_TC", "ROUTER_SMALL",
    "SCORE_SOFTMAX", "SCORE_SOFTMAX_SELECT_BIAS", "SCORE_SIGMOID",
    "COMBINE_AUTO", "COMBINE_FUSED", "COMBINE_SEPARATE",
    "workspace_size", "workspace_layout", "alloc_workspace", "route", "permute", "grouped_swiglu",
    "grouped_down", "down_combine", "forward", "forward_mx", "device_status", "clear_device_status", "selftest_timeout",
    "STATUS",
]

TILES_AUTO, TILES_SMALL, TILES_LARGE, TILES_PAIR, TILES_PERSISTENT = 0, 1, 2, 3, 4
ROUTER_AUTO, ROUTER_FMA, ROUTER_TC, ROUTER_SMALL = 0, 1, 2, 3
SCORE_SOFTMAX, SCORE_SOFTMAX_SELECT_BIAS, SCORE_SIGMOID = 0, 1, 2
COMBINE_AUTO, COMBINE_FUSED, COMBINE_SEPARATE = 0, 1, 2

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_ALIGNMENT", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT", 6: "MOE_ERR_UNSUPPORTED_ARCH",
          7: "MOE_ERR_DEVICE_BOUNDS"}


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().moe_status_string(status).decode()}")


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "status", "topk_ids", "topk_w", "counts", "offsets", "sorted_token_ids", "inv_perm",
        "h", "o", "h_shared", "o_shared", "logits", "router_split", "block_hist", "split", "arrivals",
        "total")]


class _Options(ctypes.Structure):
    _fields_ = [("tile_policy", ctypes.c_int), ("router_impl", ctypes.c_int),
                ("stage_events", ctypes.c_void_p * 7), ("launches", ctypes.c_int), ("scoring", ctypes.c_int),
                ("combine", ctypes.c_int), ("reserved", ctypes.c_int * 3)]


_P, _I, _Z, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
_SIGS = {
    "moe_status_string": ([_I], ctypes.c_char_p),
    "moe_abi_version": ([], _I),
    "moe_workspace_layout": ([_I] * 6 + [ctypes.POINTER(_Layout)], _I),
    "moe_workspace_size": ([_I] * 6 + [ctypes.POINTER(ctypes.c_size_t)], _I),
    "moe_get_device_status": ([_P, _P, ctypes.POINTER(ctypes.c_int32)], _I),
    "moe_clear_device_status": ([_P, _P], _I),
    "moe_route": ([_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _Z, _P], _I),
    "moe_route_ex": ([_P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _Z, _P], _I),
    "moe_route_scored": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _Z, _P], _I),
    "moe_permute": ([_P, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P], _I),
    "moe_grouped_swiglu": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P], _I),
    "moe_grouped_down": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _Z, _P], _I),
    "moe_down_combine": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P], _I),
    "moe_forward": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P], _I),
    "moe_forward_ex": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z,
                        ctypes.POINTER(_Options), _P], _I),
    "moe_forward_mx": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z,
                        ctypes.POINTER(_Options), _P], _I),
    "moe_selftest_timeout": ([_P, _Z, _U64, _P], _I),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises if it was never built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(_build.LIB_PATH):
            raise ImportError(f"{_build.LIB_PATH} is missing; build it with "
                              "routed_expert_ffn_prefix_b200.build.build()")
        handle = ctypes.CDLL(_build.LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes, fn.restype = args, res
        _LIB = handle
    return _LIB


def _check(status: int, what: str) -> None:
    if status != 0:
        raise MoEError(status, what)


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dims(t, ndim, name):
    """The shape of a tensor argument after checking its rank."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return tuple(t.shape)


def _check_args(specs, ws=None):
    """Checks every tensor argument before anything reaches the library: the
    library sees raw pointers and sizes only, so a tensor of the wrong shape,
    dtype or device would be read or written out of bounds.  specs: (tensor
    or None, dtype, name, shape with None for any size).  All shapes and
    dtypes are checked first, then that every tensor (and the workspace ws)
    is a CUDA tensor on one device."""
    import torch
    live = []
    for t, dtype, name, shape in specs:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if shape is not None:
            if t.dim() != len(shape) or any(w is not None and w != g for w, g in zip(shape, t.shape)):
                want = "[" + ", ".join("*" if w is None else str(w) for w in shape) + "]"
                raise ValueError(f"{name} must have shape {want}, got {list(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        live.append((t, name))
    if ws is not None:
        if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous():
            raise TypeError("the workspace must be a contiguous 1-D uint8 tensor (alloc_workspace)")
        live.append((ws, "workspace"))
    device = None
    for t, name in live:
        if not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if device is None:
            device = t.device
        elif t.device != device:
            raise ValueError(f"{name} is on {t.device}, the other arguments on {device}")


def workspace_layout(T, H, E, I, k, I_s=0) -> dict:
    L = _Layout()
    _check(lib().moe_workspace_layout(T, H, E, I, k, I_s, ctypes.byref(L)), "moe_workspace_layout")
    return {n: getattr(L, n) for n, _ in _Layout._fields_}


def workspace_size(T, H, E, I, k, I_s=0) -> int:
    n = ctypes.c_size_t()
    _check(lib().moe_workspace_size(T, H, E, I, k, I_s, ctypes.byref(n)), "moe_workspace_size")
    return n.value


def alloc_workspace(T, H, E, I, k, I_s=0, device="cuda"):
    """Device workspace for the layer shapes, status word cleared."""
    import torch
    ws = torch.empty(workspace_size(T, H, E, I, k, I_s), dtype=torch.uint8, device=device)
    clear_device_status(ws)
    return ws


def device_status(ws) -> int:
    _check_args([], ws)
    out = ctypes.c_int32()
    _check(lib().moe_get_device_status(_ptr(ws), _stream(), ctypes.byref(out)), "moe_get_device_status")
    return out.value


def clear_device_status(ws) -> None:
    _check_args([], ws)
    _check(lib().moe_clear_device_status(_ptr(ws), _stream()), "moe_clear_device_status")


def route(x, w_router, bias, k, ws, impl=ROUTER_AUTO, out=None, scoring=SCORE_SOFTMAX):
    """topk_ids [T,k] int32, topk_w [T,k] float32 (scoring: SCORE_*)."""
    import torch
    T, H = _dims(x, 2, "x")
    E = _dims(w_router, 2, "w_router")[1]
    ids, w = out if out is not None else (None, None)
    _check_args([(x, torch.bfloat16, "x", (T, H)), (w_router, torch.float32, "w_router", (H, E)),
                 (bias, torch.float32, "bias", (E,)), (ids, torch.int32, "topk_ids", (T, k)),
                 (w, torch.float32, "topk_w", (T, k))], ws)
    if out is None:
        ids = torch.empty(T, k, dtype=torch.int32, device=x.device)
        w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    _check(lib().moe_route_scored(_ptr(x), _ptr(w_router), _ptr(bias), T, H, E, k, scoring, _ptr(ids), _ptr(w),
                                  impl, _ptr(ws), ws.numel(), _stream()), "moe_route")
    return ids, w


def permute(topk_ids, E, ws):
    """counts [E], offsets [E+1], sorted_token_ids [T*k], inv_perm [T,k] (int32)."""
    import torch
    T, k = _dims(topk_ids, 2, "topk_ids")
    _check_args([(topk_ids, torch.int32, "topk_ids", (T, k))], ws)
    dev = topk_ids.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sids = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T, k, dtype=torch.int32, device=dev)
    _check(lib().moe_permute(_ptr(topk_ids), T, E, k, _ptr(counts), _ptr(offsets), _ptr(sids), _ptr(inv),
                             _ptr(ws), ws.numel(), _stream()), "moe_permute")
    return counts, offsets, sids, inv


def grouped_swiglu(x, w_gate_up, offsets, sorted_token_ids, k, ws, tiles=TILES_AUTO, out=None):
    """h [T*k, I] bf16 in permuted order."""
    import torch
    T, H = _dims(x, 2, "x")
    E, _, I2 = _dims(w_gate_up, 3, "w_gate_up")
    I = I2 // 2
    _check_args([(x, torch.bfloat16, "x", (T, H)), (w_gate_up, torch.bfloat16, "w_gate_up", (E, H, 2 * I)),
                 (offsets, torch.int32, "offsets", (E + 1,)),
                 (sorted_token_ids, torch.int32, "sorted_token_ids", (T * k,)),
                 (out, torch.bfloat16, "out", (T * k, I))], ws)
    if offsets is None or sorted_token_ids is None:
        raise TypeError("offsets and sorted_token_ids are required")
    h = out if out is not None else torch.empty(T * k, I, dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_grouped_swiglu(_ptr(x), _ptr(w_gate_up), _ptr(offsets), _ptr(sorted_token_ids), T, H, E, I, k,
                                    tiles, _ptr(h), _ptr(ws), ws.numel(), _stream()), "moe_grouped_swiglu")
    return h


def grouped_down(h, w_down, offsets, ws, tiles=TILES_AUTO, out=None):
    """o [rows, H] float32 = h . W_down[e] per group (offsets None: one group)."""
    import torch
    rows, I = _dims(h, 2, "h")
    E, _, H = _dims(w_down, 3, "w_down")
    _check_args([(h, torch.bfloat16, "h", (rows, I)), (w_down, torch.bfloat16, "w_down", (E, I, H)),
                 (offsets, torch.int32, "offsets", (E + 1,)), (out, torch.float32, "out", (rows, H))], ws)
    o = out if out is not None else torch.empty(rows, H, dtype=torch.float32, device=h.device)
    _check(lib().moe_grouped_down(_ptr(h), _ptr(w_down), _ptr(offsets), rows, H, E, I, tiles, _ptr(o),
                                  _ptr(ws), ws.numel(), _stream()), "moe_grouped_down")
    return o


def down_combine(h, w_down, topk_w, inv_perm, offsets, shared_out, ws, tiles=TILES_AUTO, out=None):
    """y [T,H] bf16."""
    import torch
    T, k = _dims(topk_w, 2, "topk_w")
    E, I, H = _dims(w_down, 3, "w_down")
    _check_args([(h, torch.bfloat16, "h", (T * k, I)), (w_down, torch.bfloat16, "w_down", (E, I, H)),
                 (topk_w, torch.float32, "topk_w", (T, k)), (inv_perm, torch.int32, "inv_perm", (T, k)),
                 (offsets, torch.int32, "offsets", (E + 1,)), (shared_out, torch.float32, "shared_out", (T, H)),
                 (out, torch.bfloat16, "out", (T, H))], ws)
    if h is None or inv_perm is None or offsets is None:
        raise TypeError("h, inv_perm and offsets are required")
    y = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=h.device)
    _check(lib().moe_down_combine(_ptr(h), _ptr(w_down), _ptr(topk_w), _ptr(inv_perm), _ptr(offsets),
                                  _ptr(shared_out), T, H, E, I, k, tiles, _ptr(y), _ptr(ws), ws.numel(),
                                  _stream()), "moe_down_combine")
    return y


def forward(x, w_router, bias, w_gate_up, w_down, k, ws, w_sh_gate_up=None, w_sh_down=None,
            tiles=TILES_AUTO, router=ROUTER_AUTO, out=None, stage_events=None, info=None,
            scoring=SCORE_SOFTMAX, combine=COMBINE_AUTO):
    """The whole layer: y [T,H] bf16 (scoring: the router's SCORE_* rule;
    combine: COMBINE_* -- in the down GEMM's epilogue or in its own kernel).

    stage_events: optional list of 7 torch.cuda.Event recorded at the stage
    boundaries (see include/moe.h); info: optional dict that receives the
    number of kernels enqueued under "launches"."""
    import torch
    T, H = _dims(x, 2, "x")
    E, _, I2 = _dims(w_gate_up, 3, "w_gate_up")
    I = I2 // 2
    I_s = 0
    if (w_sh_gate_up is None) != (w_sh_down is None):
        raise TypeError("the shared expert needs both w_sh_gate_up and w_sh_down")
    if w_sh_gate_up is not None:
        I_s = _dims(w_sh_gate_up, 2, "w_sh_gate_up")[1] // 2
    E_r = _dims(w_router, 2, "w_router")[1]
    if E_r != E:
        raise ValueError(f"w_router has {E_r} experts, w_gate_up {E}")
    _check_args([(x, torch.bfloat16, "x", (T, H)), (w_router, torch.float32, "w_router", (H, E)),
                 (bias, torch.float32, "bias", (E,)), (w_gate_up, torch.bfloat16, "w_gate_up", (E, H, 2 * I)),
                 (w_down, torch.bfloat16, "w_down", (E, I, H)),
                 (w_sh_gate_up, torch.bfloat16, "w_sh_gate_up", (H, 2 * I_s)),
                 (w_sh_down, torch.bfloat16, "w_sh_down", (I_s, H)), (out, torch.bfloat16, "out", (T, H))], ws)
    y = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    opt = _Options(tiles, router)
    opt.scoring = scoring
    opt.combine = combine
    if stage_events is not None:
        for i, ev in enumerate(stage_events):
            if ev is not None:
                opt.stage_events[i] = ev.cuda_event
    _check(lib().moe_forward_ex(_ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate_up), _ptr(w_down),
                                _ptr(w_sh_gate_up), _ptr(w_sh_down), I_s, T, H, E, I, k, _ptr(y), _ptr(ws),
                                ws.numel(), ctypes.byref(opt), _stream()), "moe_forward")
    if info is not None:
        info["launches"] = opt.launches
    return y


def forward_mx(x, w_router, bias, w_gate_up_codes, w_gate_up_scales, w_down_codes, w_down_scales, k, ws,
               w_sh_gate_up=None, w_sh_down=None, tiles=TILES_AUTO, router=ROUTER_AUTO, out=None,
               stage_events=None, info=None, scoring=SCORE_SOFTMAX, combine=COMBINE_AUTO):
    """The layer on block-scaled FP8 expert weights W [E, K, N]: codes of the
    transpose uint8 [E, N, K] (OCP E4M3, K contiguous) and scales uint8
    [E, K/32, N] (OCP E8M0) for W_gate_up (K = H, N = 2I) and W_down (K = I,
    N = H); y [T,H] bf16 (include/moe.h)."""
    import torch
    T, H = _dims(x, 2, "x")
    E, I2, _ = _dims(w_gate_up_codes, 3, "w_gate_up_codes")
    I = I2 // 2
    I_s = 0
    if (w_sh_gate_up is None) != (w_sh_down is None):
        raise TypeError("the shared expert needs both w_sh_gate_up and w_sh_down")
    if w_sh_gate_up is not None:
        I_s = _dims(w_sh_gate_up, 2, "w_sh_gate_up")[1] // 2
    if H % 32 or I % 32:
        raise ValueError("H and I must be multiples of the 32-weight scale block")
    _check_args([(x, torch.bfloat16, "x", (T, H)), (w_router, torch.float32, "w_router", (H, E)),
                 (bias, torch.float32, "bias", (E,)),
                 (w_gate_up_codes, torch.uint8, "w_gate_up_codes", (E, 2 * I, H)),
                 (w_gate_up_scales, torch.uint8, "w_gate_up_scales", (E, H // 32, 2 * I)),
                 (w_down_codes, torch.uint8, "w_down_codes", (E, H, I)),
                 (w_down_scales, torch.uint8, "w_down_scales", (E, I // 32, H)),
                 (w_sh_gate_up, torch.bfloat16, "w_sh_gate_up", (H, 2 * I_s)),
                 (w_sh_down, torch.bfloat16, "w_sh_down", (I_s, H)), (out, torch.bfloat16, "out", (T, H))], ws)
    y = out if out is not None else torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    opt = _Options(tiles, router)
    opt.scoring = scoring
    opt.combine = combine
    if stage_events is not None:
        for i, ev in enumerate(stage_events):
            if ev is not None:
                opt.stage_events[i] = ev.cuda_event
    _check(lib().moe_forward_mx(_ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate_up_codes), _ptr(w_gate_up_scales),
                                _ptr(w_down_codes), _ptr(w_down_scales), _ptr(w_sh_gate_up), _ptr(w_sh_down), I_s,
                                T, H, E, I, k, _ptr(y), _ptr(ws), ws.numel(), ctypes.byref(opt), _stream()),
           "moe_forward_mx")
    if info is not None:
        info["launches"] = opt.launches
    return y


def selftest_timeout(ws, timeout_ns: int) -> None:
    _check_args([], ws)
    _check(lib().moe_selftest_timeout(_ptr(ws), ws.numel(), timeout_ns, _stream()), "moe_selftest_timeout")


def workspace_view(ws, T, H, E, I, k, I_s=0) -> dict:
    """Typed views of the intermediates inside a workspace (after forward)."""
    import torch
    L = workspace_layout(T, H, E, I, k, I_s)

    def view(name, dtype, shape):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        return ws[L[name]:L[name] + nbytes].view(dtype).view(*shape)

    return dict(topk_ids=view("topk_ids", torch.int32, (T, k)), topk_w=view("topk_w", torch.float32, (T, k)),
                counts=view("counts", torch.int32, (E,)), offsets=view("offsets", torch.int32, (E + 1,)),
                sorted_token_ids=view("sorted_token_ids", torch.int32, (T * k,)),
                inv_perm=view("inv_perm", torch.int32, (T, k)), h=view("h", torch.bfloat16, (T * k, I)),
                logits=view("logits", torch.float32, (T, E)))
