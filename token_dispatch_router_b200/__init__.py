"""Python binding of the B200 MoE-layer forward library (libmoe_b200.so).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
The functions take torch CUDA tensors (PyTorch is used for device memory and streams),
check dtype/shape/contiguity, and call the C ABI of include/moe.h through ctypes on the
current torch stream. There is no CPU fallback: without the compiled library, or without
a CUDA device, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "CUDA error",
          4: "workspace missing or too small", 5: "device wait timed out",
          6: "device index out of range"}


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} ({code})")
        self.code = code


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("n", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("renormalize", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("tile_round", ctypes.c_int32),
                ("tile_round_mode", ctypes.c_int32), ("ffn_variant", ctypes.c_int32),
                ("route_topk", ctypes.c_int32)]


class moe_workspace_layout(ctypes.Structure):
    _fields_ = [(f, ctypes.c_size_t) for f in (
        "logits", "topk_ids", "topk_w", "counts", "offsets", "assign_to_perm",
        "perm_to_assign", "permute_scratch", "a_act", "y_perm", "round_ids", "round_counts",
        "add_tok", "add_w", "add_ptr", "add_idx", "add_cursor", "slot_token", "n_assign",
        "total")]


class moe_omni_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("n_rows", ctypes.c_int32),
                ("n_cols", ctypes.c_int32), ("K", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("output_mode", ctypes.c_int32)]


class moe_omni_layout(ctypes.Structure):
    _fields_ = [(f, ctypes.c_size_t) for f in (
        "logits", "topk_ids", "topk_w", "counts", "offsets", "assign_to_perm",
        "perm_to_assign", "h", "scratch", "y32", "total")]


_P = ctypes.c_void_p
_S = ctypes.POINTER(moe_shape)
_O = ctypes.POINTER(moe_omni_shape)
_SIGS = {
    "moe_permute_workspace_size": (ctypes.c_size_t, [_S]),
    "moe_forward_workspace_size": (ctypes.c_size_t, [_S]),
    "moe_forward_workspace_layout": (ctypes.c_int, [_S, ctypes.POINTER(moe_workspace_layout)]),
    "moe_route": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_permute": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute_static": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]),
    "moe_grouped_ffn": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_combine": (ctypes.c_int, [_S, _P, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_forward_h": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                     ctypes.c_size_t, _P]),
    "moe_backward_workspace_size": (ctypes.c_size_t, [_S]),
    "moe_backward_router": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_backward": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]),
    "moe_omni_workspace_size": (ctypes.c_size_t, [_O]),
    "moe_omni_workspace_layout": (ctypes.c_int, [_O, ctypes.POINTER(moe_omni_layout)]),
    "moe_omni_route": (ctypes.c_int, [_O, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_omni_schedule": (ctypes.c_int, [_O, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_omni_experts": (ctypes.c_int, [_O, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_omni_forward": (ctypes.c_int, [_O, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                        _P]),
    "moe_get_device_status": (ctypes.c_int, [_P]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "moe_profile_reset": (ctypes.c_int, []),
    "moe_kernel_count": (ctypes.c_int, []),
    "moe_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_profile_query": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                                         ctypes.POINTER(ctypes.c_double)]),
    "moe_launch_count": (ctypes.c_int64, []),
    "moe_selftest_timeout": (ctypes.c_int, [ctypes.c_uint64, _P]),
}

_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the C ABI. Raises if the library is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run python -m "
                           "token_dispatch_router_b200.build)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(code: int, where: str) -> None:
    if code != 0:
        raise MoEError(code, where)


def make_shape(T: int, d: int, E: int, K: int, n: int = 0, capacity_factor: float = 0.0,
               renormalize: bool = True, dtype=torch.bfloat16, tile_round: int = 0,
               ffn_variant: int = 0, route_topk: int = 0,
               tile_round_mode: int = 0) -> moe_shape:
    """tile_round = R > 0 rounds each expert's count to whole R-row tiles: tile_round_mode
    0 = down (drops its weakest assignments), 1 = up (adds the strongest tokens that did not
    route to it), 2 = to the nearest tile; up and nearest run in moe_forward only.
    ffn_variant selects the bf16 grouped-GEMM tiles: 0 = automatic, 1 = single-CTA 128 x 256
    tiles, 2 = CTA-pair 256 x 256 tiles with the gate/up rows gathered in the GEMM, 3 = CTA
    pairs with the rows copied first (all compute the same result). route_topk selects the
    top-K form of the warp-per-token routers: 0 = automatic, 1 = K rounds of a warp arg-max,
    2 = bitonic merges (E <= 64, K <= 8)."""
    dt = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    return moe_shape(T, d, E, K, n, float(capacity_factor), 1 if renormalize else 0, dt,
                     int(tile_round), int(tile_round_mode), int(ffn_variant), int(route_topk))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _act_dtype(shape: moe_shape):
    return torch.bfloat16 if shape.dtype == MOE_BF16 else torch.float32


def permute_workspace_size(shape: moe_shape) -> int:
    return int(load_library().moe_permute_workspace_size(ctypes.byref(shape)))


def forward_workspace_size(shape: moe_shape) -> int:
    return int(load_library().moe_forward_workspace_size(ctypes.byref(shape)))


def forward_workspace_layout(shape: moe_shape) -> moe_workspace_layout:
    L = moe_workspace_layout()
    _check(load_library().moe_forward_workspace_layout(ctypes.byref(shape), ctypes.byref(L)),
           "moe_forward_workspace_layout")
    return L


def route(shape: moe_shape, x=None, w_r=None, bias=None, logits_in=None, logits_out=None,
          topk_ids=None, topk_w=None):
    """moe_route. Returns (topk_ids [T,K] int32, topk_w [T,K] fp32, logits_out or None)."""
    lib = load_library()
    T, E, K = shape.T, shape.E, shape.K
    dev = (logits_in if logits_in is not None else x).device
    dt = _act_dtype(shape)
    if logits_in is None:
        _dev(x, "x", dt, (T, shape.d))
        _dev(w_r, "w_r", dt, (shape.d, E))
    else:
        _dev(logits_in, "logits_in", torch.float32, (T, E))
    if bias is not None:
        _dev(bias, "bias", torch.float32, (E,))
    if topk_ids is None:
        topk_ids = torch.empty(T, K, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, K, dtype=torch.float32, device=dev)
    if logits_out is not None:
        _dev(logits_out, "logits_out", torch.float32, (T, E))
    _check(lib.moe_route(ctypes.byref(shape), _ptr(x), _ptr(w_r), _ptr(bias), _ptr(logits_in),
                         _ptr(logits_out), _ptr(topk_ids), _ptr(topk_w), _stream()), "moe_route")
    return topk_ids, topk_w, logits_out


def permute(shape: moe_shape, topk_ids: torch.Tensor, x=None, materialize: bool = False,
            workspace=None):
    """moe_permute. Returns dict(counts, offsets, assign_to_perm, perm_to_assign[, x_perm])."""
    lib = load_library()
    T, E, K = shape.T, shape.E, shape.K
    dev = topk_ids.device
    _dev(topk_ids, "topk_ids", torch.int32, (T, K))
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    a2p = torch.empty(T * K, dtype=torch.int32, device=dev)
    p2a = torch.empty(T * K, dtype=torch.int32, device=dev)  # tail past offsets[E] unwritten
    x_perm = None
    if materialize:
        _dev(x, "x", _act_dtype(shape), (T, shape.d))
        x_perm = torch.empty(T * K, shape.d, dtype=x.dtype, device=dev)
    need = permute_workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.moe_permute(ctypes.byref(shape), _ptr(topk_ids), _ptr(counts), _ptr(offsets),
                           _ptr(a2p), _ptr(p2a), _ptr(x if materialize else None), _ptr(x_perm),
                           _ptr(workspace), workspace.numel(), _stream()), "moe_permute")
    out = dict(counts=counts, offsets=offsets, assign_to_perm=a2p, perm_to_assign=p2a)
    if materialize:
        out["x_perm"] = x_perm
    return out


def dispatch(shape: moe_shape, x=None, w_r=None, bias=None, logits_in=None, logits_out=None,
             materialize: bool = False, workspace=None, out=None):
    """moe_dispatch (moe_route then moe_permute in one call). Returns dict(topk_ids, topk_w,
    counts, offsets, assign_to_perm, perm_to_assign[, x_perm][, logits_out]); `out` may hold
    preallocated tensors under those names."""
    lib = load_library()
    T, E, K = shape.T, shape.E, shape.K
    src = logits_in if logits_in is not None else x
    dev = src.device
    dt = _act_dtype(shape)
    if logits_in is None:
        _dev(x, "x", dt, (T, shape.d))
        _dev(w_r, "w_r", dt, (shape.d, E))
    else:
        _dev(logits_in, "logits_in", torch.float32, (T, E))
    if bias is not None:
        _dev(bias, "bias", torch.float32, (E,))
    if logits_out is not None:
        _dev(logits_out, "logits_out", torch.float32, (T, E))
    elif logits_in is None and shape.tile_round > 0:  # rounding reads the router logits
        logits_out = torch.empty(T, E, dtype=torch.float32, device=dev)
    o = dict(out or {})

    def get(name, shape_, dtype):
        if name not in o:
            o[name] = torch.empty(*shape_, dtype=dtype, device=dev)
        return o[name]

    ids = get("topk_ids", (T, K), torch.int32)
    w = get("topk_w", (T, K), torch.float32)
    counts = get("counts", (E,), torch.int32)
    offsets = get("offsets", (E + 1,), torch.int32)
    a2p = get("assign_to_perm", (T * K,), torch.int32)
    p2a = get("perm_to_assign", (T * K,), torch.int32)
    x_perm = None
    if materialize:
        _dev(x, "x", dt, (T, shape.d))
        x_perm = get("x_perm", (T * K, shape.d), x.dtype)
    need = permute_workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.moe_dispatch(ctypes.byref(shape), _ptr(x), _ptr(w_r), _ptr(bias), _ptr(logits_in),
                            _ptr(logits_out), _ptr(ids), _ptr(w), _ptr(counts), _ptr(offsets),
                            _ptr(a2p), _ptr(p2a), _ptr(x_perm), _ptr(workspace),
                            workspace.numel(), _stream()), "moe_dispatch")
    res = dict(topk_ids=ids, topk_w=w, counts=counts, offsets=offsets, assign_to_perm=a2p,
               perm_to_assign=p2a)
    if materialize:
        res["x_perm"] = x_perm
    if logits_out is not None:
        res["logits_out"] = logits_out
    return res


def permute_static(shape: moe_shape, topk_ids: torch.Tensor, x=None, materialize: bool = False):
    """moe_permute_static: moe_permute without a workspace, for callers that may not
    allocate device memory while they run (its scratch is a fixed array inside the
    library; see include/moe.h for the size limit and the sharing rules). The output
    tensors here are allocated by torch only for the convenience of this binding."""
    lib = load_library()
    T, E, K = shape.T, shape.E, shape.K
    dev = topk_ids.device
    _dev(topk_ids, "topk_ids", torch.int32, (T, K))
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    a2p = torch.empty(T * K, dtype=torch.int32, device=dev)
    p2a = torch.empty(T * K, dtype=torch.int32, device=dev)  # tail past offsets[E] unwritten
    x_perm = None
    if materialize:
        _dev(x, "x", _act_dtype(shape), (T, shape.d))
        x_perm = torch.empty(T * K, shape.d, dtype=x.dtype, device=dev)
    _check(lib.moe_permute_static(ctypes.byref(shape), _ptr(topk_ids), _ptr(counts),
                                  _ptr(offsets), _ptr(a2p), _ptr(p2a),
                                  _ptr(x if materialize else None), _ptr(x_perm), _stream()),
           "moe_permute_static")
    out = dict(counts=counts, offsets=offsets, assign_to_perm=a2p, perm_to_assign=p2a)
    if materialize:
        out["x_perm"] = x_perm
    return out


def grouped_ffn(shape: moe_shape, x, offsets, perm_to_assign, w_gate, w_up, w_down,
                a_act=None, y_perm=None):
    """moe_grouped_ffn. Returns (a_act [T*K, n], y_perm [T*K, d])."""
    lib = load_library()
    T, d, E, K, n = shape.T, shape.d, shape.E, shape.K, shape.n
    dt = _act_dtype(shape)
    _dev(x, "x", dt, (T, d))
    _dev(offsets, "offsets", torch.int32, (E + 1,))
    _dev(perm_to_assign, "perm_to_assign", torch.int32, (T * K,))
    _dev(w_gate, "w_gate", dt, (E, d, n))
    _dev(w_up, "w_up", dt, (E, d, n))
    _dev(w_down, "w_down", dt, (E, n, d))
    if a_act is None:
        a_act = torch.empty(T * K, n, dtype=dt, device=x.device)
    if y_perm is None:
        y_perm = torch.empty(T * K, d, dtype=dt, device=x.device)
    _check(lib.moe_grouped_ffn(ctypes.byref(shape), _ptr(x), _ptr(offsets), _ptr(perm_to_assign),
                               _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(a_act), _ptr(y_perm),
                               _stream()), "moe_grouped_ffn")
    return a_act, y_perm


def combine(shape: moe_shape, y_perm, assign_to_perm, topk_w, out=None):
    """moe_combine. Returns out [T, d]."""
    lib = load_library()
    T, d, K = shape.T, shape.d, shape.K
    dt = _act_dtype(shape)
    _dev(y_perm, "y_perm", dt)
    if y_perm.dim() != 2 or y_perm.shape[1] != d or y_perm.shape[0] < T * K:
        raise ValueError("y_perm must be [>= T*K, d]")
    _dev(assign_to_perm, "assign_to_perm", torch.int32, (T * K,))
    _dev(topk_w, "topk_w", torch.float32, (T, K))
    if out is None:
        out = torch.empty(T, d, dtype=dt, device=y_perm.device)
    _check(lib.moe_combine(ctypes.byref(shape), _ptr(y_perm), _ptr(assign_to_perm), _ptr(topk_w),
                           _ptr(out), _stream()), "moe_combine")
    return out


def forward(shape: moe_shape, x, w_r, w_gate, w_up, w_down, bias=None, logits_in=None, out=None,
            workspace=None):
    """moe_forward (the whole layer). Returns (out [T, d], workspace)."""
    lib = load_library()
    T, d, E, n = shape.T, shape.d, shape.E, shape.n
    dt = _act_dtype(shape)
    _dev(x, "x", dt, (T, d))
    if logits_in is None:
        _dev(w_r, "w_r", dt, (d, E))
    else:
        _dev(logits_in, "logits_in", torch.float32, (T, E))
    _dev(w_gate, "w_gate", dt, (E, d, n))
    _dev(w_up, "w_up", dt, (E, d, n))
    _dev(w_down, "w_down", dt, (E, n, d))
    if bias is not None:
        _dev(bias, "bias", torch.float32, (E,))
    need = forward_workspace_size(shape)
    if need == 0:
        raise MoEError(1, "moe_forward_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty(T, d, dtype=dt, device=x.device)
    _check(lib.moe_forward(ctypes.byref(shape), _ptr(x), _ptr(w_r), _ptr(bias), _ptr(logits_in),
                           _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(out), _ptr(workspace),
                           workspace.numel(), _stream()), "moe_forward")
    return out, workspace


def forward_h(shape: moe_shape, x, w_r, w_gate, w_up, w_down, bias=None, logits_in=None,
              out=None, workspace=None, h=None):
    """moe_forward_h: the layer, keeping the gate/up pre-activations for the backward.
    Returns (out [T, d], workspace, h [T*K, 2n])."""
    lib = load_library()
    T, d, E, n, K = shape.T, shape.d, shape.E, shape.n, shape.K
    dt = _act_dtype(shape)
    _dev(x, "x", dt, (T, d))
    if logits_in is None:
        _dev(w_r, "w_r", dt, (d, E))
    else:
        _dev(logits_in, "logits_in", torch.float32, (T, E))
    _dev(w_gate, "w_gate", dt, (E, d, n))
    _dev(w_up, "w_up", dt, (E, d, n))
    _dev(w_down, "w_down", dt, (E, n, d))
    if bias is not None:
        _dev(bias, "bias", torch.float32, (E,))
    need = forward_workspace_size(shape)
    if need == 0:
        raise MoEError(1, "moe_forward_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty(T, d, dtype=dt, device=x.device)
    if h is None:
        h = torch.empty(T * K, 2 * n, dtype=dt, device=x.device)
    _check(lib.moe_forward_h(ctypes.byref(shape), _ptr(x), _ptr(w_r), _ptr(bias), _ptr(logits_in),
                             _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(out), _ptr(h),
                             _ptr(workspace), workspace.numel(), _stream()), "moe_forward_h")
    return out, workspace, h


def backward(shape: moe_shape, d_out, topk_w, offsets, perm_to_assign, assign_to_perm,
             w_down, h, w_gate=None, w_up=None, d_h=None, d_w=None, d_x=None,
             input_grad: bool = False, workspace=None):
    """moe_backward. Returns (d_h [T*K, 2n] = dG | dU per kept slot, d_w [T, K], d_x [T, d]
    or None); the input gradient is computed when input_grad (then w_gate, w_up needed)."""
    lib = load_library()
    T, d, E, n, K = shape.T, shape.d, shape.E, shape.n, shape.K
    dt = _act_dtype(shape)
    _dev(d_out, "d_out", dt, (T, d))
    _dev(w_down, "w_down", dt, (E, n, d))
    _dev(h, "h", dt, (T * K, 2 * n))
    dev = d_out.device
    if d_h is None:
        d_h = torch.empty(T * K, 2 * n, dtype=dt, device=dev)
    if d_w is None:
        d_w = torch.empty(T, K, dtype=torch.float32, device=dev)
    if input_grad:
        _dev(w_gate, "w_gate", dt, (E, d, n))
        _dev(w_up, "w_up", dt, (E, d, n))
        if d_x is None:
            d_x = torch.empty(T, d, dtype=dt, device=dev)
    else:
        d_x = None
    need = int(lib.moe_backward_workspace_size(ctypes.byref(shape)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.moe_backward(ctypes.byref(shape), _ptr(d_out), _ptr(topk_w), _ptr(offsets),
                            _ptr(perm_to_assign), _ptr(assign_to_perm), _ptr(w_gate), _ptr(w_up),
                            _ptr(w_down), _ptr(h), _ptr(d_h), _ptr(d_w), _ptr(d_x),
                            _ptr(workspace), workspace.numel(), _stream()), "moe_backward")
    return d_h, d_w, d_x


def backward_router(shape: moe_shape, x, w_r, topk_ids, topk_w, d_w, logits=None, d_x=None,
                    with_bias: bool = False):
    """moe_backward_router. Adds the router's term into d_x when given. Returns (d_logits
    [T, E], d_w_r [d, E], d_bias [E] or None)."""
    lib = load_library()
    T, d, E = shape.T, shape.d, shape.E
    dt = _act_dtype(shape)
    _dev(x, "x", dt, (T, d))
    _dev(w_r, "w_r", dt, (d, E))
    dev = x.device
    d_logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    d_w_r = torch.empty(d, E, dtype=torch.float32, device=dev)
    d_bias = torch.empty(E, dtype=torch.float32, device=dev) if with_bias else None
    if d_x is not None:
        _dev(d_x, "d_x", dt, (T, d))
    _check(lib.moe_backward_router(ctypes.byref(shape), _ptr(x), _ptr(w_r), _ptr(logits),
                                   _ptr(topk_ids), _ptr(topk_w), _ptr(d_w), _ptr(d_logits),
                                   _ptr(d_w_r), _ptr(d_bias), _ptr(d_x), _stream()),
           "moe_backward_router")
    return d_logits, d_w_r, d_bias


def workspace_views(shape: moe_shape, workspace: torch.Tensor) -> dict:
    """Typed views of moe_forward's intermediates inside its workspace."""
    L = forward_workspace_layout(shape)
    T, E, K, d, n = shape.T, shape.E, shape.K, shape.d, shape.n
    A = int(L.n_assign)  # T * K, plus E * (R - 1) added entries when rounding up
    dt = _act_dtype(shape)
    eb = 2 if dt == torch.bfloat16 else 4

    def view(off, count, dtype, shp, esz):
        return workspace[off:off + count * esz].view(dtype).view(*shp)

    v = dict(logits=view(L.logits, T * E, torch.float32, (T, E), 4),
             topk_ids=view(L.topk_ids, T * K, torch.int32, (T, K), 4),
             topk_w=view(L.topk_w, T * K, torch.float32, (T, K), 4),
             counts=view(L.counts, E, torch.int32, (E,), 4),
             offsets=view(L.offsets, E + 1, torch.int32, (E + 1,), 4),
             assign_to_perm=view(L.assign_to_perm, A, torch.int32, (A,), 4),
             perm_to_assign=view(L.perm_to_assign, A, torch.int32, (A,), 4),
             a_act=view(L.a_act, A * n, dt, (A, n), eb),
             y_perm=view(L.y_perm, A * d, dt, (A, d), eb))
    if A > T * K:  # rounding up or to the nearest tile
        NA = A - T * K
        v.update(round_ids=view(L.round_ids, A, torch.int32, (A,), 4),
                 add_tok=view(L.add_tok, NA, torch.int32, (NA,), 4),
                 add_w=view(L.add_w, NA, torch.float32, (NA,), 4),
                 add_ptr=view(L.add_ptr, T + 1, torch.int32, (T + 1,), 4),
                 add_idx=view(L.add_idx, NA, torch.int32, (NA,), 4),
                 slot_token=view(L.slot_token, A, torch.int32, (A,), 4))
    return v


# ------------------------------------------------------------------ atomic experts
def make_omni_shape(T: int, d: int, n_rows: int, n_cols: int, K: int,
                    renormalize: bool = True, output_mode: int = 0) -> moe_omni_shape:
    """N = n_rows * n_cols rank-1 experts on a Cartesian grid, top-K per token. output_mode
    (moe_omni_forward): 0 = token-centric gather (deterministic), 1 = expert-centric
    scatter-add."""
    return moe_omni_shape(T, d, n_rows, n_cols, K, 1 if renormalize else 0, int(output_mode))


def omni_workspace_size(shape: moe_omni_shape) -> int:
    return int(load_library().moe_omni_workspace_size(ctypes.byref(shape)))


def omni_workspace_layout(shape: moe_omni_shape) -> moe_omni_layout:
    L = moe_omni_layout()
    _check(load_library().moe_omni_workspace_layout(ctypes.byref(shape), ctypes.byref(L)),
           "moe_omni_workspace_layout")
    return L


def omni_route(shape: moe_omni_shape, x=None, w_row=None, w_col=None, logits_in=None,
               logits_out=None, topk_ids=None, topk_w=None):
    """moe_omni_route. Returns (topk_ids [T,K] int32, topk_w [T,K] fp32, logits or None)."""
    lib = load_library()
    T, K, P = shape.T, shape.K, shape.n_rows + shape.n_cols
    dev = (logits_in if logits_in is not None else x).device
    if logits_in is None:
        _dev(x, "x", torch.bfloat16, (T, shape.d))
        _dev(w_row, "w_row", torch.bfloat16, (shape.d, shape.n_rows))
        _dev(w_col, "w_col", torch.bfloat16, (shape.d, shape.n_cols))
        if logits_out is None:
            logits_out = torch.empty(T, P, dtype=torch.float32, device=dev)
        _dev(logits_out, "logits_out", torch.float32, (T, P))
    else:
        _dev(logits_in, "logits_in", torch.float32, (T, P))
    if topk_ids is None:
        topk_ids = torch.empty(T, K, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, K, dtype=torch.float32, device=dev)
    _check(lib.moe_omni_route(ctypes.byref(shape), _ptr(x), _ptr(w_row), _ptr(w_col),
                              _ptr(logits_in), _ptr(logits_out), _ptr(topk_ids), _ptr(topk_w),
                              _stream()), "moe_omni_route")
    return topk_ids, topk_w, logits_out


def omni_schedule(shape: moe_omni_shape, topk_ids, workspace=None):
    """moe_omni_schedule. Returns dict(counts, offsets, assign_to_perm, perm_to_assign)."""
    lib = load_library()
    T, K = shape.T, shape.K
    N = shape.n_rows * shape.n_cols
    dev = topk_ids.device
    _dev(topk_ids, "topk_ids", torch.int32, (T, K))
    counts = torch.empty(N, dtype=torch.int32, device=dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    a2p = torch.empty(T * K, dtype=torch.int32, device=dev)
    p2a = torch.empty(T * K, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(omni_workspace_size(shape), dtype=torch.uint8, device=dev)
    _check(lib.moe_omni_schedule(ctypes.byref(shape), _ptr(topk_ids), _ptr(counts),
                                 _ptr(offsets), _ptr(a2p), _ptr(p2a), _ptr(workspace),
                                 workspace.numel(), _stream()), "moe_omni_schedule")
    return dict(counts=counts, offsets=offsets, assign_to_perm=a2p, perm_to_assign=p2a)


def omni_experts(shape: moe_omni_shape, x, w_in, w_out, topk_ids, topk_w, offsets,
                 perm_to_assign, h=None, out=None):
    """moe_omni_experts. Returns (out [T, d] bf16, h [T*K] fp32)."""
    lib = load_library()
    T, K, d = shape.T, shape.K, shape.d
    N = shape.n_rows * shape.n_cols
    _dev(x, "x", torch.bfloat16, (T, d))
    _dev(w_in, "w_in", torch.bfloat16, (N, d))
    _dev(w_out, "w_out", torch.bfloat16, (N, d))
    _dev(topk_ids, "topk_ids", torch.int32, (T, K))
    _dev(topk_w, "topk_w", torch.float32, (T, K))
    _dev(offsets, "offsets", torch.int32, (N + 1,))
    _dev(perm_to_assign, "perm_to_assign", torch.int32, (T * K,))
    if h is None:
        h = torch.empty(T * K, dtype=torch.float32, device=x.device)
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _dev(h, "h", torch.float32, (T * K,))
    _dev(out, "out", torch.bfloat16, (T, d))
    _check(lib.moe_omni_experts(ctypes.byref(shape), _ptr(x), _ptr(w_in), _ptr(w_out),
                                _ptr(topk_ids), _ptr(topk_w), _ptr(offsets),
                                _ptr(perm_to_assign), _ptr(h), _ptr(out), _stream()),
           "moe_omni_experts")
    return out, h


def omni_forward(shape: moe_omni_shape, x, w_row, w_col, w_in, w_out, logits_in=None,
                 out=None, workspace=None):
    """moe_omni_forward. Returns (out [T, d] bf16, workspace)."""
    lib = load_library()
    T, d = shape.T, shape.d
    N = shape.n_rows * shape.n_cols
    _dev(x, "x", torch.bfloat16, (T, d))
    if logits_in is None:
        _dev(w_row, "w_row", torch.bfloat16, (d, shape.n_rows))
        _dev(w_col, "w_col", torch.bfloat16, (d, shape.n_cols))
    else:
        _dev(logits_in, "logits_in", torch.float32, (T, shape.n_rows + shape.n_cols))
    _dev(w_in, "w_in", torch.bfloat16, (N, d))
    _dev(w_out, "w_out", torch.bfloat16, (N, d))
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _dev(out, "out", torch.bfloat16, (T, d))
    if workspace is None:
        workspace = torch.empty(omni_workspace_size(shape), dtype=torch.uint8, device=x.device)
    _check(lib.moe_omni_forward(ctypes.byref(shape), _ptr(x), _ptr(w_row), _ptr(w_col),
                                _ptr(logits_in), _ptr(w_in), _ptr(w_out), _ptr(out),
                                _ptr(workspace), workspace.numel(), _stream()),
           "moe_omni_forward")
    return out, workspace


def omni_workspace_views(shape: moe_omni_shape, workspace: torch.Tensor) -> dict:
    """Typed views of moe_omni_forward's intermediates inside its workspace (perm_to_assign
    grouped by expert, any order inside an expert; assign_to_perm is not written)."""
    L = omni_workspace_layout(shape)
    T, K = shape.T, shape.K
    N, P, M = shape.n_rows * shape.n_cols, shape.n_rows + shape.n_cols, shape.T * shape.K

    def view(off, count, dtype, shp):
        return workspace[off:off + count * 4].view(dtype).view(*shp)

    return dict(logits=view(L.logits, T * P, torch.float32, (T, P)),
                topk_ids=view(L.topk_ids, M, torch.int32, (T, K)),
                topk_w=view(L.topk_w, M, torch.float32, (T, K)),
                counts=view(L.counts, N, torch.int32, (N,)),
                offsets=view(L.offsets, N + 1, torch.int32, (N + 1,)),
                assign_to_perm=view(L.assign_to_perm, M, torch.int32, (M,)),
                perm_to_assign=view(L.perm_to_assign, M, torch.int32, (M,)),
                h=view(L.h, M, torch.float32, (M,)))


def device_status() -> int:
    return int(load_library().moe_get_device_status(_stream()))


def selftest_timeout(limit_ns: int) -> int:
    """Run the bounded-wait self test; returns the device status it leaves (5 = timeout)."""
    lib = load_library()
    _check(lib.moe_selftest_timeout(int(limit_ns), _stream()), "moe_selftest_timeout")
    return device_status()


class Profiler:
    """Per-kernel device time from the library's opt-in event profiler."""

    def __init__(self):
        self.lib = load_library()

    def __enter__(self):
        self.lib.moe_profile_reset()
        self.lib.moe_profile_enable(1)
        return self

    def __exit__(self, *exc):
        self.lib.moe_profile_enable(0)

    def results(self) -> dict:
        out = {}
        for i in range(self.lib.moe_kernel_count()):
            n = ctypes.c_int64(0)
            ms = ctypes.c_double(0.0)
            _check(self.lib.moe_profile_query(i, ctypes.byref(n), ctypes.byref(ms)),
                   "moe_profile_query")
            if n.value:
                out[self.lib.moe_kernel_name(i).decode()] = (int(n.value), float(ms.value))
        return out


def launch_count() -> int:
    return int(load_library().moe_launch_count())
