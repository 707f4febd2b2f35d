"""B200 (sm_100a) MoE-layer forward: Python binding of ``libmoe_b200.so``.

The functions here carry the names of the C ABI in ``include/moe.h`` and only
marshal arguments: they check tensor devices/dtypes/shapes, pass raw device
pointers and the current CUDA stream, and raise :class:`MoeError` on a
non-OK status.  Every step of the layer runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback.  Importing this package does not need a
GPU, but it does need the built library (``python -m
routing_dispatch_experts_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_ALIGNMENT = 3
MOE_ERR_WORKSPACE = 4
MOE_ERR_CUDA = 5
MOE_ERR_DEVICE_TIMEOUT = 6
MOE_ERR_DEVICE_INDEX = 7
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_ALIGNMENT", 4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA",
                6: "MOE_ERR_DEVICE_TIMEOUT", 7: "MOE_ERR_DEVICE_INDEX"}
MOE_F32, MOE_BF16 = 0, 1


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("ep", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class moe_stats(ctypes.Structure):
    _fields_ = [("rows_sent", ctypes.c_int64), ("dup_removed", ctypes.c_int64),
                ("tokens_single_rank", ctypes.c_int64), ("home_rank_rows", ctypes.c_int64),
                ("max_expert_rows", ctypes.c_int32), ("min_expert_rows", ctypes.c_int32)]


STATS_FIELDS = ("rows_sent", "dup_removed", "tokens_single_rank", "home_rank_rows",
                "max_expert_rows", "min_expert_rows")


class moe_router_counts(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int64), ("near_tie_tokens", ctypes.c_int64),
                ("changed_tokens", ctypes.c_int64), ("changed_experts", ctypes.c_int64),
                ("changed_slots", ctypes.c_int64)]


ROUTER_COUNT_FIELDS = ("tokens", "near_tie_tokens", "changed_tokens", "changed_experts",
                       "changed_slots")


class moe_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
        "rank_offsets", "send_token", "slot_send_row", "stats")]


class moe_ep_peer_dest(ctypes.Structure):
    _fields_ = [("recv_x", ctypes.c_void_p), ("recv_idx", ctypes.c_void_p),
                ("recv_gate", ctypes.c_void_p), ("row0", ctypes.c_int64), ("rows", ctypes.c_int64)]


class moe_ep_peer_return(ctypes.Structure):
    _fields_ = [("y_back", ctypes.c_void_p), ("row0", ctypes.c_int64), ("rows", ctypes.c_int64)]


class moe_forward_buffers(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p),
                ("topk_gate", ctypes.c_void_p), ("layout", moe_layout),
                ("x_perm", ctypes.c_void_p), ("h", ctypes.c_void_p), ("y_perm", ctypes.c_void_p)]


_lib = None

# exported C symbols, in header order (checked against include/moe.h by the tests)
SYMBOLS = ("moe_status_string", "moe_scratch_size", "moe_forward_workspace_size",
           "moe_workspace_init", "moe_packed_weights_size", "moe_pack_weights", "moe_route",
           "moe_unpacked_workspace_size", "moe_route_unpacked", "moe_grouped_swiglu_unpacked",
           "moe_route_selection_bias", "moe_router_stats", "moe_capacity_keep",
           "moe_dispatch_layout", "moe_coselection_counts", "moe_fit_placement", "moe_permute", "moe_permute_by_token", "moe_grouped_swiglu",
           "moe_grouped_swiglu_gather", "moe_combine", "moe_forward", "moe_forward_selection_bias", "moe_forward_timed",
           "moe_forward_routed", "moe_ep_pack", "moe_ep_expert_workspace_size",
           "moe_ep_expert_forward", "moe_ep_home_combine", "moe_ep_dispatch_peer",
           "moe_ep_expert_forward_peer", "moe_ep_signal_wait", "moe_debug_ep_signal_wait",
           "moe_get_device_status", "moe_debug_dispatch_layout_stall",
           "moe_debug_grouped_swiglu_engine", "moe_debug_forward_options",
           "moe_dispatch_layout_static")
FORWARD_STAGES = ("route", "layout", "permute", "gate_up", "down", "combine")


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m routing_dispatch_experts_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.POINTER(moe_shape)
        sz = ctypes.POINTER(ctypes.c_size_t)
        sig = {
            "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "moe_scratch_size": ([S, sz], ctypes.c_int),
            "moe_forward_workspace_size": ([S, sz], ctypes.c_int),
            "moe_workspace_init": ([P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_packed_weights_size": ([S, sz], ctypes.c_int),
            "moe_pack_weights": ([S, P, P, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_route": ([S, P, P, P, P, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_unpacked_workspace_size": ([S, sz], ctypes.c_int),
            "moe_route_unpacked": ([S, P, P, P, P, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_grouped_swiglu_unpacked": ([S, P, P, P, P, P, P, P, P, ctypes.c_size_t, P],
                                            ctypes.c_int),
            "moe_route_selection_bias": ([S, P, P, P, P, P, P, P, P, ctypes.c_size_t, P],
                                         ctypes.c_int),
            "moe_router_stats": ([S, P, P, P, P, ctypes.c_double, P, P, P], ctypes.c_int),
            "moe_capacity_keep": ([S, P, P, ctypes.c_double, P, P, ctypes.POINTER(ctypes.c_int64),
                                   P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_dispatch_layout": ([S, P, P, ctypes.POINTER(moe_layout), P, ctypes.c_size_t, P],
                                    ctypes.c_int),
            "moe_coselection_counts": ([S, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_fit_placement": ([ctypes.c_int32, ctypes.c_int32, P, P], ctypes.c_int),
            "moe_permute": ([S, P, P, P, P], ctypes.c_int),
            "moe_permute_by_token": ([S, P, P, P, P], ctypes.c_int),
            "moe_grouped_swiglu": ([S, P, P, P, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_combine": ([S, P, P, P, P, P], ctypes.c_int),
            "moe_grouped_swiglu_gather": ([S, P, P, P, P, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_forward_timed": ([S, P, P, P, P, P, ctypes.POINTER(moe_forward_buffers), P,
                                   ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p), P],
                                  ctypes.c_int),
            "moe_forward": ([S, P, P, P, P, P, ctypes.POINTER(moe_forward_buffers), P,
                             ctypes.c_size_t, P], ctypes.c_int),
            "moe_forward_routed": ([S, P, P, P, P, P, P, ctypes.POINTER(moe_forward_buffers), P,
                                    ctypes.c_size_t, P], ctypes.c_int),
            "moe_forward_selection_bias": ([S, P, P, P, P, P, P,
                                            ctypes.POINTER(moe_forward_buffers), P,
                                            ctypes.c_size_t, P], ctypes.c_int),
            "moe_ep_pack": ([S, P, P, P, P, ctypes.POINTER(moe_layout), P, P, P, ctypes.c_int64, P],
                            ctypes.c_int),
            "moe_ep_expert_workspace_size": ([S, sz], ctypes.c_int),
            "moe_ep_expert_forward": ([S, P, P, P, P, P, P, ctypes.c_size_t, P], ctypes.c_int),
            "moe_ep_home_combine": ([S, P, P, ctypes.c_int64, P, P], ctypes.c_int),
            "moe_ep_dispatch_peer": ([S, P, P, P, P, ctypes.POINTER(moe_layout),
                                      ctypes.POINTER(moe_ep_peer_dest), P], ctypes.c_int),
            "moe_ep_expert_forward_peer": ([S, P, P, P, P, ctypes.POINTER(moe_ep_peer_return), P,
                                            ctypes.c_size_t, P], ctypes.c_int),
            "moe_ep_signal_wait": ([ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32,
                                    ctypes.c_int32, ctypes.c_uint64, P, P], ctypes.c_int),
            "moe_debug_ep_signal_wait": ([ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_uint64, P, ctypes.c_int64, P],
                                         ctypes.c_int),
            "moe_get_device_status": ([P, P, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "moe_debug_dispatch_layout_stall": ([S, P, P, ctypes.POINTER(moe_layout), P,
                                                 ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64, P],
                                                ctypes.c_int),
            "moe_dispatch_layout_static": ([S, P, P, ctypes.POINTER(moe_layout), P, P], ctypes.c_int),
            "moe_debug_grouped_swiglu_engine": ([S, P, P, P, P, P, P, P, ctypes.c_size_t,
                                                 ctypes.c_int32, P], ctypes.c_int),
            "moe_debug_forward_options": ([S, P, P, P, P, P, ctypes.POINTER(moe_forward_buffers),
                                           P, ctypes.c_size_t, ctypes.c_int32, P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


# ------------------------------------------------------------------ helpers
@dataclass(frozen=True)
class Shape:
    T: int
    d: int
    E: int
    k: int
    f: int
    ep: int = 1
    dtype: torch.dtype = torch.bfloat16

    @property
    def c(self) -> moe_shape:
        return moe_shape(self.T, self.d, self.E, self.k, self.f, self.ep,
                         MOE_BF16 if self.dtype == torch.bfloat16 else MOE_F32)

    @property
    def R(self) -> int:
        return self.T * self.k


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, shape, name):
    if t is None:
        raise ValueError(f"{name}: required")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _need_n(t, dtype, n, name):
    """dtype and element count of an index or gate array (any shape)."""
    if t is None:
        raise ValueError(f"{name}: required")
    if t.dtype != dtype or t.numel() != n:
        raise ValueError(f"{name}: expected {dtype} with {n} elements, "
                         f"got {t.dtype} {tuple(t.shape)}")


def _need_packed(shape: "Shape", packed):
    """The packed weights buffer: uint8, at least the size pack_weights makes."""
    n = packed_weights_size(shape)
    if packed is None or packed.dtype != torch.uint8 or packed.numel() < n:
        got = "None" if packed is None else f"{packed.dtype} x {packed.numel()}"
        raise ValueError(f"packed: expected uint8 of at least {n} bytes (pack_weights), got {got}")


def _need_bias(shape: "Shape", bias):
    if bias is not None:
        _need(bias, torch.float32, (shape.E,), "bias")


def scratch_size(shape: Shape) -> int:
    n = ctypes.c_size_t()
    s = shape.c
    _check(lib().moe_scratch_size(ctypes.byref(s), ctypes.byref(n)), "moe_scratch_size")
    return n.value


def forward_workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t()
    s = shape.c
    _check(lib().moe_forward_workspace_size(ctypes.byref(s), ctypes.byref(n)),
           "moe_forward_workspace_size")
    return n.value


def packed_weights_size(shape: Shape) -> int:
    n = ctypes.c_size_t()
    s = shape.c
    _check(lib().moe_packed_weights_size(ctypes.byref(s), ctypes.byref(n)),
           "moe_packed_weights_size")
    return n.value


def workspace(shape: Shape, forward: bool = False, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (uint8) of the size the ABI asks for."""
    n = forward_workspace_size(shape) if forward else scratch_size(shape)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().moe_workspace_init(_p(ws), ws.numel(), _stream(stream)), "moe_workspace_init")


def pack_weights(shape: Shape, w_router, w_gate, w_up, w_down, stream=None) -> torch.Tensor:
    """Pack W_r [d,E], W_g/W_u [E,d,f], W_d [E,f,d] into the kernels' layout.
    w_router=None packs the experts alone; w_gate=w_up=w_down=None the
    router alone."""
    if w_router is not None:
        _need(w_router, shape.dtype, (shape.d, shape.E), "w_router")
    if w_gate is not None or w_up is not None or w_down is not None:
        _need(w_gate, shape.dtype, (shape.E, shape.d, shape.f), "w_gate")
        _need(w_up, shape.dtype, (shape.E, shape.d, shape.f), "w_up")
        _need(w_down, shape.dtype, (shape.E, shape.f, shape.d), "w_down")
    dev = (w_router if w_router is not None else w_gate).device
    n = packed_weights_size(shape)
    packed = torch.zeros(n, dtype=torch.uint8, device=dev)
    s = shape.c
    _check(lib().moe_pack_weights(ctypes.byref(s), _p(w_router), _p(w_gate), _p(w_up), _p(w_down),
                                  _p(packed), n, _stream(stream)), "moe_pack_weights")
    return packed


def route(shape: Shape, x, packed, bias, ws, logits=None, stream=None):
    """moe_route: returns (logits [T,E] f32, topk_idx [T,k] i32, topk_gate [T,k] f32).

    x=None runs only the top-k step on the given `logits`."""
    dev = ws.device
    if x is not None:
        _need(x, shape.dtype, (shape.T, shape.d), "x")
        _need_packed(shape, packed)
        logits = torch.empty((shape.T, shape.E), dtype=torch.float32, device=dev)
    else:
        _need(logits, torch.float32, (shape.T, shape.E), "logits")
    _need_bias(shape, bias)
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device=dev)
    gate = torch.empty((shape.T, shape.k), dtype=torch.float32, device=dev)
    s = shape.c
    _check(lib().moe_route(ctypes.byref(s), _p(x), _p(packed), _p(bias), _p(logits), _p(idx),
                           _p(gate), _p(ws), ws.numel(), _stream(stream)), "moe_route")
    return logits, idx, gate


def unpacked_workspace(shape: Shape, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for the *_unpacked calls."""
    n = ctypes.c_size_t()
    s = shape.c
    _check(lib().moe_unpacked_workspace_size(ctypes.byref(s), ctypes.byref(n)),
           "moe_unpacked_workspace_size")
    return torch.zeros(n.value, dtype=torch.uint8, device=device)


def route_unpacked(shape: Shape, x, w_router, bias, ws, stream=None):
    """moe_route_unpacked: the router on W_r [d, E]; (logits, idx, gate)."""
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need(w_router, shape.dtype, (shape.d, shape.E), "w_router")
    _need_bias(shape, bias)
    dev = ws.device
    logits = torch.empty((shape.T, shape.E), dtype=torch.float32, device=dev)
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device=dev)
    gate = torch.empty((shape.T, shape.k), dtype=torch.float32, device=dev)
    s = shape.c
    _check(lib().moe_route_unpacked(ctypes.byref(s), _p(x), _p(w_router), _p(bias), _p(logits),
                                    _p(idx), _p(gate), _p(ws), ws.numel(), _stream(stream)),
           "moe_route_unpacked")
    return logits, idx, gate


def grouped_swiglu_unpacked(shape: Shape, x_perm, expert_offsets, w_gate, w_up, w_down, ws,
                            stream=None):
    """moe_grouped_swiglu_unpacked: (h, y_perm) from W_g/W_u [E,d,f], W_d [E,f,d]."""
    _need(x_perm, shape.dtype, (shape.R, shape.d), "x_perm")
    _need_n(expert_offsets, torch.int32, shape.E + 1, "expert_offsets")
    _need(w_gate, shape.dtype, (shape.E, shape.d, shape.f), "w_gate")
    _need(w_up, shape.dtype, (shape.E, shape.d, shape.f), "w_up")
    _need(w_down, shape.dtype, (shape.E, shape.f, shape.d), "w_down")
    h = torch.empty((shape.R, shape.f), dtype=shape.dtype, device=x_perm.device)
    y_perm = torch.empty((shape.R, shape.d), dtype=shape.dtype, device=x_perm.device)
    s = shape.c
    _check(lib().moe_grouped_swiglu_unpacked(ctypes.byref(s), _p(x_perm), _p(expert_offsets),
                                             _p(w_gate), _p(w_up), _p(w_down), _p(h), _p(y_perm),
                                             _p(ws), ws.numel(), _stream(stream)),
           "moe_grouped_swiglu_unpacked")
    return h, y_perm


def route_selection_bias(shape: Shape, x, packed, bias, selection_bias, ws, logits=None,
                         stream=None):
    """moe_route_selection_bias: experts chosen on logits + selection_bias,
    gates from the logits alone.  Returns (logits, topk_idx, topk_gate);
    x=None runs only the selection on the given `logits`."""
    dev = ws.device
    if x is not None:
        _need(x, shape.dtype, (shape.T, shape.d), "x")
        _need_packed(shape, packed)
        logits = torch.empty((shape.T, shape.E), dtype=torch.float32, device=dev)
    else:
        _need(logits, torch.float32, (shape.T, shape.E), "logits")
    _need_bias(shape, bias)
    _need(selection_bias, torch.float32, (shape.E,), "selection_bias")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device=dev)
    gate = torch.empty((shape.T, shape.k), dtype=torch.float32, device=dev)
    s = shape.c
    _check(lib().moe_route_selection_bias(ctypes.byref(s), _p(x), _p(packed), _p(bias),
                                          _p(selection_bias), _p(logits), _p(idx), _p(gate),
                                          _p(ws), ws.numel(), _stream(stream)),
           "moe_route_selection_bias")
    return logits, idx, gate


def router_stats(shape: Shape, logits, topk_idx=None, recorded_idx=None, threshold=1e-5,
                 selection_bias=None, want_margin=False, stream=None):
    """moe_router_stats: (dict of the counters, margin [T] float64 or None).
    The counters are read back to the host (a synchronisation)."""
    _need(logits, torch.float32, (shape.T, shape.E), "logits")
    if topk_idx is not None:
        _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    if recorded_idx is not None:
        _need(recorded_idx, torch.int32, (shape.T, shape.k), "recorded_idx")
    if selection_bias is not None:
        _need(selection_bias, torch.float32, (shape.E,), "selection_bias")
    dev = logits.device
    counts = torch.zeros(len(ROUTER_COUNT_FIELDS), dtype=torch.int64, device=dev)
    margin = torch.empty(shape.T, dtype=torch.float64, device=dev) if want_margin else None
    s = shape.c
    _check(lib().moe_router_stats(ctypes.byref(s), _p(logits), _p(selection_bias), _p(topk_idx),
                                  _p(recorded_idx), float(threshold), _p(margin), _p(counts),
                                  _stream(stream)), "moe_router_stats")
    return dict(zip(ROUTER_COUNT_FIELDS, counts.cpu().tolist())), margin


def capacity_keep(shape: Shape, topk_idx, topk_gate, capacity_factor: float, ws, stream=None):
    """moe_capacity_keep: (keep [T,k] int32, kept_gate [T,k] fp32, capacity)."""
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    if topk_gate is not None:
        _need(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    dev = topk_idx.device
    keep = torch.empty((shape.T, shape.k), dtype=torch.int32, device=dev)
    kept = torch.empty((shape.T, shape.k), dtype=torch.float32, device=dev)
    cap = ctypes.c_int64(0)
    s = shape.c
    _check(lib().moe_capacity_keep(ctypes.byref(s), _p(topk_idx), _p(topk_gate),
                                   float(capacity_factor), _p(keep), _p(kept), ctypes.byref(cap),
                                   _p(ws), ws.numel(), _stream(stream)), "moe_capacity_keep")
    return keep, kept, cap.value


def _layout_tensors(shape: Shape, dev):
    R = shape.R
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(expert_counts=torch.empty(shape.E, **i32),
               expert_offsets=torch.empty(shape.E + 1, **i32),
               row_token=torch.empty(R, **i32), slot_row=torch.empty(R, **i32),
               stats=torch.zeros(6, dtype=torch.int64, device=dev))
    if shape.ep > 1:
        out.update(rank_counts=torch.empty(shape.ep, **i32),
                   rank_offsets=torch.empty(shape.ep + 1, **i32),
                   send_token=torch.full((R,), -1, **i32),
                   slot_send_row=torch.empty(R, **i32))
    return out


def _c_layout(t: dict) -> moe_layout:
    return moe_layout(*[_p(t.get(n)) for n in (
        "expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
        "rank_offsets", "send_token", "slot_send_row", "stats")])


def _host_map(shape: Shape, expert_rank: Optional[Sequence[int]]):
    if expert_rank is None:
        return None
    if len(expert_rank) != shape.E:
        raise ValueError("expert_rank must have E entries")
    return (ctypes.c_int32 * shape.E)(*[int(r) for r in expert_rank])


def stats_dict(stats: torch.Tensor) -> dict:
    """Decode the device moe_stats (6 int64 words as allocated here)."""
    v = stats.cpu().tolist()
    lo = v[4] & 0xFFFFFFFF
    hi = (v[4] >> 32) & 0xFFFFFFFF
    return dict(rows_sent=v[0], dup_removed=v[1], tokens_single_rank=v[2],
                home_rank_rows=v[3], max_expert_rows=lo, min_expert_rows=hi)


def dispatch_layout(shape: Shape, topk_idx, ws, expert_rank=None, stream=None) -> dict:
    """moe_dispatch_layout: returns the layout tensors (see moe.h)."""
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    out = _layout_tensors(shape, ws.device)
    lay = _c_layout(out)
    s = shape.c
    _check(lib().moe_dispatch_layout(ctypes.byref(s), _p(topk_idx), _host_map(shape, expert_rank),
                                     ctypes.byref(lay), _p(ws), ws.numel(), _stream(stream)),
           "moe_dispatch_layout")
    return out


def debug_dispatch_layout_stall(shape: Shape, topk_idx, ws, stall_block: int, wait_limit_ns: int,
                                expert_rank=None, stream=None) -> dict:
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    out = _layout_tensors(shape, ws.device)
    lay = _c_layout(out)
    s = shape.c
    _check(lib().moe_debug_dispatch_layout_stall(
        ctypes.byref(s), _p(topk_idx), _host_map(shape, expert_rank), ctypes.byref(lay), _p(ws),
        ws.numel(), stall_block, wait_limit_ns, _stream(stream)), "moe_debug_dispatch_layout_stall")
    return out


def dispatch_layout_static(shape: Shape, topk_idx, expert_rank=None, stream=None):
    """moe_dispatch_layout_static: the layout with the library's own scratch
    (no workspace).  Returns (layout tensors, device status tensor [1])."""
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    out = _layout_tensors(shape, topk_idx.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=topk_idx.device)
    lay = _c_layout(out)
    s = shape.c
    _check(lib().moe_dispatch_layout_static(ctypes.byref(s), _p(topk_idx),
                                            _host_map(shape, expert_rank), ctypes.byref(lay),
                                            _p(status), _stream(stream)),
           "moe_dispatch_layout_static")
    return out, status


def coselection_counts(shape: Shape, topk_idx, ws, stream=None) -> torch.Tensor:
    """moe_coselection_counts: W [E, E] (uint64 counts held in an int64
    tensor on the device)."""
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    W = torch.empty((shape.E, shape.E), dtype=torch.int64, device=topk_idx.device)
    s = shape.c
    _check(lib().moe_coselection_counts(ctypes.byref(s), _p(topk_idx), _p(W), _p(ws), ws.numel(),
                                        _stream(stream)), "moe_coselection_counts")
    return W


def fit_placement(E: int, ep: int, counts) -> list:
    """moe_fit_placement on counts [E, E] (any int64 tensor or array; copied
    to the host): returns the expert -> rank map as a list."""
    import numpy as np
    c = np.ascontiguousarray(counts.cpu().numpy() if isinstance(counts, torch.Tensor) else counts,
                             dtype=np.uint64)
    if c.shape != (E, E):
        raise ValueError(f"counts: expected ({E}, {E}), got {c.shape}")
    out = (ctypes.c_int32 * E)()
    _check(lib().moe_fit_placement(E, ep, c.ctypes.data_as(ctypes.c_void_p), out),
           "moe_fit_placement")
    return list(out)


def permute(shape: Shape, x, row_token, stream=None):
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need_n(row_token, torch.int32, shape.R, "row_token")
    x_perm = torch.empty((shape.R, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    _check(lib().moe_permute(ctypes.byref(s), _p(x), _p(row_token), _p(x_perm), _stream(stream)),
           "moe_permute")
    return x_perm


def permute_by_token(shape: Shape, x, slot_row, stream=None):
    """moe_permute_by_token: x_perm via a token-order copy (x read once)."""
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need_n(slot_row, torch.int32, shape.R, "slot_row")
    x_perm = torch.empty((shape.R, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    _check(lib().moe_permute_by_token(ctypes.byref(s), _p(x), _p(slot_row), _p(x_perm),
                                      _stream(stream)), "moe_permute_by_token")
    return x_perm


def grouped_swiglu(shape: Shape, x_perm, expert_offsets, packed, ws, stream=None, engine=None):
    """moe_grouped_swiglu: returns (h [R,f], y_perm [R,d]).  engine (test
    hook, moe_debug_grouped_swiglu_engine): 1 = one CTA per tile, 2 = CTA
    pairs."""
    _need(x_perm, shape.dtype, (shape.R, shape.d), "x_perm")
    _need_n(expert_offsets, torch.int32, shape.E + 1, "expert_offsets")
    _need_packed(shape, packed)
    h = torch.empty((shape.R, shape.f), dtype=shape.dtype, device=x_perm.device)
    y_perm = torch.empty((shape.R, shape.d), dtype=shape.dtype, device=x_perm.device)
    s = shape.c
    if engine is None:
        _check(lib().moe_grouped_swiglu(ctypes.byref(s), _p(x_perm), _p(expert_offsets),
                                        _p(packed), _p(h), _p(y_perm), _p(ws), ws.numel(),
                                        _stream(stream)), "moe_grouped_swiglu")
    else:
        _check(lib().moe_debug_grouped_swiglu_engine(ctypes.byref(s), _p(x_perm), None,
                                                     _p(expert_offsets), _p(packed), _p(h),
                                                     _p(y_perm), _p(ws), ws.numel(), int(engine),
                                                     _stream(stream)),
               "moe_debug_grouped_swiglu_engine")
    return h, y_perm


def grouped_swiglu_gather(shape: Shape, x, row_token, expert_offsets, packed, ws, stream=None,
                          engine=None):
    """moe_grouped_swiglu_gather: (h, y_perm) with rows gathered from x.
    engine: as in grouped_swiglu (test hook)."""
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need_n(row_token, torch.int32, shape.R, "row_token")
    _need_n(expert_offsets, torch.int32, shape.E + 1, "expert_offsets")
    _need_packed(shape, packed)
    h = torch.empty((shape.R, shape.f), dtype=shape.dtype, device=x.device)
    y_perm = torch.empty((shape.R, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    if engine is None:
        _check(lib().moe_grouped_swiglu_gather(ctypes.byref(s), _p(x), _p(row_token),
                                               _p(expert_offsets), _p(packed), _p(h), _p(y_perm),
                                               _p(ws), ws.numel(), _stream(stream)),
               "moe_grouped_swiglu_gather")
    else:
        _check(lib().moe_debug_grouped_swiglu_engine(ctypes.byref(s), _p(x), _p(row_token),
                                                     _p(expert_offsets), _p(packed), _p(h),
                                                     _p(y_perm), _p(ws), ws.numel(), int(engine),
                                                     _stream(stream)),
               "moe_debug_grouped_swiglu_engine")
    return h, y_perm


def combine(shape: Shape, y_perm, slot_row, topk_gate=None, stream=None):
    _need(y_perm, shape.dtype, (shape.R, shape.d), "y_perm")
    _need_n(slot_row, torch.int32, shape.R, "slot_row")
    if topk_gate is not None:
        _need_n(topk_gate, torch.float32, shape.R, "topk_gate")
    y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=y_perm.device)
    s = shape.c
    _check(lib().moe_combine(ctypes.byref(s), _p(y_perm), _p(slot_row), _p(topk_gate), _p(y),
                             _stream(stream)), "moe_combine")
    return y


class ForwardBuffers:
    """Caller-owned intermediates of moe_forward, readable after the call."""

    def __init__(self, shape: Shape, device="cuda"):
        self.shape = shape
        R = shape.R
        self.logits = torch.empty((shape.T, shape.E), dtype=torch.float32, device=device)
        self.topk_idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device=device)
        self.topk_gate = torch.empty((shape.T, shape.k), dtype=torch.float32, device=device)
        self.layout = _layout_tensors(shape, device)
        self.x_perm = torch.empty((R, shape.d), dtype=shape.dtype, device=device)
        self.h = torch.empty((R, shape.f), dtype=shape.dtype, device=device)
        self.y_perm = torch.empty((R, shape.d), dtype=shape.dtype, device=device)

    @property
    def c(self) -> moe_forward_buffers:
        return moe_forward_buffers(_p(self.logits), _p(self.topk_idx), _p(self.topk_gate),
                                   _c_layout(self.layout), _p(self.x_perm), _p(self.h),
                                   _p(self.y_perm))


def _forward_args(shape: Shape, x, packed, bias, y, buffers):
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need_packed(shape, packed)
    _need_bias(shape, bias)
    if y is not None:
        _need(y, shape.dtype, (shape.T, shape.d), "y")
    if buffers is not None and buffers.shape != shape:
        raise ValueError(f"buffers: made for {buffers.shape}, not {shape}")


def forward(shape: Shape, x, packed, bias, ws, expert_rank=None, y=None,
            buffers: Optional[ForwardBuffers] = None, stream=None):
    """moe_forward: the whole layer; returns y [T, d]."""
    _forward_args(shape, x, packed, bias, y, buffers)
    if y is None:
        y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    b = buffers.c if buffers is not None else None
    _check(lib().moe_forward(ctypes.byref(s), _p(x), _p(packed), _p(bias),
                             _host_map(shape, expert_rank), _p(y),
                             ctypes.byref(b) if b is not None else None, _p(ws), ws.numel(),
                             _stream(stream)), "moe_forward")
    return y


FWD_COMBINE_IN_DOWN = 1  # moe_debug_forward_options: combine in the down GEMM's epilogue


def forward_options(shape: Shape, x, packed, bias, ws, options: int, expert_rank=None, y=None,
                    buffers: Optional[ForwardBuffers] = None, stream=None):
    """moe_debug_forward_options: moe_forward with the given option bits."""
    _forward_args(shape, x, packed, bias, y, buffers)
    if y is None:
        y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    b = buffers.c if buffers is not None else None
    _check(lib().moe_debug_forward_options(ctypes.byref(s), _p(x), _p(packed), _p(bias),
                                           _host_map(shape, expert_rank), _p(y),
                                           ctypes.byref(b) if b is not None else None, _p(ws),
                                           ws.numel(), int(options), _stream(stream)),
           "moe_debug_forward_options")
    return y


def forward_selection_bias(shape: Shape, x, packed, bias, selection_bias, ws, expert_rank=None,
                           y=None, buffers: Optional[ForwardBuffers] = None, stream=None):
    """moe_forward_selection_bias: the layer with a selection-only expert
    bias in the router; returns y [T, d]."""
    _forward_args(shape, x, packed, bias, y, buffers)
    _need(selection_bias, torch.float32, (shape.E,), "selection_bias")
    if y is None:
        y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    b = buffers.c if buffers is not None else None
    _check(lib().moe_forward_selection_bias(ctypes.byref(s), _p(x), _p(packed), _p(bias),
                                            _p(selection_bias), _host_map(shape, expert_rank),
                                            _p(y), ctypes.byref(b) if b is not None else None,
                                            _p(ws), ws.numel(), _stream(stream)),
           "moe_forward_selection_bias")
    return y


def forward_timed(shape: Shape, x, packed, bias, ws, events, expert_rank=None, y=None,
                  buffers: Optional[ForwardBuffers] = None, stream=None):
    """moe_forward_timed: moe_forward recording `events` (7 torch.cuda.Event
    with timing) around its stages (FORWARD_STAGES)."""
    _forward_args(shape, x, packed, bias, y, buffers)
    if len(events) != len(FORWARD_STAGES) + 1:
        raise ValueError("need one event per stage plus one")
    if y is None:
        y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=x.device)
    ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    s = shape.c
    b = buffers.c if buffers is not None else None
    _check(lib().moe_forward_timed(ctypes.byref(s), _p(x), _p(packed), _p(bias),
                                   _host_map(shape, expert_rank), _p(y),
                                   ctypes.byref(b) if b is not None else None, _p(ws), ws.numel(),
                                   ev, _stream(stream)), "moe_forward_timed")
    return y


def forward_routed(shape: Shape, x, packed, topk_idx, topk_gate, ws, expert_rank=None, y=None,
                   buffers: Optional[ForwardBuffers] = None, stream=None):
    """moe_forward_routed: the layer below the router on a given routing
    (topk_idx [T,k] int32, topk_gate [T,k] fp32 or None for unit gates);
    returns y [T, d]."""
    _forward_args(shape, x, packed, None, y, buffers)
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    if topk_gate is not None:
        _need(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    if y is None:
        y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=x.device)
    s = shape.c
    b = buffers.c if buffers is not None else None
    _check(lib().moe_forward_routed(ctypes.byref(s), _p(x), _p(packed), _p(topk_idx),
                                    _p(topk_gate), _host_map(shape, expert_rank), _p(y),
                                    ctypes.byref(b) if b is not None else None, _p(ws),
                                    ws.numel(), _stream(stream)), "moe_forward_routed")
    return y


def ep_pack(shape: Shape, x, topk_idx, topk_gate, layout: dict, send_rows: int,
            expert_rank=None, stream=None):
    """moe_ep_pack: (send_x [send_rows, d], send_idx [send_rows, k] int32,
    send_gate [send_rows, k] fp32) for this rank's send plan."""
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    if topk_gate is not None:
        _need(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    _need_n(layout["rank_offsets"], torch.int32, shape.ep + 1, "rank_offsets")
    dev = x.device
    send_x = torch.empty((send_rows, shape.d), dtype=shape.dtype, device=dev)
    send_idx = torch.empty((send_rows, shape.k), dtype=torch.int32, device=dev)
    send_gate = torch.empty((send_rows, shape.k), dtype=torch.float32, device=dev)
    lay = _c_layout(layout)
    s = shape.c
    _check(lib().moe_ep_pack(ctypes.byref(s), _p(x), _p(topk_idx), _p(topk_gate),
                             _host_map(shape, expert_rank), ctypes.byref(lay), _p(send_x),
                             _p(send_idx), _p(send_gate), int(send_rows), _stream(stream)),
           "moe_ep_pack")
    return send_x, send_idx, send_gate


def ep_expert_workspace(shape: Shape, device="cuda") -> torch.Tensor:
    n = ctypes.c_size_t()
    s = shape.c
    _check(lib().moe_ep_expert_workspace_size(ctypes.byref(s), ctypes.byref(n)),
           "moe_ep_expert_workspace_size")
    return torch.zeros(n.value, dtype=torch.uint8, device=device)


def ep_expert_forward(shape: Shape, recv_x, recv_idx, recv_gate, packed_local, ws, stream=None):
    """moe_ep_expert_forward over shape.T received rows: y_ret [T, d]."""
    _need(recv_x, shape.dtype, (shape.T, shape.d), "recv_x")
    _need(recv_idx, torch.int32, (shape.T, shape.k), "recv_idx")
    _need(recv_gate, torch.float32, (shape.T, shape.k), "recv_gate")
    y_ret = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=recv_x.device)
    s = shape.c
    _check(lib().moe_ep_expert_forward(ctypes.byref(s), _p(recv_x), _p(recv_idx), _p(recv_gate),
                                       _p(packed_local), _p(y_ret), _p(ws), ws.numel(),
                                       _stream(stream)), "moe_ep_expert_forward")
    return y_ret


def ep_home_combine(shape: Shape, y_back, slot_send_row, stream=None):
    """moe_ep_home_combine: y [T, d] from the returned rows."""
    _need_n(slot_send_row, torch.int32, shape.R, "slot_send_row")
    if y_back.dtype != shape.dtype or y_back.dim() != 2 or y_back.shape[1] != shape.d:
        raise ValueError(f"y_back: expected {shape.dtype} [rows, {shape.d}]")
    y = torch.empty((shape.T, shape.d), dtype=shape.dtype, device=y_back.device)
    s = shape.c
    _check(lib().moe_ep_home_combine(ctypes.byref(s), _p(y_back), _p(slot_send_row),
                                     int(y_back.shape[0]), _p(y), _stream(stream)),
           "moe_ep_home_combine")
    return y


def ep_dispatch_peer(shape: Shape, x, topk_idx, topk_gate, layout: dict, dests,
                     expert_rank=None, stream=None):
    """moe_ep_dispatch_peer: this rank's send rows stored straight into the
    destination ranks' receive buffers.  dests: P tuples (recv_x, recv_idx,
    recv_gate, row0, rows), the buffers as tensors (or None for rows == 0)
    addressable from this process."""
    _need(x, shape.dtype, (shape.T, shape.d), "x")
    _need(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    if topk_gate is not None:
        _need(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    _need_n(layout["rank_offsets"], torch.int32, shape.ep + 1, "rank_offsets")
    if len(dests) != shape.ep:
        raise ValueError(f"dests: expected {shape.ep} entries")
    arr = (moe_ep_peer_dest * shape.ep)()
    for r, (rx, ri, rg, row0, rows) in enumerate(dests):
        if rows > 0:
            for t, dt, w, nm in ((rx, shape.dtype, shape.d, "recv_x"),
                                 (ri, torch.int32, shape.k, "recv_idx"),
                                 (rg, torch.float32, shape.k, "recv_gate")):
                if (t.dtype != dt or t.dim() != 2 or t.shape[1] != w or not t.is_contiguous()
                        or row0 + rows > t.shape[0]):
                    raise ValueError(f"{nm} of rank {r}: expected contiguous {dt} "
                                     f"[>= {row0 + rows}, {w}]")
        arr[r] = moe_ep_peer_dest(_p(rx), _p(ri), _p(rg), int(row0), int(rows))
    lay = _c_layout(layout)
    s = shape.c
    _check(lib().moe_ep_dispatch_peer(ctypes.byref(s), _p(x), _p(topk_idx), _p(topk_gate),
                                      _host_map(shape, expert_rank), ctypes.byref(lay), arr,
                                      _stream(stream)), "moe_ep_dispatch_peer")


def ep_expert_forward_peer(shape: Shape, recv_x, recv_idx, recv_gate, packed_local, rets, ws,
                           stream=None):
    """moe_ep_expert_forward_peer over shape.T received rows: the return rows
    stored straight into the source ranks' buffers.  rets: P tuples (y_back,
    row0, rows), y_back a tensor (or None for rows == 0) addressable from
    this process."""
    _need(recv_x, shape.dtype, (shape.T, shape.d), "recv_x")
    _need(recv_idx, torch.int32, (shape.T, shape.k), "recv_idx")
    _need(recv_gate, torch.float32, (shape.T, shape.k), "recv_gate")
    if len(rets) != shape.ep:
        raise ValueError(f"rets: expected {shape.ep} entries")
    arr = (moe_ep_peer_return * shape.ep)()
    for r, (yb, row0, rows) in enumerate(rets):
        if rows > 0 and (yb.dtype != shape.dtype or yb.dim() != 2 or yb.shape[1] != shape.d
                         or not yb.is_contiguous() or row0 + rows > yb.shape[0]):
            raise ValueError(f"y_back of rank {r}: expected contiguous {shape.dtype} "
                             f"[>= {row0 + rows}, {shape.d}]")
        arr[r] = moe_ep_peer_return(_p(yb), int(row0), int(rows))
    s = shape.c
    _check(lib().moe_ep_expert_forward_peer(ctypes.byref(s), _p(recv_x), _p(recv_idx),
                                            _p(recv_gate), _p(packed_local), arr, _p(ws),
                                            ws.numel(), _stream(stream)),
           "moe_ep_expert_forward_peer")


def ep_signal_wait(flags, rank: int, epoch: int, ws, wait_limit_ns=None, stream=None):
    """moe_ep_signal_wait (or its test hook with wait_limit_ns): flags = every
    rank's flag array (uint64 [P] tensors, stored as int64), addressable
    from this process."""
    P = len(flags)
    arr = (ctypes.c_void_p * P)(*[_p(f) for f in flags])
    for f in flags:
        if f.dtype != torch.int64 or f.numel() < P:
            raise ValueError(f"flags: expected int64 tensors of >= {P} slots")
    if wait_limit_ns is None:
        _check(lib().moe_ep_signal_wait(arr, rank, P, epoch, _p(ws), _stream(stream)),
               "moe_ep_signal_wait")
    else:
        _check(lib().moe_debug_ep_signal_wait(arr, rank, P, epoch, _p(ws), int(wait_limit_ns),
                                              _stream(stream)), "moe_debug_ep_signal_wait")


def get_device_status(ws, stream=None) -> int:
    out = ctypes.c_int(0)
    _check(lib().moe_get_device_status(_p(ws), _stream(stream), ctypes.byref(out)),
           "moe_get_device_status")
    return out.value


def check_device_status(ws, stream=None):
    st = get_device_status(ws, stream)
    if st != MOE_OK:
        raise MoeError(st, "device status")
