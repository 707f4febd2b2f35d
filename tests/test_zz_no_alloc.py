"""moe_dispatch_layout_static: the dispatch layout for callers that cannot
allocate device memory (for example an operator whose device memory is
planned ahead and who is handed only inputs and outputs), with its scratch
in the library's own fixed device array instead of a caller workspace.

Called straight through the C ABI (ctypes), compared with the workspace
entry point moe_dispatch_layout on the same inputs, over calls in a row that
reuse the shared array.  The layout is integer work, so the comparison is
exact.  This file sorts last so that a run stopping at its first failure has
run every other test already.
"""
import ctypes

import pytest
import torch

import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

pytestmark = pytest.mark.gpu

KEYS = ("expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
        "rank_offsets", "slot_send_row", "stats")


def _static_call(shape, idx, rmap):
    """One moe_dispatch_layout_static call through ctypes; returns outputs."""
    L = moe.lib()
    out = moe._layout_tensors(shape, idx.device)
    lay = moe._c_layout(out)
    status = torch.full((1,), -1, dtype=torch.int32, device=idx.device)
    s = shape.c
    cmap = None if rmap is None else (ctypes.c_int32 * shape.E)(*rmap)
    rc = L.moe_dispatch_layout_static(ctypes.byref(s), ctypes.c_void_p(idx.data_ptr()), cmap,
                                      ctypes.byref(lay), ctypes.c_void_p(status.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == moe.MOE_OK, moe.STATUS_NAMES.get(rc, rc)
    return out, status


def _workspace_call(shape, idx, rmap):
    ws = moe.workspace(shape)
    out = moe.dispatch_layout(shape, idx, ws, expert_rank=rmap)
    assert moe.get_device_status(ws) == moe.MOE_OK
    return out


def _compare(shape, a, b):
    for key in KEYS:
        if key not in a:
            continue
        assert torch.equal(a[key], b[key]), key
    if shape.ep > 1:
        n = int(a["rank_offsets"][-1])
        assert torch.equal(a["send_token"][:n], b["send_token"][:n])


def test_static_layout_matches_workspace_layout_on_consecutive_calls():
    cases = [
        (16384, 64, 4, 8, None),                                   # the fine-grained workload
        (5000, 64, 6, 32, W.permutation_placement(64, 32, seed=3)),
        (20000, 128, 8, 16, None),
        (16384, 64, 4, 8, None),                                   # repeat after larger calls
    ]
    for T, E, k, ep, rmap in cases:
        shape = moe.Shape(T=T, d=256, E=E, k=k, f=64, ep=ep)
        idx = W.uniform_routing(T, E, k, seed=T + E).cuda()
        ref = _workspace_call(shape, idx, rmap)
        for _ in range(2):  # two calls in a row on the shared array
            got, status = _static_call(shape, idx, rmap)
            torch.cuda.synchronize()
            assert int(status.item()) == moe.MOE_OK
            _compare(shape, got, ref)


def test_static_layout_rejects_shapes_beyond_its_scratch():
    L = moe.lib()
    s = moe.Shape(T=200000, d=256, E=256, k=16, f=64, ep=256).c
    lay = moe.moe_layout(*([ctypes.c_void_p(256)] * 9))
    rc = L.moe_dispatch_layout_static(ctypes.byref(s), ctypes.c_void_p(256), None,
                                      ctypes.byref(lay), None, None)
    assert rc == moe.MOE_ERR_WORKSPACE


def test_static_layout_status_does_not_leak_into_the_next_call():
    """The shared array keeps the previous call's contents, status word
    included.  A call that meets an expert index outside [0, E) reports
    MOE_ERR_DEVICE_INDEX; the next, valid call clears that word first and
    reports MOE_OK with the same layout as the workspace entry point."""
    T, E, k, ep = 3000, 64, 4, 8
    shape = moe.Shape(T=T, d=256, E=E, k=k, f=64, ep=ep)
    good = W.uniform_routing(T, E, k, seed=17).cuda()
    bad = good.clone()
    bad[T // 2, 1] = E
    _, status = _static_call(shape, bad, None)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.MOE_ERR_DEVICE_INDEX
    ref = _workspace_call(shape, good, None)
    for _ in range(2):
        got, status = _static_call(shape, good, None)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.MOE_OK
        _compare(shape, got, ref)
