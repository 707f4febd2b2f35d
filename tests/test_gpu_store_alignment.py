"""The GEMMs' unstaged epilogues write each row's 64-byte column group as
two 32-byte stores when the output and its row pitch are 32-byte aligned,
and as four 16-byte stores otherwise (the boundary asks only 16-byte
alignment of h and y_perm).  Outputs placed 16 bytes past a 32-byte
boundary take the second path; they must equal the aligned call's bit for
bit, on both engines (one CTA per tile; CTA pairs) and with the gathered
gate/up GEMM, and stay within the oracle's tolerance."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe

from util import TOL, Case

pytestmark = pytest.mark.gpu


def _offset_buffer(rows, cols, dtype, shift):
    """A [rows, cols] view whose first element sits `shift` bytes past a
    256-byte boundary."""
    esz = torch.empty((), dtype=dtype).element_size()
    raw = torch.empty(rows * cols * esz + 256, dtype=torch.uint8, device="cuda")
    assert raw.data_ptr() % 256 == 0
    return raw[shift: shift + rows * cols * esz].view(dtype).view(rows, cols)


def _call(shape, x_perm, off, packed, ws, h, y, engine):
    s = shape.c
    r = moe.lib().moe_debug_grouped_swiglu_engine(
        ctypes.byref(s), ctypes.c_void_p(x_perm.data_ptr()), None,
        ctypes.c_void_p(off.data_ptr()), ctypes.c_void_p(packed.data_ptr()),
        ctypes.c_void_p(h.data_ptr()), ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(ws.data_ptr()), ws.numel(), engine, None)
    assert r == moe.MOE_OK, r


def _call_gather(shape, x, row_token, off, packed, ws, h, y):
    s = shape.c
    r = moe.lib().moe_grouped_swiglu_gather(
        ctypes.byref(s), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(row_token.data_ptr()),
        ctypes.c_void_p(off.data_ptr()), ctypes.c_void_p(packed.data_ptr()),
        ctypes.c_void_p(h.data_ptr()), ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert r == moe.MOE_OK, r


@pytest.mark.parametrize("engine", [1, 2])
def test_unaligned_outputs_equal_aligned(engine):
    # top-2 workload's expert shapes (d = 2048: 32 k-blocks, unstaged gate/up;
    # f = 1024: the down GEMM unstaged on pairs), ragged groups
    c = Case(3, T=700, near_ties=False)
    shape, w = c.shape, c.w
    ws = moe.workspace(shape)
    _, idx, _ = moe.route(shape, c.dx, c.packed, c.dbias, ws)
    lay = moe.dispatch_layout(shape, idx, ws)
    x_perm = moe.permute(shape, c.dx, lay["row_token"])
    off = lay["expert_offsets"]
    outs = {}
    for shift in (0, 16):
        h = _offset_buffer(shape.R, w.f, w.torch_dtype, shift)
        y = _offset_buffer(shape.R, w.d, w.torch_dtype, shift)
        assert (h.data_ptr() % 32 == 0) == (shift == 0)
        _call(shape, x_perm, off, c.packed, ws, h, y, engine)
        moe.check_device_status(ws)
        outs[shift] = (h.clone(), y.clone())
    assert torch.equal(outs[0][0], outs[16][0])
    assert torch.equal(outs[0][1], outs[16][1])
    rows = np.arange(0, shape.R, 37)
    ref = oracle.grouped_swiglu(x_perm.cpu(), off.cpu().numpy(), c.wg, c.wu, c.wd, rows=rows)
    yg = outs[16][1].cpu().double().numpy()[rows]
    assert np.abs(yg - ref).max() <= TOL["bf16"] * np.abs(ref).max()


def test_unaligned_outputs_equal_aligned_gather():
    c = Case(4, T=500, near_ties=False)
    shape, w = c.shape, c.w
    ws = moe.workspace(shape)
    _, idx, _ = moe.route(shape, c.dx, c.packed, c.dbias, ws)
    lay = moe.dispatch_layout(shape, idx, ws)
    outs = {}
    for shift in (0, 16):
        h = _offset_buffer(shape.R, w.f, w.torch_dtype, shift)
        y = _offset_buffer(shape.R, w.d, w.torch_dtype, shift)
        _call_gather(shape, c.dx, lay["row_token"], lay["expert_offsets"], c.packed, ws, h, y)
        moe.check_device_status(ws)
        outs[shift] = (h.clone(), y.clone())
    assert torch.equal(outs[0][0], outs[16][0])
    assert torch.equal(outs[0][1], outs[16][1])
