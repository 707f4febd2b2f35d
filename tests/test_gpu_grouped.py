"""GPU parity of moe_grouped_swiglu (tcgen05 grouped GEMMs for bf16, FMA
kernels for fp32) against the oracle's grouped SwiGLU, on expert-grouped
rows built on the CPU: ragged experts (tails of every size, empty experts,
one expert holding most rows) and several M / N tiles."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import TOL

pytestmark = pytest.mark.gpu


def _rows(w, T, skew, seed):
    if skew:
        g = torch.Generator().manual_seed(seed)
        p = torch.arange(1, w.E + 1, dtype=torch.float64).pow(-1.5)
        idx = torch.stack([torch.multinomial(p, w.k, replacement=False, generator=g) for _ in range(T)]).int()
    else:
        idx = W.uniform_routing(T, w.E, w.k, seed=seed)
    return idx


@pytest.mark.parametrize("cfg,T,skew", [(1, 2048, False), (2, 3000, False), (2, 1000, True),
                                        (3, 600, False), (3, 2000, True), (4, 300, False),
                                        (5, 200, False), (5, 333, True)])
def test_grouped_swiglu_matches_oracle(cfg, T, skew):
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, T=T)
    idx = _rows(w, T, skew, seed=T + cfg)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    x_perm = x[torch.from_numpy(lay["row_token"]).long()].contiguous()
    wr = W.make_router(w)
    wg, wu, wd = W.make_experts(w)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape)
    off = torch.from_numpy(lay["expert_offsets"])
    h, y_perm = moe.grouped_swiglu(shape, x_perm.cuda(), off.cuda(), packed, ws)
    moe.check_device_status(ws)
    R = T * w.k
    # sampled rows for the larger shapes: every expert's first and last row
    # plus a seeded sample
    if R * w.d * w.f > 4e9:
        pick = set(W.sample_tokens(R, 256, seed=1).tolist())
        for e in range(w.E):
            if off[e + 1] > off[e]:
                pick |= {int(off[e]), int(off[e + 1]) - 1}
        rows = np.array(sorted(pick))
    else:
        rows = np.arange(R)
    ref = oracle.grouped_swiglu(x_perm, off.numpy(), wg, wu, wd, rows=rows)
    yg = y_perm.cpu().double().numpy()[rows]
    scale = np.abs(ref).max()
    err = np.abs(yg - ref).max()
    assert err <= TOL[w.dtype] * scale, (err, scale)
    # every row was written (no NaN / garbage from unwritten memory)
    assert torch.isfinite(y_perm.float()).all()


def test_grouped_swiglu_single_expert_dense():
    """E = 1 (one group of all rows) through the tensor-core path, against a
    float64 dense SwiGLU."""
    T, d, f = 777, 256, 128
    g = torch.Generator().manual_seed(3)
    x = torch.randn(T, d, generator=g).bfloat16()
    wg = (torch.randn(1, d, f, generator=g) / 16).bfloat16()
    wu = (torch.randn(1, d, f, generator=g) / 16).bfloat16()
    wd = (torch.randn(1, f, d, generator=g) / 11).bfloat16()
    wr = torch.zeros(d, 1).bfloat16()
    shape = moe.Shape(T=T, d=d, E=1, k=1, f=f)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape)
    off = torch.tensor([0, T], dtype=torch.int32)
    h, y = moe.grouped_swiglu(shape, x.cuda(), off.cuda(), packed, ws)
    xd = x.double()
    hr = torch.nn.functional.silu(xd @ wg[0].double()) * (xd @ wu[0].double())
    yr = hr @ wd[0].double()
    assert (h.cpu().double() - hr).abs().max() <= 1e-2 * hr.abs().max()
    assert (y.cpu().double() - yr).abs().max() <= 2e-2 * yr.abs().max()


def test_grouped_swiglu_deterministic():
    w = W.WORKLOADS[3]
    T = 1500
    x = W.make_x(w, T=T)
    idx = W.uniform_routing(T, w.E, w.k, seed=2)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    x_perm = x[torch.from_numpy(lay["row_token"]).long()].contiguous().cuda()
    wg, wu, wd = W.make_experts(w)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f)
    packed = moe.pack_weights(shape, W.make_router(w).cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape)
    off = torch.from_numpy(lay["expert_offsets"]).cuda()
    a = moe.grouped_swiglu(shape, x_perm, off, packed, ws)[1]
    b = moe.grouped_swiglu(shape, x_perm, off, packed, ws)[1]
    assert torch.equal(a, b)


@pytest.mark.parametrize("cfg,T,skew", [(2, 3000, False), (2, 1000, True), (3, 777, False),
                                        (4, 300, True), (5, 129, False)])
def test_gather_fused_permute_matches(cfg, T, skew):
    """The gate/up GEMM reading rows of x through row_token (TMA gather)
    gives bit-for-bit the outputs of moe_permute + moe_grouped_swiglu, and
    matches the oracle."""
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, T=T)
    idx = _rows(w, T, skew, seed=T + 2 * cfg)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    rt = torch.from_numpy(lay["row_token"])
    wg, wu, wd = W.make_experts(w)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    packed = moe.pack_weights(shape, W.make_router(w).cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape)
    off = torch.from_numpy(lay["expert_offsets"]).cuda()
    dx, drt = x.cuda(), rt.cuda()
    h1, y1 = moe.grouped_swiglu_gather(shape, dx, drt, off, packed, ws)
    h0, y0 = moe.grouped_swiglu(shape, moe.permute(shape, dx, drt), off, packed, ws)
    moe.check_device_status(ws)
    assert torch.equal(h1, h0)
    assert torch.equal(y1, y0)
    R = T * w.k
    rows = np.arange(R) if R * w.d * w.f < 4e9 else np.unique(W.sample_tokens(R, 200, seed=2).numpy())
    ref = oracle.grouped_swiglu(x[rt.long()], lay["expert_offsets"], wg, wu, wd, rows=rows)
    err = np.abs(y1.cpu().double().numpy()[rows] - ref).max()
    assert err <= TOL[w.dtype] * np.abs(ref).max()
