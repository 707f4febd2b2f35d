"""The grouped GEMM on CTA pairs (256-row tiles, tcgen05 cta_group::2):
h and y_perm bit-identical to the one-CTA-per-tile engine (every output is
summed over the same K blocks in the same order), on group sizes that put a
pair tile's second half partly or wholly past its group (1, 127, 128, 129,
255, 256, 257, 383 rows), empty groups and whole workloads; and within the
oracle's tolerance on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import TOL, Case

pytestmark = pytest.mark.gpu


def _both(shape, x_perm, off, packed):
    ws = moe.workspace(shape)
    h1, y1 = moe.grouped_swiglu(shape, x_perm, off, packed, ws, engine=1)
    h2, y2 = moe.grouped_swiglu(shape, x_perm, off, packed, ws, engine=2)
    h0, y0 = moe.grouped_swiglu(shape, x_perm, off, packed, ws)
    moe.check_device_status(ws)
    return (h1, y1), (h2, y2), (h0, y0)


@pytest.mark.parametrize("cfg", [3, 5])
def test_pair_engine_bit_identical_on_ragged_groups(cfg):
    c = Case(cfg, T=64, near_ties=False)
    w = c.w
    sizes = [1, 127, 128, 129, 255, 256, 257, 383, 0, 512, 3]
    sizes = (sizes * ((w.E + len(sizes) - 1) // len(sizes)))[: w.E]
    off = torch.tensor([0] + list(np.cumsum(sizes)), dtype=torch.int32)
    R = int(off[-1])
    # k rows per token: choose T so that T * k covers R (extra rows unused)
    T = (R + w.k - 1) // w.k
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    g = torch.Generator().manual_seed(cfg)
    x_perm = torch.randn((T * w.k, w.d), generator=g).to(w.torch_dtype).cuda()
    off_full = off.clone()
    off_full[-1] = R  # rows past R belong to no group
    a, b, d = _both(shape, x_perm, off_full.cuda(), c.packed)
    assert torch.equal(a[0][:R], b[0][:R]) and torch.equal(a[1][:R], b[1][:R])
    assert torch.equal(b[0][:R], d[0][:R]) and torch.equal(b[1][:R], d[1][:R])
    rows = np.array(sorted({int(off[e]) for e in range(w.E) if sizes[e]} |
                           {int(off[e + 1]) - 1 for e in range(w.E) if sizes[e]} |
                           set(range(0, R, 97))))
    ref = oracle.grouped_swiglu(x_perm.cpu(), off.numpy(), c.wg, c.wu, c.wd, rows=rows)
    yg = b[1].cpu().double().numpy()[rows]
    assert np.abs(yg - ref).max() <= TOL["bf16"] * np.abs(ref).max()


@pytest.mark.parametrize("cfg,T", [(3, 4096), (4, 2048), (5, 2048)])
def test_pair_engine_bit_identical_on_workload_routing(cfg, T):
    c = Case(cfg, T=T, near_ties=False)
    ws = moe.workspace(c.shape)
    _, idx, _ = moe.route(c.shape, c.dx, c.packed, c.dbias, ws)
    lay = moe.dispatch_layout(c.shape, idx, ws)
    x_perm = moe.permute(c.shape, c.dx, lay["row_token"])
    a, b, d = _both(c.shape, x_perm, lay["expert_offsets"], c.packed)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(b[1], d[1])


@pytest.mark.parametrize("cfg,T", [(3, 3000), (5, 1500)])
def test_pair_gather_equals_permute_then_grouped(cfg, T):
    """The permute fused into the gate/up operand load: the pair engine's
    TMA gather4 of x rows, the one-CTA engine's cp.async gather, and the
    separate permute + grouped GEMM give the same h and y_perm bit for bit,
    with some rows of x picked by no expert group's tail (ragged groups)."""
    c = Case(cfg, T=T, near_ties=False)
    ws = moe.workspace(c.shape)
    _, idx, _ = moe.route(c.shape, c.dx, c.packed, c.dbias, ws)
    lay = moe.dispatch_layout(c.shape, idx, ws)
    x_perm = moe.permute(c.shape, c.dx, lay["row_token"])
    h0, y0 = moe.grouped_swiglu(c.shape, x_perm, lay["expert_offsets"], c.packed, ws, engine=2)
    outs = [moe.grouped_swiglu_gather(c.shape, c.dx, lay["row_token"], lay["expert_offsets"],
                                      c.packed, ws, engine=e) for e in (1, 2, None)]
    moe.check_device_status(ws)
    for h, y in outs:
        assert torch.equal(h, h0) and torch.equal(y, y0)
