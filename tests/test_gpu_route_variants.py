"""GPU parity of the routing variants and router observability against the
oracle's pinned functions:

- selection-only expert bias ("Expert Coupling in MoE Pretraining", Fig. 11:
  the auxiliary-loss-free router): indices bit-exact against
  oracle.topk_selection_bias on the same fp32 logits, gates within 1e-6, in
  the given-logits kernel, the fused bf16 router and the whole forward;
- router statistics ("MoE Pretraining: Parallelism Layout Changes the Model,
  Not Quality", Finding 3 and Practical Implications): per-token margins
  equal to oracle.margin on the same fp32 values, the near-tie count, and
  the differences against a recorded routing equal to
  oracle.routing_changes;
- expert capacity ("Revisiting MoE and Dense Speed-Accuracy Comparisons",
  2.1): the keep mask bit-exact against oracle.capacity_keep, and the layer
  output with the dropped assignments removed against the oracle;
- top-16 routing over 64 fine-grained experts (the "MoE Pretraining ..."
  page, Finding 4): the whole forward against the oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import NEAR_TIE, TOL, Case, check_output, routing_mismatches

pytestmark = pytest.mark.gpu


def _logits_with_ties(T, E, seed):
    g = torch.Generator().manual_seed(seed)
    l = torch.randn((T, E), generator=g)
    # exact ties, signed zeros and repeated values in a third of the rows
    rows = torch.arange(0, T, 3)
    l[rows, 1] = l[rows, 0]
    l[rows[::2], 2] = 0.0
    l[rows[::2], 3] = -0.0
    l[rows[1::2], E - 1] = l[rows[1::2], 0]
    return l.contiguous()


@pytest.mark.parametrize("T,E,k", [(1000, 16, 4), (777, 64, 6), (513, 128, 8), (300, 256, 16),
                                   (64, 64, 16), (5, 8, 8)])
def test_selection_bias_given_logits(T, E, k):
    l = _logits_with_ties(T, E, T + E)
    g = torch.Generator().manual_seed(k)
    b = (torch.randn(E, generator=g) * 0.5).float()
    b[: E // 4] = 0.0  # some experts unbiased: ties stay ties
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    ws = moe.workspace(shape)
    _, idx, gate = moe.route_selection_bias(shape, None, None, None, b.cuda(), ws, logits=l.cuda())
    assert moe.get_device_status(ws) == moe.MOE_OK
    ri, rg = oracle.topk_selection_bias(l.numpy(), b.numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ri)
    np.testing.assert_allclose(gate.cpu().double().numpy(), rg, atol=1e-6, rtol=0)
    # a zero bias is plain top-k, bit for bit
    _, i0, g0 = moe.route(shape, None, None, None, ws, logits=l.cuda())
    _, i1, g1 = moe.route_selection_bias(shape, None, None, None, torch.zeros(E).cuda(), ws,
                                         logits=l.cuda())
    assert torch.equal(i0, i1) and torch.equal(g0, g1)


@pytest.mark.parametrize("cfg,T", [(2, 1000), (3, 300), (5, 257), (2, 19205)])
def test_selection_bias_fused_router(cfg, T):
    """bf16: the fused router picks on logits + bias and weights by logits;
    its logits equal moe_route's bit for bit (the bias is not added)."""
    c = Case(cfg, T=T, near_ties=False)
    w = c.w
    g = torch.Generator().manual_seed(cfg)
    b = (torch.randn(w.E, generator=g) * 0.05).float().cuda()
    ws = moe.workspace(c.shape)
    l0, _, _ = moe.route(c.shape, c.dx, c.packed, c.dbias, ws)
    l1, idx, gate = moe.route_selection_bias(c.shape, c.dx, c.packed, c.dbias, b, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    assert torch.equal(l0, l1)
    ri, rg = oracle.topk_selection_bias(l1.cpu().numpy(), b.cpu().numpy(), w.k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ri)
    np.testing.assert_allclose(gate.cpu().double().numpy(), rg, atol=1e-6, rtol=0)


@pytest.mark.parametrize("cfg,T", [(1, 500), (2, 1500), (3, 513)])
def test_selection_bias_forward(cfg, T):
    """The forward with a selection-only bias: its routing is the oracle's
    biased selection of its own logits, and its output equals the routed
    forward on that routing bit for bit and the oracle's within tolerance."""
    c = Case(cfg, T=T, near_ties=False)
    w = c.w
    g = torch.Generator().manual_seed(cfg + 1)
    b = (torch.randn(w.E, generator=g) * 0.05).float().cuda()
    shape = c.shape_ep(w.eps[0])
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y = moe.forward_selection_bias(shape, c.dx, c.packed, c.dbias, b, ws, buffers=buf)
    moe.check_device_status(ws)
    ri, rg = oracle.topk_selection_bias(buf.logits.cpu().numpy(), b.cpu().numpy(), w.k)
    np.testing.assert_array_equal(buf.topk_idx.cpu().numpy(), ri)
    y1 = moe.forward_routed(shape, c.dx, c.packed, buf.topk_idx, buf.topk_gate, ws)
    moe.check_device_status(ws)
    assert torch.equal(y, y1)
    lay = oracle.dispatch_layout(ri, w.E, shape.ep)
    np.testing.assert_array_equal(buf.layout["slot_row"].cpu().numpy(), lay["slot_row"])
    ref = oracle.moe_output(c.x, ri, rg, c.wg, c.wu, c.wd)
    check_output(y, ref, w.dtype)


@pytest.mark.parametrize("T,E,k", [(2000, 16, 4), (1500, 64, 2), (700, 128, 8), (300, 256, 16),
                                   (100, 8, 8)])
def test_router_stats_margin_and_changes(T, E, k):
    l = _logits_with_ties(T, E, 3 * T + k)
    # plant near-ties: the (k+1)-th value a hair below the k-th
    g = torch.Generator().manual_seed(T)
    pick = torch.randperm(T, generator=g)[: T // 10]
    if k < E:
        for t in pick.tolist():
            o = torch.argsort(-l[t], stable=True)
            l[t, o[k]] = torch.nextafter(l[t, o[k - 1]], torch.tensor(-np.inf))
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    ws = moe.workspace(shape)
    _, idx, _ = moe.route(shape, None, None, None, ws, logits=l.cuda())
    rec = idx.clone()
    rec[::7, 0] = (rec[::7, 0] + 1) % E       # some recorded rows differ
    rec[::11] = torch.flip(rec[::11], [1])    # slot order only
    counts, margin = moe.router_stats(shape, l.cuda(), idx, rec, want_margin=True)
    m_ref = oracle.margin(l.numpy().astype(np.float64), k)
    m_gpu = margin.cpu().numpy()
    assert (m_gpu == m_ref).all(), np.abs(m_gpu - m_ref).max()
    assert counts["tokens"] == T
    assert counts["near_tie_tokens"] == int((m_ref < 1e-5).sum())
    if k < E:
        assert counts["near_tie_tokens"] >= len(pick)
    ch = oracle.routing_changes(idx.cpu().numpy(), rec.cpu().numpy())
    assert (counts["changed_tokens"], counts["changed_experts"], counts["changed_slots"]) == \
        (ch["tokens"], ch["experts"], ch["slots"])
    # no recorded routing: the change counters stay zero
    c0, _ = moe.router_stats(shape, l.cuda(), idx, None, threshold=0.5)
    assert c0["changed_tokens"] == c0["changed_experts"] == c0["changed_slots"] == 0
    assert c0["near_tie_tokens"] == int((m_ref < 0.5).sum())


def test_router_stats_with_selection_bias():
    """The margin of the biased router is taken on its selection key, the
    fp32 sum logits + bias."""
    T, E, k = 900, 64, 4
    l = _logits_with_ties(T, E, 5)
    b = (torch.randn(E, generator=torch.Generator().manual_seed(9)) * 0.3).float()
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    counts, margin = moe.router_stats(shape, l.cuda(), selection_bias=b.cuda(), want_margin=True)
    key = (l.numpy() + b.numpy()[None, :]).astype(np.float32).astype(np.float64)
    m_ref = oracle.margin(key, k)
    assert (margin.cpu().numpy() == m_ref).all()
    assert counts["near_tie_tokens"] == int((m_ref < 1e-5).sum())


def test_router_stats_of_the_forward_routing_with_injected_near_ties():
    """The top-6 workload's injected near-ties, counted by the GPU on the
    forward's own logits, match the oracle's count on the same values."""
    c = Case(4, T=2048)
    shape = c.shape_ep(32)
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    moe.forward(shape, c.dx, c.packed, None, ws, buffers=buf,
                expert_rank=W.permutation_placement(64, 32, 0))
    moe.check_device_status(ws)
    counts, margin = moe.router_stats(shape, buf.logits, want_margin=True)
    m_ref = oracle.margin(buf.logits.cpu().numpy().astype(np.float64), c.w.k)
    assert (margin.cpu().numpy() == m_ref).all()
    assert counts["near_tie_tokens"] == int((m_ref < NEAR_TIE).sum())
    # most injected tokens are still near-ties in the GPU's fp32 logits
    assert counts["near_tie_tokens"] >= len(c.near_tie_tokens) // 2


@pytest.mark.parametrize("T,E,k,cf", [(1000, 16, 4, 1.0), (2000, 64, 2, 1.25), (513, 128, 8, 2.0),
                                      (300, 64, 16, 0.5), (40, 8, 2, 0.1),
                                      # several 1024-token chunks, ragged last chunk
                                      (5000, 128, 8, 1.0), (20001, 64, 4, 1.1),
                                      (3073, 256, 16, 0.75)])
def test_capacity_keep_bit_exact(T, E, k, cf):
    # skewed routing so that popular experts overflow their capacity
    g = torch.Generator().manual_seed(T + k)
    p = torch.arange(1, E + 1, dtype=torch.float64).pow(-1.2)
    idx = torch.stack([torch.multinomial(p, k, replacement=False, generator=g)
                       for _ in range(T)]).int()
    gate = torch.softmax(torch.randn((T, k), generator=g), 1)
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    ws = moe.workspace(shape)
    keep, kept, cap = moe.capacity_keep(shape, idx.cuda(), gate.cuda(), cf, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    assert cap == oracle.expert_capacity(T, k, E, cf)
    ref = oracle.capacity_keep(idx.numpy(), E, cf)
    np.testing.assert_array_equal(keep.cpu().numpy().astype(bool), ref)
    assert (~ref).any(), "the case drops nothing"
    assert torch.equal(kept.cpu(), torch.where(torch.from_numpy(ref), gate, torch.zeros(())))
    # NULL gates: unit gates where kept
    _, kept1, _ = moe.capacity_keep(shape, idx.cuda(), None, cf, ws)
    assert torch.equal(kept1.cpu(), torch.from_numpy(ref).float())


def test_layout_after_capacity_on_the_same_workspace():
    """moe_capacity_keep borrows the layout's lookback words for its
    per-chunk counts and zeroes them again: a dispatch layout on the same
    workspace afterwards equals one on a fresh workspace."""
    T, E, k = 9000, 64, 4
    g = torch.Generator().manual_seed(7)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).int().cuda()
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64, ep=8)
    ws = moe.workspace(shape)
    moe.capacity_keep(shape, idx, None, 1.0, ws)
    lay = moe.dispatch_layout(shape, idx, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    ref = moe.dispatch_layout(shape, idx, moe.workspace(shape))
    for name in ("expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
                 "rank_offsets", "send_token", "slot_send_row"):
        assert torch.equal(lay[name], ref[name]), name


def test_capacity_forward_matches_oracle():
    """The layer with limited expert capacity: the routed forward on the
    kept gates equals the oracle's per-token sum over the kept assignments."""
    c = Case(3, T=1200, near_ties=False)
    w = c.w
    ws = moe.workspace(c.shape, forward=True)
    _, idx, gate = moe.route(c.shape, c.dx, c.packed, None, ws)
    keep, kept, cap = moe.capacity_keep(c.shape, idx, gate, 1.0, ws)
    y = moe.forward_routed(c.shape, c.dx, c.packed, idx, kept, ws)
    moe.check_device_status(ws)
    ref_keep = oracle.capacity_keep(idx.cpu().numpy(), w.E, 1.0)
    np.testing.assert_array_equal(keep.cpu().numpy().astype(bool), ref_keep)
    assert (~ref_keep).any()
    g = gate.cpu().double().numpy() * ref_keep
    ref = oracle.moe_output(c.x, idx.cpu().numpy(), g, c.wg, c.wu, c.wd)
    check_output(y, ref, w.dtype)


def test_capacity_bad_index_is_reported():
    T, E, k = 500, 16, 2
    idx = W.uniform_routing(T, E, k, seed=1)
    idx[7, 1] = E
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    ws = moe.workspace(shape)
    keep, _, _ = moe.capacity_keep(shape, idx.cuda(), None, 1.0, ws)
    assert moe.get_device_status(ws) == moe.MOE_ERR_DEVICE_INDEX
    assert int(keep[7, 1]) == 0
    assert moe.get_device_status(ws) == moe.MOE_OK


def test_top16_of_64_fine_grained_forward():
    """Top-16 routing over 64 fine-grained experts: routing against the
    oracle (near-ties excepted), whole layout bit-exact, output within the
    bf16 tolerance."""
    w = dataclasses.replace(W.WORKLOADS[2], k=16)
    T = 1111
    x = W.make_x(w, 0, T)
    wr = W.make_router(w)
    wg, wu, wd = W.make_experts(w)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=16, f=w.f, ep=8)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y = moe.forward(shape, x.cuda(), packed, None, ws, buffers=buf)
    moe.check_device_status(ws)
    ref = oracle.forward(x, wr, None, wg, wu, wd, 16)
    gi = buf.topk_idx.cpu().numpy()
    bad = routing_mismatches(gi, ref["idx"])
    m = oracle.margin(ref["logits"], 16)
    assert (m[bad] < NEAR_TIE).all()
    ok = np.setdiff1d(np.arange(T), bad)
    check_output(y, ref["y"], "bf16", rows=ok)
    lay = oracle.dispatch_layout(gi, w.E, 8)
    for key in ("expert_offsets", "row_token", "slot_row", "rank_counts", "slot_send_row"):
        np.testing.assert_array_equal(buf.layout[key].cpu().numpy(), lay[key], err_msg=key)
