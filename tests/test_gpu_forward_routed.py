"""GPU parity of moe_forward_routed, the layer below the router on a routing
the caller supplies (a recorded routing table replayed).

Replaying moe_forward's own routing gives its output bit for bit: the
standalone dispatch layout equals the forward's, and the same expert and
combine kernels follow.  On a routing drawn independently of the router
(uniform experts, random softmax gates) the output matches the oracle's
experts and combine within the dtype's tolerance, and NULL gates are unit
gates."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import TOL, Case

LAYOUT_KEYS = ("expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
               "rank_offsets", "slot_send_row")

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,T,ep", [
    (1, 700, 1),     # fp32: CUDA-core experts
    (2, 2311, 8),    # bf16, fused expert FFN with the row gather
    (3, 513, 8),     # bf16, separate grouped GEMMs
])
def test_replaying_the_forward_routing_is_bit_exact(cfg, T, ep):
    c = Case(cfg, T=T, near_ties=False)
    shape = c.shape_ep(ep)
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y0 = moe.forward(shape, c.dx, c.packed, c.dbias, ws, buffers=buf)
    idx, gate = buf.topk_idx.clone(), buf.topk_gate.clone()
    buf2 = moe.ForwardBuffers(shape)
    y1 = moe.forward_routed(shape, c.dx, c.packed, idx, gate, ws, buffers=buf2)
    moe.check_device_status(ws)
    assert torch.equal(y0, y1)
    for name in ("expert_offsets", "row_token", "slot_row"):
        assert torch.equal(buf.layout[name], buf2.layout[name]), name


@pytest.mark.parametrize("cfg,T", [(1, 300), (2, 1500), (3, 257)])
def test_given_routing_matches_oracle(cfg, T):
    c = Case(cfg, T=T, near_ties=False)
    w = c.w
    idx = W.uniform_routing(T, w.E, w.k, seed=T + 7)
    g = torch.Generator().manual_seed(T)
    gate = torch.softmax(torch.randn((T, w.k), generator=g), 1)
    ws = moe.workspace(c.shape, forward=True)
    y = moe.forward_routed(c.shape, c.dx, c.packed, idx.cuda(), gate.cuda(), ws)
    moe.check_device_status(ws)
    toks = np.arange(T)
    ref = oracle.moe_output(c.x, idx.numpy(), gate.double().numpy(), c.wg, c.wu, c.wd,
                            tokens=toks)
    err = np.abs(y.cpu().double().numpy() - ref).max()
    assert err <= TOL[w.dtype] * np.abs(ref).max()


def test_null_gates_are_unit_gates():
    c = Case(2, T=1000, near_ties=False)
    w = c.w
    idx = W.uniform_routing(c.T, w.E, w.k, seed=3).cuda()
    ws = moe.workspace(c.shape, forward=True)
    y0 = moe.forward_routed(c.shape, c.dx, c.packed, idx, None, ws)
    ones = torch.ones((c.T, w.k), dtype=torch.float32, device="cuda")
    y1 = moe.forward_routed(c.shape, c.dx, c.packed, idx, ones, ws)
    moe.check_device_status(ws)
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("cfg,T,ep", [(1, 300, 1), (2, 1500, 8), (3, 257, 16)])
def test_repeated_expert_within_a_token(cfg, T, ep):
    """A recorded routing may name one expert twice for a token (top-k never
    does).  Each assignment is its own expert-grouped row, the token still
    goes to that expert's rank once, and the output sums both gated copies:
    layout bit-exact against the oracle's, output within the tolerance of
    the oracle's per-token definition."""
    c = Case(cfg, T=T, near_ties=False)
    w = c.w
    idx = W.uniform_routing(T, w.E, w.k, seed=T + 11)
    g = torch.Generator().manual_seed(T + 1)
    rep = torch.randperm(T, generator=g)[: T // 3]
    idx[rep, 1] = idx[rep, 0]                  # slot 1 repeats slot 0
    if w.k > 2:
        idx[rep[: len(rep) // 2], w.k - 1] = idx[rep[: len(rep) // 2], 0]  # three copies
    gate = torch.softmax(torch.randn((T, w.k), generator=g), 1)
    shape = c.shape_ep(ep)
    rmap = W.permutation_placement(w.E, ep, 5)
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y = moe.forward_routed(shape, c.dx, c.packed, idx.cuda(), gate.cuda(), ws,
                           expert_rank=rmap, buffers=buf)
    moe.check_device_status(ws)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, ep, rmap)
    for key in LAYOUT_KEYS:
        if ep == 1 and (key.startswith("rank") or key == "slot_send_row"):
            continue
        np.testing.assert_array_equal(buf.layout[key].cpu().numpy(), lay[key], err_msg=key)
    if ep > 1:
        n = lay["stats"]["rows_sent"]
        np.testing.assert_array_equal(buf.layout["send_token"][:n].cpu().numpy(), lay["send_token"])
    assert moe.stats_dict(buf.layout["stats"]) == lay["stats"]
    ref = oracle.moe_output(c.x, idx.numpy(), gate.double().numpy(), c.wg, c.wu, c.wd,
                            tokens=np.arange(T))
    err = np.abs(y.cpu().double().numpy() - ref).max()
    assert err <= TOL[w.dtype] * np.abs(ref).max()
