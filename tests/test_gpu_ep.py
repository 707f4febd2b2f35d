"""The expert-parallel layer with its deduplicated dispatch ("Expert
Coupling in MoE Pretraining", Abstract; Fig. 7 B vs D vs D+P), P ranks
emulated on one GPU in one process (their kernels run one after another,
none waits on another): the library's send plan, pack, receiving-rank
experts and home combine, with the rows moved by block copies between the
ranks' buffers.

Checked against the oracle: every rank's send plan (rank_counts, send
rows) bit-exact, the count matrix's rows equal to the deduplicated rows of
Table I, and the output of every token within the bf16 tolerance of the
oracle's layer (and of the single-GPU forward) -- the partial sums per rank
are rounded once to bf16 before the home rank adds them."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import ep as EP
from routing_dispatch_experts_b200 import workloads as W

from util import TOL, check_output, routing_mismatches

pytestmark = pytest.mark.gpu


def _setup(cfg, T, P, placement, seed=0):
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, seed, T)
    wr = W.make_router(w, seed)
    bias = W.make_bias(w, seed)
    wg, wu, wd = W.make_experts(w, seed)
    rmap = (W.contiguous_placement(w.E, P) if placement == "contiguous"
            else W.permutation_placement(w.E, P, seed=P))
    Tr = T // P
    shape = moe.Shape(T=Tr, d=w.d, E=w.E, k=w.k, f=w.f, ep=P, dtype=w.torch_dtype)
    router = moe.pack_weights(shape, wr.cuda(), None, None, None)
    dbias = None if bias is None else bias.cuda()
    ranks = []
    for r in range(P):
        mine = EP.local_experts(rmap, r)
        ls = moe.Shape(T=Tr, d=w.d, E=len(mine), k=min(w.k, len(mine)), f=w.f, dtype=w.torch_dtype)
        local = moe.pack_weights(ls, None, wg[mine].cuda(), wu[mine].cuda(), wd[mine].cuda())
        ranks.append(EP.EPRank(shape, r, rmap, router, local, bias=dbias))
    xs = [x[r * Tr:(r + 1) * Tr].cuda() for r in range(P)]
    return w, x, wr, bias, (wg, wu, wd), rmap, ranks, xs, shape


@pytest.mark.parametrize("cfg,T,P,placement", [
    (3, 4096, 8, "contiguous"), (3, 4096, 16, "permutation"),  # top-2 (Table I rows)
    (2, 4096, 8, "contiguous"),                                # fine-grained: fused expert FFN
    (1, 1024, 4, "contiguous"),                                # fp32
    (4, 2048, 32, "permutation"),                              # top-6 over 32 ranks: 2 experts each
    (5, 1024, 16, "contiguous"),                               # large: top-8 of 128, Zipf bias
])
def test_ep_forward_matches_oracle(cfg, T, P, placement):
    w, x, wr, bias, (wg, wu, wd), rmap, ranks, xs, shape = _setup(cfg, T, P, placement)
    ys, counts = EP.forward_emulated(ranks, xs)
    torch.cuda.synchronize()
    for r in ranks:
        moe.check_device_status(r.ws)
    y = torch.cat(ys)
    # the routing each rank chose, and the oracle's send plan for it
    idx = torch.cat([r.plan(xx).idx for r, xx in zip(ranks, xs)]).cpu().numpy()
    sent = 0
    for r in range(P):
        lay = oracle.dispatch_layout(idx[r * shape.T:(r + 1) * shape.T], w.E, P, rmap)
        assert counts[r] == lay["rank_counts"].tolist()
        sent += lay["stats"]["rows_sent"]
    C = np.array(counts)
    assert C.sum() == sent  # deduplicated rows: one per (token, destination rank)
    # every token against the oracle (routing from the oracle's double
    # logits; tokens at near-ties compared on the GPU's own routing)
    ref = oracle.forward(x, wr, bias, wg, wu, wd, w.k)
    bad = routing_mismatches(idx, ref["idx"])
    m = oracle.margin(ref["logits"], w.k)
    assert (m[bad] < 1e-5).all()
    ok = np.setdiff1d(np.arange(T), bad)
    check_output(y, ref["y"], w.dtype, rows=ok)
    # and against the single-GPU forward of the same tokens
    full = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, ep=P, dtype=w.torch_dtype)
    packed = moe.pack_weights(full, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(full, forward=True)
    y1 = moe.forward(full, x.cuda(), packed, None if bias is None else bias.cuda(), ws,
                     expert_rank=rmap)
    moe.check_device_status(ws)
    scale = float(y1.float().abs().max())
    assert float((y.float() - y1.float()).abs().max()) <= TOL[w.dtype] * scale


def test_ep_dedup_and_correlated_placement_cut_rows():
    """Rows on the wire for the top-2 workload at EP 8: per-expert dispatch
    (B) sends every assignment whose expert is on another rank; the
    deduplicated dispatch (D) one row per (token, rank); a correlated
    placement fit on a calibration batch (D+P) fewer still ('Expert
    Coupling', Fig. 7)."""
    cfg, T, P = 3, 4096, 8
    w, x, wr, bias, _, rmap, ranks, xs, shape = _setup(cfg, T, P, "contiguous")
    _, counts = EP.forward_emulated(ranks, xs)
    idx = torch.cat([r.plan(xx).idx for r, xx in zip(ranks, xs)]).cpu().numpy()
    home = np.repeat(np.arange(P), T // P)
    owner = np.array(rmap)[idx]
    b_rows = int((owner != home[:, None]).sum())
    d_rows = int(sum(counts[r][s] for r in range(P) for s in range(P) if s != r))
    assert d_rows < b_rows
    cal = W.make_x(w, 0, 4096, stream="calib").cuda()
    full = moe.Shape(T=4096, d=w.d, E=w.E, k=w.k, f=w.f, ep=P, dtype=w.torch_dtype)
    ws = moe.workspace(full)
    _, cidx, _ = moe.route(full, cal, ranks[0].packed_router, None, ws)
    fit = moe.fit_placement(w.E, P, moe.coselection_counts(full, cidx, ws))
    own = np.array(fit)[idx]
    dp_rows = sum(len(set(own[t]) - {home[t]}) for t in range(T))
    assert dp_rows < d_rows


@pytest.mark.parametrize("cfg,T,P,placement", [
    (3, 4096, 8, "contiguous"), (2, 4096, 8, "permutation"), (1, 1024, 4, "contiguous"),
    (5, 1024, 16, "contiguous"),
])
def test_peer_exchange_equals_the_collective_exchange(cfg, T, P, placement):
    """moe_ep_dispatch_peer + moe_ep_expert_forward_peer store the same rows
    at the same positions as pack + all-to-all and experts + reverse
    all-to-all: every rank's output bit-identical."""
    *_, ranks, xs, shape = _setup(cfg, T, P, placement)
    ys, counts = EP.forward_emulated(ranks, xs)
    yp, counts_p = EP.forward_peer_emulated(ranks, xs)
    torch.cuda.synchronize()
    assert counts_p == counts
    for r in range(P):
        assert torch.equal(yp[r], ys[r]), r


def test_peer_dispatch_stores_no_row_past_its_block():
    """A destination block smaller than the rows the plan sends there: the
    rows past it are not stored (the rows around the block keep their
    sentinel), the rows inside it equal the pack's."""
    cfg, T, P = 3, 2048, 4
    *_, ranks, xs, shape = _setup(cfg, T, P, "contiguous")
    rk, x = ranks[1], xs[1]
    plan = rk.plan(x)
    n = [int(v) for v in plan.layout["rank_counts"].tolist()]
    send_x, send_idx, send_gate = moe.ep_pack(shape, x, plan.idx, plan.gate, plan.layout, sum(n),
                                              expert_rank=rk.expert_rank)
    off = np.concatenate([[0], np.cumsum(n)])
    pad = 7
    bufs = []
    dests = []
    for r in range(P):
        rows = max(n[r] - 5, 0) if r == 2 else n[r]
        bx = torch.full((pad + n[r] + pad, shape.d), 3.0, dtype=shape.dtype, device="cuda")
        bi = torch.full((pad + n[r] + pad, shape.k), -9, dtype=torch.int32, device="cuda")
        bg = torch.full((pad + n[r] + pad, shape.k), -2.0, dtype=torch.float32, device="cuda")
        bufs.append((bx, bi, bg, rows))
        dests.append((bx, bi, bg, pad, rows))
    moe.ep_dispatch_peer(shape, x, plan.idx, plan.gate, plan.layout, dests,
                         expert_rank=rk.expert_rank)
    torch.cuda.synchronize()
    for r, (bx, bi, bg, rows) in enumerate(bufs):
        lo, hi = int(off[r]), int(off[r]) + rows
        assert torch.equal(bx[pad:pad + rows], send_x[lo:hi])
        assert torch.equal(bi[pad:pad + rows], send_idx[lo:hi])
        assert torch.equal(bg[pad:pad + rows], send_gate[lo:hi])
        assert (bx[:pad] == 3.0).all() and (bx[pad + rows:] == 3.0).all()
        assert (bi[:pad] == -9).all() and (bi[pad + rows:] == -9).all()
        assert (bg[:pad] == -2.0).all() and (bg[pad + rows:] == -2.0).all()


def test_signal_wait_passes_when_every_slot_is_set():
    """One kernel: rank 0 of 3 stores its epoch into slot 0 of each array
    and finds slots 1 and 2 of its own array already at the epoch (set
    beforehand, as ranks 1 and 2 would)."""
    P = 3
    flags = [torch.zeros(P, dtype=torch.int64, device="cuda") for _ in range(P)]
    ws = moe.workspace(moe.Shape(T=1, d=64, E=4, k=1, f=64))
    flags[0][1:] = 5
    moe.ep_signal_wait(flags, 0, 5, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    assert [int(f[0]) for f in flags] == [5, 5, 5]
    # a single rank meets only itself
    one = [torch.zeros(1, dtype=torch.int64, device="cuda")]
    moe.ep_signal_wait(one, 0, 1, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK and int(one[0][0]) == 1


def test_signal_wait_gives_up_on_a_flag_nothing_sets():
    """Rank 0 of 2 with rank 1's slot never set: the bounded wait ends after
    its limit with MOE_ERR_DEVICE_TIMEOUT (detail: rank 1), and the context
    stays usable (a following rendezvous that finds its slots passes)."""
    P = 2
    flags = [torch.zeros(P, dtype=torch.int64, device="cuda") for _ in range(P)]
    ws = moe.workspace(moe.Shape(T=1, d=64, E=4, k=1, f=64))
    moe.ep_signal_wait(flags, 0, 1, ws, wait_limit_ns=2_000_000)
    assert moe.get_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    flags[0][1] = 2
    moe.ep_signal_wait(flags, 0, 2, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK


@pytest.mark.parametrize("cfg,T,P,placement", [(3, 4096, 8, "contiguous"), (1, 1024, 4, "contiguous"),
                                               (2, 2048, 8, "permutation")])
def test_peer_rank_phases_equal_the_collective_exchange(cfg, T, P, placement):
    """PeerEPRank's own buffer layout and phases (dispatch, experts, finish)
    for P ranks on one GPU with caller buffers, driven in phase order (no
    rendezvous: nothing waits on another kernel): every rank's output
    bit-identical to the collective path; the buffers sized for more tokens
    than the ranks hold, and reused for a second forward."""
    *_, ranks, xs, shape = _setup(cfg, T, P, placement)
    ys, counts = EP.forward_emulated(ranks, xs)
    n = EP.peer_buffer_bytes(shape, shape.T + 3)
    bufs = [torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda") for _ in range(P)]
    peers = [EP.PeerEPRank(shape, r, rk.expert_rank, rk.packed_router, rk.packed_local,
                           max_tokens=shape.T + 3, bias=rk.bias, buffers=bufs)
             for r, rk in enumerate(ranks)]
    for _ in range(2):
        yp, counts_p = EP.forward_peer_ranks_emulated(peers, xs)
        torch.cuda.synchronize()
        assert counts_p == counts
        for r in range(P):
            assert torch.equal(yp[r], ys[r]), r
    with pytest.raises(RuntimeError):
        peers[0].forward(xs[0])
