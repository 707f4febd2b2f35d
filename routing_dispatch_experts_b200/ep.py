"""Expert-parallel MoE layer: one rank's forward over P ranks, around an
exchange of rows between the ranks.

The deduplicated dispatch of "Expert Coupling in MoE Pretraining"
(Abstract: each token is sent to each GPU that holds one of its experts
once; Fig. 7: baseline dispatch B vs deduplicated D, with or without
correlated placement P): tokens are split over the ranks, experts are
placed by an expert -> rank map, and every rank

  1. routes its tokens and builds the send plan (moe_route,
     moe_dispatch_layout with ep = P),
  2. learns how many rows every rank sends every rank (exchange of the
     rank_counts),
  3. packs and sends its rows (moe_ep_pack, all-to-all),
  4. runs its experts over the rows it received (moe_ep_expert_forward),
  5. returns one row per received row (reverse all-to-all),
  6. sums each token's returned rows (moe_ep_home_combine).

Steps 1, 3, 4 and 6 are the library's CUDA kernels; this module only
sequences them and moves rows through an Exchange:

  TorchExchange  torch.distributed collectives (NCCL between GPUs, gloo on
                 CPU tensors), one process per rank;
  LocalExchange  P ranks emulated in one process (their buffers on one
                 device), for single-GPU tests of the whole path.

or, with peer memory, without a separate exchange: moe_ep_dispatch_peer
stores each send row straight into its destination's receive buffer and
moe_ep_expert_forward_peer each return row straight into its source's
buffer (peer_blocks gives where; PeerEPRank runs it over a symmetric-memory
allocation with moe_ep_signal_wait between the phases; forward_peer_emulated
runs the same kernels with the ranks' buffers on one device).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

from . import Shape, check_device_status, dispatch_layout, ep_dispatch_peer, ep_expert_forward, \
    ep_expert_forward_peer, ep_expert_workspace, ep_home_combine, ep_pack, ep_signal_wait, route, \
    workspace

# ------------------------------------------------------------------ exchange


def splits(counts: Sequence[Sequence[int]], rank: int):
    """(send splits, receive splits) of `rank` from the count matrix
    counts[src][dst] = rows src sends dst: it sends row block dst of its
    send rows to dst, and receives from every src in rank order."""
    P = len(counts)
    return [int(counts[rank][d]) for d in range(P)], [int(counts[s][rank]) for s in range(P)]


def peer_blocks(counts: Sequence[Sequence[int]], rank: int):
    """Where `rank`'s rows go in a peer-memory exchange, from the count
    matrix counts[src][dst]:
      dests[r] = (row0, rows) of its block in rank r's receive rows: after
                 the blocks of the ranks below it (row0 = sum_{s < rank}
                 counts[s][r]), rows = counts[rank][r];
      rets[s]  = (row0, rows) of the block it received from rank s, in s's
                 send-row order (row0 = sum_{r < rank} counts[s][r], s's
                 rank_offsets[rank]), rows = counts[s][rank].
    The same positions as the all-to-all of TorchExchange.rows."""
    P = len(counts)
    dests = [(sum(int(counts[q][r]) for q in range(rank)), int(counts[rank][r])) for r in range(P)]
    rets = [(sum(int(counts[q][r]) for r in range(rank)), int(counts[q][rank])) for q in range(P)]
    return dests, rets


class TorchExchange:
    """Rows between ranks with torch.distributed (one process per rank)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def counts(self, rank_counts: torch.Tensor) -> List[List[int]]:
        """Every rank's rank_counts, as the host matrix counts[src][dst]."""
        mine = rank_counts.to(torch.int64).reshape(-1)
        allc = torch.empty(self.world * self.world, dtype=torch.int64, device=mine.device)
        self.dist.all_gather_into_tensor(allc, mine, group=self.group)
        return allc.reshape(self.world, self.world).tolist()

    def rows(self, send: torch.Tensor, send_splits: List[int], recv_splits: List[int]) -> torch.Tensor:
        """all-to-all-v of the rows of `send` (blocks of send_splits rows to
        ranks 0..P-1), received in source-rank order."""
        out = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                          device=send.device)
        self.dist.all_to_all_single(out, send.contiguous(), output_split_sizes=recv_splits,
                                    input_split_sizes=send_splits, group=self.group)
        return out


class LocalExchange:
    """P ranks in one process: each collective takes every rank's input at
    once and returns every rank's output (plain block copies)."""

    def __init__(self, world: int):
        self.world = world

    def counts(self, rank_counts: Sequence[torch.Tensor]) -> List[List[int]]:
        return [[int(v) for v in rc.tolist()] for rc in rank_counts]

    def rows(self, sends: Sequence[torch.Tensor], counts: List[List[int]]) -> List[torch.Tensor]:
        P = self.world
        blocks = [torch.split(sends[s], counts[s]) for s in range(P)]
        return [torch.cat([blocks[s][r] for s in range(P)]) for r in range(P)]

    def rows_back(self, rets: Sequence[torch.Tensor], counts: List[List[int]]) -> List[torch.Tensor]:
        P = self.world
        blocks = [torch.split(rets[r], [counts[s][r] for s in range(P)]) for r in range(P)]
        return [torch.cat([blocks[r][s] for r in range(P)]) for s in range(P)]


# ----------------------------------------------------------------- one rank


@dataclasses.dataclass
class Plan:
    """What a rank keeps between the phases of its forward."""
    idx: torch.Tensor
    gate: torch.Tensor
    layout: dict
    counts: Optional[List[List[int]]] = None


class EPRank:
    """One rank of the expert-parallel layer.

    shape          T = this rank's tokens, E = all experts, ep = P ranks
    rank           this rank's index in [0, P)
    expert_rank    expert -> rank map (a partition with E/P experts per
                   rank), or None for contiguous placement
    packed_router  moe_pack_weights output holding the router (all ranks
                   route with the same router)
    packed_local   moe_pack_weights output for this rank's E/P experts, in
                   ascending expert order
    """

    def __init__(self, shape: Shape, rank: int, expert_rank, packed_router, packed_local,
                 bias=None):
        if shape.ep < 2:
            raise ValueError("expert parallelism needs ep >= 2 ranks")
        self.shape = shape
        self.rank = rank
        self.expert_rank = None if expert_rank is None else list(expert_rank)
        self.packed_router = packed_router
        self.packed_local = packed_local
        self.bias = bias
        self.ws = workspace(shape, device=packed_router.device)

    # phase 1: routing and the send plan
    def plan(self, x) -> Plan:
        _, idx, gate = route(self.shape, x, self.packed_router, self.bias, self.ws)
        lay = dispatch_layout(self.shape, idx, self.ws, expert_rank=self.expert_rank)
        return Plan(idx=idx, gate=gate, layout=lay)

    # phase 2: the send rows (after the count exchange)
    def send(self, x, plan: Plan, counts: List[List[int]]):
        plan.counts = counts
        n = sum(counts[self.rank])
        return ep_pack(self.shape, x, plan.idx, plan.gate, plan.layout, n,
                       expert_rank=self.expert_rank)

    # phase 3: this rank's experts over the rows it received
    def experts(self, recv_x, recv_idx, recv_gate, ws=None):
        rs = dataclasses.replace(self.shape, T=int(recv_x.shape[0]))
        if ws is None:
            ws = ep_expert_workspace(rs, device=recv_x.device)
        return ep_expert_forward(rs, recv_x, recv_idx, recv_gate, self.packed_local, ws)

    # phase 4: this rank's outputs from the returned rows
    def finish(self, plan: Plan, y_back):
        return ep_home_combine(self.shape, y_back, plan.layout["slot_send_row"])

    def forward(self, x, ex: TorchExchange):
        """The whole forward of this rank, exchanging through `ex` (every
        rank calls it with its own tokens)."""
        plan = self.plan(x)
        counts = ex.counts(plan.layout["rank_counts"])
        send_x, send_idx, send_gate = self.send(x, plan, counts)
        s_sp, r_sp = splits(counts, self.rank)
        recv_x = ex.rows(send_x, s_sp, r_sp)
        recv_idx = ex.rows(send_idx, s_sp, r_sp)
        recv_gate = ex.rows(send_gate, s_sp, r_sp)
        y_ret = self.experts(recv_x, recv_idx, recv_gate)
        y_back = ex.rows(y_ret, r_sp, s_sp)
        return self.finish(plan, y_back), counts


def forward_emulated(ranks: Sequence[EPRank], xs: Sequence[torch.Tensor]):
    """Every rank's forward with the ranks emulated in one process (one
    device): the same phases as EPRank.forward, the exchanges done by
    LocalExchange.  Returns (per-rank outputs, count matrix)."""
    P = len(ranks)
    ex = LocalExchange(P)
    plans = [r.plan(x) for r, x in zip(ranks, xs)]
    counts = ex.counts([p.layout["rank_counts"] for p in plans])
    sends = [r.send(x, p, counts) for r, x, p in zip(ranks, xs, plans)]
    recv_x = ex.rows([s[0] for s in sends], counts)
    recv_idx = ex.rows([s[1] for s in sends], counts)
    recv_gate = ex.rows([s[2] for s in sends], counts)
    rets = [r.experts(recv_x[i], recv_idx[i], recv_gate[i]) for i, r in enumerate(ranks)]
    backs = ex.rows_back(rets, counts)
    return [r.finish(p, b) for r, p, b in zip(ranks, plans, backs)], counts


def forward_peer_emulated(ranks: Sequence[EPRank], xs: Sequence[torch.Tensor]):
    """forward_emulated through the peer-memory kernels: every rank's send
    rows stored straight into the receiving ranks' buffers, every return row
    straight into its source's buffer (the ranks' buffers on one device, the
    phases in order on one stream, so no rendezvous is needed).  Returns
    (per-rank outputs, count matrix)."""
    P = len(ranks)
    sh = ranks[0].shape
    dev = xs[0].device
    plans = [r.plan(x) for r, x in zip(ranks, xs)]
    counts = LocalExchange(P).counts([p.layout["rank_counts"] for p in plans])
    n_recv = [sum(counts[q][r] for q in range(P)) for r in range(P)]
    n_send = [sum(counts[q]) for q in range(P)]
    recv = [(torch.empty((n, sh.d), dtype=sh.dtype, device=dev),
             torch.empty((n, sh.k), dtype=torch.int32, device=dev),
             torch.empty((n, sh.k), dtype=torch.float32, device=dev)) for n in n_recv]
    backs = [torch.empty((n, sh.d), dtype=sh.dtype, device=dev) for n in n_send]
    for q, (rk, x, p) in enumerate(zip(ranks, xs, plans)):
        p.counts = counts
        dests, _ = peer_blocks(counts, q)
        ep_dispatch_peer(rk.shape, x, p.idx, p.gate, p.layout,
                         [recv[r] + dests[r] for r in range(P)], expert_rank=rk.expert_rank)
    for r, rk in enumerate(ranks):
        _, rets = peer_blocks(counts, r)
        rs = dataclasses.replace(rk.shape, T=n_recv[r])
        ws = ep_expert_workspace(rs, device=dev)
        ep_expert_forward_peer(rs, *recv[r], rk.packed_local,
                               [(backs[q],) + rets[q] for q in range(P)], ws)
    return [rk.finish(p, b) for rk, p, b in zip(ranks, plans, backs)], counts


class PeerEPRank(EPRank):
    """One rank of the expert-parallel layer over peer memory (one process
    per GPU, the ranks' GPUs peer-connected): the receive rows, the return
    rows and the rendezvous flags of every rank live in one buffer per rank,
    by default a symmetric-memory allocation (torch.distributed.
    _symmetric_memory) sized for at most `max_tokens` tokens per rank;
    every forward takes two rendezvous epochs (after the dispatch stores,
    after the return stores), which also keep the next forward's stores out
    of buffers still being read.

    `buffers` (a list of every rank's byte buffer, as peer_buffer_bytes
    sizes them, all addressable from this process) replaces the
    symmetric-memory allocation: the phases (plan, dispatch, experts,
    finish) can then be driven for P ranks in one process on one device,
    in phase order with no rendezvous."""

    def __init__(self, shape: Shape, rank: int, expert_rank, packed_router, packed_local,
                 group=None, max_tokens=None, bias=None, buffers=None):
        super().__init__(shape, rank, expert_rank, packed_router, packed_local, bias)
        P = shape.ep
        self.max_tokens = shape.T if max_tokens is None else int(max_tokens)
        self.off, n = _peer_layout(shape, self.max_tokens)
        self.cap_recv = P * self.max_tokens      # rows from every source, one per token at most
        self.cap_send = self.max_tokens * min(shape.k, P)  # send rows of this rank's tokens
        if buffers is None:
            import torch.distributed as dist
            import torch.distributed._symmetric_memory as symm
            self.ex = TorchExchange(group)
            self.buf = symm.empty(n, dtype=torch.uint8, device=packed_router.device)
            self.buf.zero_()
            self.hdl = symm.rendezvous(self.buf, group if group is not None else dist.group.WORLD)
            bufs = [self.hdl.get_buffer(q, (n,), torch.uint8) for q in range(P)]
        else:
            if len(buffers) != P or any(b.numel() < n for b in buffers):
                raise ValueError(f"buffers: expected {P} byte buffers of >= {n} bytes")
            self.ex = None
            bufs = list(buffers)
        self.views = [self._views(b) for b in bufs]
        self.epoch = 0

    def _views(self, b):
        sh, o = self.shape, self.off
        cr, cs = self.cap_recv, self.cap_send

        def at(name, dt, shape):
            nb = torch.tensor([], dtype=dt).element_size()
            for s_ in shape:
                nb *= s_
            return b[o[name]:o[name] + nb].view(dt).view(shape)
        return {"flags": at("flags", torch.int64, (sh.ep,)),
                "recv_x": at("recv_x", sh.dtype, (cr, sh.d)),
                "recv_idx": at("recv_idx", torch.int32, (cr, sh.k)),
                "recv_gate": at("recv_gate", torch.float32, (cr, sh.k)),
                "y_back": at("y_back", sh.dtype, (cs, sh.d))}

    def _rendezvous(self):
        self.epoch += 1
        ep_signal_wait([v["flags"] for v in self.views], self.rank, self.epoch, self.ws)

    # phase 2 (after plan and the count exchange): this rank's send rows
    # stored straight into every rank's receive rows
    def dispatch(self, x, plan: Plan, counts: List[List[int]]):
        plan.counts = counts
        dests, _ = peer_blocks(counts, self.rank)
        V = self.views
        ep_dispatch_peer(self.shape, x, plan.idx, plan.gate, plan.layout,
                         [(V[r]["recv_x"], V[r]["recv_idx"], V[r]["recv_gate"]) + dests[r]
                          for r in range(self.shape.ep)], expert_rank=self.expert_rank)

    # phase 3: this rank's experts over its receive rows, the return rows
    # stored straight into their sources' return rows
    def experts_peer(self, plan: Plan):
        _, rets = peer_blocks(plan.counts, self.rank)
        n_recv = sum(rows for _, rows in rets)
        me, V = self.views[self.rank], self.views
        rs = dataclasses.replace(self.shape, T=n_recv)
        ws = ep_expert_workspace(rs, device=me["recv_x"].device)
        ep_expert_forward_peer(rs, me["recv_x"][:n_recv], me["recv_idx"][:n_recv],
                               me["recv_gate"][:n_recv], self.packed_local,
                               [(V[q]["y_back"],) + rets[q] for q in range(self.shape.ep)], ws)

    # phase 4: this rank's outputs from its return rows
    def finish_peer(self, plan: Plan):
        n_send = sum(plan.counts[self.rank])
        return self.finish(plan, self.views[self.rank]["y_back"][:n_send])

    def forward(self, x, ex=None):
        """The whole forward of this rank (every rank calls it with its own
        tokens, one process per GPU); raises if a rendezvous timed out."""
        if self.ex is None:
            raise RuntimeError("forward needs the symmetric-memory buffers of a process group; "
                               "with caller buffers drive the phases in order")
        plan = self.plan(x)
        counts = self.ex.counts(plan.layout["rank_counts"])
        self.dispatch(x, plan, counts)
        self._rendezvous()
        self.experts_peer(plan)
        self._rendezvous()
        check_device_status(self.ws)
        return self.finish_peer(plan), counts


def _peer_layout(shape: Shape, max_tokens: int):
    """Byte offsets of the parts of one rank's peer buffer, and its size."""
    P, d, k = shape.ep, shape.d, shape.k
    cap_recv, cap_send = P * max_tokens, max_tokens * min(k, P)
    es = torch.tensor([], dtype=shape.dtype).element_size()
    parts = [("flags", 8 * P), ("recv_x", es * d * cap_recv), ("recv_idx", 4 * k * cap_recv),
             ("recv_gate", 4 * k * cap_recv), ("y_back", es * d * cap_send)]
    off, n = {}, 0
    for name, b in parts:
        off[name] = n
        n += (b + 255) // 256 * 256
    return off, n


def peer_buffer_bytes(shape: Shape, max_tokens: int) -> int:
    """Bytes of one rank's peer buffer (receive rows, return rows, flags)."""
    return _peer_layout(shape, max_tokens)[1]


def forward_peer_ranks_emulated(ranks: Sequence[PeerEPRank], xs: Sequence[torch.Tensor]):
    """PeerEPRank's phases for P ranks in one process (caller buffers on one
    device), in phase order: plans, count matrix, every rank's dispatch,
    every rank's experts, every rank's finish.  Returns (per-rank outputs,
    count matrix)."""
    P = len(ranks)
    plans = [r.plan(x) for r, x in zip(ranks, xs)]
    counts = LocalExchange(P).counts([p.layout["rank_counts"] for p in plans])
    for r, x, p in zip(ranks, xs, plans):
        r.dispatch(x, p, counts)
    for r, p in zip(ranks, plans):
        r.experts_peer(p)
    return [r.finish_peer(p) for r, p in zip(ranks, plans)], counts


def local_experts(expert_rank: Sequence[int], rank: int) -> List[int]:
    """The experts a rank holds, ascending (the order of their local ids)."""
    return [e for e, r in enumerate(expert_rank) if r == rank]
