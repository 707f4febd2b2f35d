"""The multi-GPU path of bench.py on CPU: world_size-2 gloo ranks.

The layer shards by tokens with no exchange in the forward (replicas), so
the N > 1 path is the plumbing around it: every rank draws its own
reproducible tokens, the step time is the slowest rank's (max over ranks),
and the whole-job value counts every rank's tokens.  Run as two spawned
processes over gloo on 127.0.0.1."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from routing_dispatch_experts_b200 import workloads as W
        ms = [3.0, 5.0][rank]
        m = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        w = W.WORKLOADS[2]
        x = W.make_x(w, bench.replica_seed(0, rank), 64)
        q.put((rank, m, bench.job_value(w.T, world, m), float(x.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicate_the_bench_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import bench
    from routing_dispatch_experts_b200 import workloads as W
    w = W.WORKLOADS[2]
    # the step time is the slowest rank's on every rank
    assert [r[1] for r in res] == [5.0, 5.0]
    # whole-job throughput: both ranks' tokens over that time
    assert res[0][2] == pytest.approx(2 * w.T / 5e-3)
    # each replica draws its own tokens, reproducibly
    sums = [r[3] for r in res]
    assert sums[0] != sums[1]
    for rank in range(2):
        x = W.make_x(w, bench.replica_seed(0, rank), 64)
        assert float(x.float().sum()) == sums[rank]


def test_exchange_splits_match_brute_force():
    """Rows a rank sends each rank: one per assignment (B) or one per
    (token, destination rank) (D), against a loop over the tokens."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    g = np.random.default_rng(3)
    for P, E, k in ((2, 8, 2), (4, 16, 4), (8, 64, 6)):
        idx = np.stack([g.permutation(E)[:k] for _ in range(200)])
        m = g.permutation(np.repeat(np.arange(P), E // P))
        B = np.zeros(P, np.int64)
        D = np.zeros(P, np.int64)
        for t in range(len(idx)):
            for e in idx[t]:
                B[m[e]] += 1
            for r in set(int(m[e]) for e in idx[t]):
                D[r] += 1
        assert (bench.exchange_splits(idx, m, P, False) == B).all()
        assert (bench.exchange_splits(idx, m, P, True) == D).all()


def _exchange_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        g = np.random.default_rng(10 + rank)
        E, k = 8, 2
        idx = np.stack([g.permutation(E)[:k] for _ in range(100)])
        contig = [e // (E // world) for e in range(E)]
        other = [(e + 1) % E // (E // world) for e in range(E)]
        res = bench.ep_exchange(idx, contig, other, rank, world, 16, torch.float32,
                                torch.device("cpu"))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_ep_exchange_runs_on_gloo_ranks():
    """bench.ep_exchange's collectives on two CPU ranks: the same call
    sequence on every rank, and B puts at least as many rows on the wire
    as D."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_exchange_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        res = out[r]
        assert res["ranks"] == world and res["row_bytes"] == 64
        assert res["B"]["wire_rows_max_rank"] >= res["D"]["wire_rows_max_rank"] > 0
        assert all(res[n]["ms"] >= 0 for n in ("B", "D", "D+P"))
    assert out[0]["B"] == out[1]["B"]  # the slowest rank's time and rows, on every rank
