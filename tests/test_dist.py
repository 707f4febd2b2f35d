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
