"""The expert-parallel exchange on CPU: world_size 2 and 4 gloo ranks run the
send plan, count exchange, row all-to-all, return all-to-all and home
combine of routing_dispatch_experts_b200.ep (TorchExchange, splits), with
the per-rank compute done by the oracle in double (the CUDA kernels of the
same steps are checked on the GPU in test_gpu_ep.py).  The concatenated
output equals the oracle's single-process layer.

Failure injection on the host: a rank that raises after the count exchange
(and leaves the group) makes its peer's next collective end with an error
within the process group's timeout, never a hang."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOKENS_PER_RANK = 48


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(world):
    from routing_dispatch_experts_b200 import workloads as W
    w = W.WORKLOADS[1]  # fp32, E = 16, top-4
    T = TOKENS_PER_RANK * world
    x = W.make_x(w, 0, T)
    wr = W.make_router(w)
    wg, wu, wd = W.make_experts(w)
    rmap = W.permutation_placement(w.E, world, seed=world)
    return w, x, wr, wg, wu, wd, rmap


def _worker(rank, world, port, q, fail_rank):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=15))
    try:
        import oracle
        from routing_dispatch_experts_b200.ep import TorchExchange, local_experts, splits
        w, x_all, wr, wg, wu, wd, rmap = _inputs(world)
        T = TOKENS_PER_RANK
        x = x_all[rank * T:(rank + 1) * T]
        idx, gate = oracle.topk(oracle.router_logits(x, wr), w.k)
        lay = oracle.dispatch_layout(idx, w.E, world, rmap)
        ex = TorchExchange()
        counts = ex.counts(torch.from_numpy(lay["rank_counts"]))
        if rank == fail_rank:
            raise RuntimeError("injected failure")
        s_sp, r_sp = splits(counts, rank)
        assert s_sp == lay["rank_counts"].tolist()
        # the send rows, as moe_ep_pack lays them out: grouped by destination,
        # experts as the destination's local ids (E/P for "held elsewhere")
        E_loc = w.E // world
        local_id = {e: local_experts(rmap, rmap[e]).index(e) for e in range(w.E)}
        st = lay["send_token"]
        dest = np.searchsorted(lay["rank_offsets"], np.arange(len(st)), side="right") - 1
        send_x = x[torch.from_numpy(st).long()]
        send_idx = np.array([[local_id[e] if rmap[e] == dest[s] else E_loc for e in idx[t]]
                             for s, t in enumerate(st)], np.int32).reshape(-1, w.k)
        send_gate = gate[st]
        recv_x = ex.rows(send_x, s_sp, r_sp)
        recv_idx = ex.rows(torch.from_numpy(send_idx), s_sp, r_sp).numpy()
        recv_gate = ex.rows(torch.from_numpy(send_gate), s_sp, r_sp).numpy()
        # this rank's experts on the received rows (oracle, double)
        mine = np.array(local_experts(rmap, rank))
        here = recv_idx < E_loc
        gidx = np.where(here, mine[np.minimum(recv_idx, E_loc - 1)], 0).astype(np.int32)
        y_ret = oracle.moe_output(recv_x, gidx, np.where(here, recv_gate, 0.0), wg, wu, wd)
        y_back = ex.rows(torch.from_numpy(y_ret), r_sp, s_sp).numpy()
        assert y_back.shape[0] == len(st)
        # home combine: each token's distinct send rows
        ssr = lay["slot_send_row"].reshape(T, w.k)
        y = np.stack([y_back[sorted(set(ssr[t].tolist()))].sum(0) for t in range(T)])
        q.put((rank, "ok", y, counts))
    except Exception as e:  # reported to the test, which decides
        q.put((rank, "error", repr(e), None))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def _run(world, fail_rank=-1):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return res


@pytest.mark.parametrize("world", [2, 4])
def test_ep_exchange_round_trip_equals_the_layer(world):
    sys.path.insert(0, ROOT)
    import oracle
    res = _run(world)
    assert [r[1] for r in res] == ["ok"] * world, [r[2] for r in res if r[1] != "ok"]
    w, x, wr, wg, wu, wd, rmap = _inputs(world)
    ref = oracle.forward(x, wr, None, wg, wu, wd, w.k)
    y = np.concatenate([r[2] for r in res])
    np.testing.assert_allclose(y, ref["y"], rtol=1e-12, atol=1e-12)
    # every rank saw the same count matrix; its row sums are the
    # deduplicated rows each rank sends (one per token and destination)
    counts = res[0][3]
    assert all(r[3] == counts for r in res)
    lay = oracle.dispatch_layout(ref["idx"][:TOKENS_PER_RANK], w.E, world, rmap)
    assert counts[0] == lay["rank_counts"].tolist()


def test_ep_exchange_peer_failure_is_an_error_not_a_hang():
    res = _run(2, fail_rank=1)
    assert res[1][1] == "error" and "injected failure" in res[1][2]
    # the surviving rank's collective ended with an error
    assert res[0][1] == "error"
