"""Host plan of the peer-memory exchange: peer_blocks puts every rank's
send block where the all-to-all puts it (LocalExchange.rows), and every
return block back where the reverse all-to-all does (rows_back) -- checked
with labelled rows over random count matrices, including empty blocks."""
import numpy as np
import pytest
import torch

from routing_dispatch_experts_b200.ep import LocalExchange, peer_blocks


def _counts(P, seed):
    g = np.random.default_rng(seed)
    c = g.integers(0, 6, size=(P, P))
    c[g.random((P, P)) < 0.3] = 0  # empty blocks
    return c.tolist()


@pytest.mark.parametrize("P,seed", [(2, 0), (3, 1), (4, 2), (8, 3), (8, 4), (16, 5)])
def test_peer_blocks_place_rows_like_the_all_to_all(P, seed):
    counts = _counts(P, seed)
    # send row j of rank s carries the label (s, j)
    sends = [torch.tensor([[s, j] for j in range(sum(counts[s]))], dtype=torch.int64).reshape(-1, 2)
             for s in range(P)]
    want = LocalExchange(P).rows(sends, counts)
    got = [torch.full((sum(counts[q][r] for q in range(P)), 2), -1, dtype=torch.int64)
           for r in range(P)]
    for s in range(P):
        dests, _ = peer_blocks(counts, s)
        off = np.concatenate([[0], np.cumsum(counts[s])])
        for r, (row0, rows) in enumerate(dests):
            assert rows == counts[s][r]
            got[r][row0:row0 + rows] = sends[s][off[r]:off[r] + rows]
    for r in range(P):
        assert torch.equal(got[r], want[r]), r


@pytest.mark.parametrize("P,seed", [(2, 0), (4, 2), (8, 3), (16, 5)])
def test_peer_returns_go_back_to_the_send_rows(P, seed):
    counts = _counts(P, seed)
    # received row i of rank r carries the label (r, i)
    n_recv = [sum(counts[q][r] for q in range(P)) for r in range(P)]
    rets = [torch.tensor([[r, i] for i in range(n_recv[r])], dtype=torch.int64).reshape(-1, 2)
            for r in range(P)]
    want = LocalExchange(P).rows_back(rets, counts)
    got = [torch.full((sum(counts[s]), 2), -1, dtype=torch.int64) for s in range(P)]
    for r in range(P):
        _, back = peer_blocks(counts, r)
        assert sum(rows for _, rows in back) == n_recv[r]
        base = 0
        for s, (row0, rows) in enumerate(back):
            got[s][row0:row0 + rows] = rets[r][base:base + rows]
            base += rows
    for s in range(P):
        assert torch.equal(got[s], want[s]), s
