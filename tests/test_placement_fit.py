"""moe_fit_placement, the library's host-side greedy correlated placement
("Expert Coupling in MoE Pretraining", Abstract: co-selected experts share a
GPU; Table III: W[e,e']), against the oracle's fit on the same routing.
Host code only: no GPU.  The counts come from the oracle here; the GPU
counts are compared with the oracle's in test_gpu_placement.py."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import build
from routing_dispatch_experts_b200 import workloads as W


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


@pytest.mark.parametrize("T,E,k,ep", [(4096, 64, 2, 8), (4096, 64, 2, 16), (2000, 64, 6, 32),
                                      (3000, 128, 8, 16), (500, 256, 16, 64), (100, 16, 4, 4),
                                      (0, 16, 2, 4), (37, 12, 3, 3)])
def test_fit_matches_oracle(T, E, k, ep):
    g = torch.Generator().manual_seed(T + E)
    # correlated routing: tokens draw their experts from a few planted groups
    groups = torch.randperm(E, generator=g).reshape(-1, max(1, E // 8))
    rows = []
    for t in range(T):
        grp = groups[t % len(groups)]
        pool = torch.cat([grp, torch.randperm(E, generator=g)])
        seen = []
        for e in pool.tolist():
            if e not in seen:
                seen.append(e)
            if len(seen) == k:
                break
        rows.append(seen)
    idx = np.array(rows, np.int32).reshape(T, k)
    counts = oracle.coselection_counts(idx, E)
    got = moe.fit_placement(E, ep, counts)
    assert got == oracle.fit_correlated_placement(idx, E, ep)
    assert sorted(got.count(r) for r in range(ep)) == [E // ep] * ep


def test_fit_ties_take_the_lowest_index():
    """All counts equal (or zero): the fit degenerates to contiguous."""
    E, ep = 32, 4
    assert moe.fit_placement(E, ep, np.zeros((E, E), np.int64)) == W.contiguous_placement(E, ep)
    assert moe.fit_placement(E, ep, np.ones((E, E), np.int64)) == W.contiguous_placement(E, ep)


def test_fit_rejects_bad_arguments():
    L = moe.lib()
    out = (moe.ctypes.c_int32 * 16)()
    c = np.zeros(256, np.uint64)
    assert L.moe_fit_placement(16, 3, c.ctypes.data_as(moe.ctypes.c_void_p), out) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_fit_placement(16, 4, None, out) == moe.MOE_ERR_INVALID_ARG
