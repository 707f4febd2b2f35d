"""GPU co-selection counts W[e,e'] ("Expert Coupling in MoE Pretraining",
Table III) bit-exact against oracle.coselection_counts, the placement fit on
them equal to the oracle's, and a forward under the GPU-fitted placement
removing more duplicate send rows than the contiguous one (Table I)."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import Case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k", [(5000, 64, 2), (3000, 64, 6), (2048, 128, 8), (700, 256, 16),
                                   (1, 16, 4), (0, 16, 4), (999, 12, 5)])
def test_coselection_counts_bit_exact(T, E, k):
    idx = W.uniform_routing(T, E, k, seed=T + k)
    if T > 10:
        idx[::5, 1] = idx[::5, 0]  # repeated experts count as the oracle counts them
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    ws = moe.workspace(shape)
    Wg = moe.coselection_counts(shape, idx.cuda(), ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    np.testing.assert_array_equal(Wg.cpu().numpy(), oracle.coselection_counts(idx.numpy(), E))


def test_coselection_bad_index():
    T, E, k = 300, 16, 2
    idx = W.uniform_routing(T, E, k, seed=3)
    idx[5, 0] = -1
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    ws = moe.workspace(shape)
    Wg = moe.coselection_counts(shape, idx.cuda(), ws)
    assert moe.get_device_status(ws) == moe.MOE_ERR_DEVICE_INDEX
    ok = np.delete(idx.numpy(), 5, axis=0)
    np.testing.assert_array_equal(Wg.cpu().numpy(), oracle.coselection_counts(ok, E))


@pytest.mark.parametrize("ep", [8, 16])
def test_gpu_fit_on_calibration_batch(ep):
    """The top-2 workload: the GPU routes a calibration batch (another
    stream of the same distribution), counts co-selections and the library
    fits the placement; it equals the oracle's fit on the same routing, and
    the forward under it removes more duplicate rows than contiguous
    placement ('Expert Coupling', Table I)."""
    c = Case(3, T=4096, near_ties=False)
    w = c.w
    cal = W.make_x(w, 0, 4096, stream="calib").cuda()
    shape = c.shape_ep(ep)
    ws = moe.workspace(shape, forward=True)
    _, cidx, _ = moe.route(shape, cal, c.packed, None, ws)
    Wg = moe.coselection_counts(shape, cidx, ws)
    moe.check_device_status(ws)
    fit = moe.fit_placement(w.E, ep, Wg)
    assert fit == oracle.fit_correlated_placement(cidx.cpu().numpy(), w.E, ep)
    stats = {}
    for name, rmap in (("contiguous", W.contiguous_placement(w.E, ep)), ("fit", fit)):
        buf = moe.ForwardBuffers(shape)
        moe.forward(shape, c.dx, c.packed, None, ws, expert_rank=rmap, buffers=buf)
        moe.check_device_status(ws)
        stats[name] = moe.stats_dict(buf.layout["stats"])
        ref = oracle.dispatch_layout(buf.topk_idx.cpu().numpy(), w.E, ep, rmap)["stats"]
        assert stats[name] == ref
    assert stats["fit"]["dup_removed"] > stats["contiguous"]["dup_removed"]
