"""The router and the expert FFN called on weights in the pages' layouts
(W_r [d, E] "ME"; W_g, W_u [E, d, f] "EMH"; W_d [E, f, d] "EHM"; "Revisiting
MoE and Dense Speed-Accuracy Comparisons", Table 1) through the C ABI give
the packed path's results bit for bit."""
import pytest
import torch

import routing_dispatch_experts_b200 as moe

from util import Case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,T", [(1, 700), (2, 1000), (3, 300), (5, 257)])
def test_route_unpacked_equals_packed(cfg, T):
    c = Case(cfg, T=T, near_ties=False)
    ws = moe.workspace(c.shape)
    a = moe.route(c.shape, c.dx, c.packed, c.dbias, ws)
    uws = moe.unpacked_workspace(c.shape)
    b = moe.route_unpacked(c.shape, c.dx, c.wr.cuda(), c.dbias, uws)
    assert moe.get_device_status(uws) == moe.MOE_OK
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("cfg,T", [(1, 600), (2, 900), (3, 257)])
def test_grouped_unpacked_equals_packed(cfg, T):
    c = Case(cfg, T=T, near_ties=False)
    ws = moe.workspace(c.shape)
    _, idx, _ = moe.route(c.shape, c.dx, c.packed, c.dbias, ws)
    lay = moe.dispatch_layout(c.shape, idx, ws)
    x_perm = moe.permute(c.shape, c.dx, lay["row_token"])
    h0, y0 = moe.grouped_swiglu(c.shape, x_perm, lay["expert_offsets"], c.packed, ws)
    uws = moe.unpacked_workspace(c.shape)
    h1, y1 = moe.grouped_swiglu_unpacked(c.shape, x_perm, lay["expert_offsets"], c.wg.cuda(),
                                         c.wu.cuda(), c.wd.cuda(), uws)
    assert moe.get_device_status(uws) == moe.MOE_OK
    assert torch.equal(h0, h1) and torch.equal(y0, y1)
