"""GPU parity of moe_permute (bit-exact copy) and moe_combine (k*x identity
bit-exact; gate-weighted sums within fp32-accumulation tolerance)."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,T", [(1, 2048), (2, 16384), (2, 77), (3, 1025), (5, 301), (5, 1)])
def test_permute_bit_exact(cfg, T):
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, T=T)
    idx = W.uniform_routing(T, w.E, w.k, seed=T)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    rt = torch.from_numpy(lay["row_token"])
    x_perm = moe.permute(shape, x.cuda(), rt.cuda())
    assert torch.equal(x_perm.cpu(), x[rt.long()])


@pytest.mark.parametrize("cfg,T", [(1, 2048), (2, 1000), (3, 1025), (4, 77), (5, 301), (5, 1)])
def test_permute_by_token_bit_exact(cfg, T):
    """The token-order copy writes the same x_perm as the gather."""
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, T=T)
    idx = W.uniform_routing(T, w.E, w.k, seed=T + 3)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    x_perm = moe.permute_by_token(shape, x.cuda(), torch.from_numpy(lay["slot_row"]).cuda())
    assert torch.equal(x_perm.cpu(), x[torch.from_numpy(lay["row_token"]).long()])


@pytest.mark.parametrize("cfg,T", [(1, 2048), (2, 4099), (3, 513), (4, 300), (5, 129)])
def test_identity_experts_unit_gates_give_k_x(cfg, T):
    """Permute, then combine with the experts replaced by the identity and
    unit gates: k*x exactly (k*x is exact in fp32, then rounded once)."""
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, T=T)
    idx = W.uniform_routing(T, w.E, w.k, seed=5 + T)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    dx = x.cuda()
    rt = torch.from_numpy(lay["row_token"])
    x_perm = moe.permute(shape, dx, rt.cuda())
    y = moe.combine(shape, x_perm, torch.from_numpy(lay["slot_row"]).cuda(), None)
    ref = torch.from_numpy(oracle.combine(x[rt.long()], lay["slot_row"], None, k=w.k))
    assert torch.equal(y.cpu(), ref.to(w.torch_dtype))
    assert torch.equal(y.cpu(), (x.double() * w.k).to(w.torch_dtype))


@pytest.mark.parametrize("cfg,T", [(1, 2048), (2, 3001), (4, 257), (5, 100)])
def test_weighted_combine(cfg, T):
    w = W.WORKLOADS[cfg]
    idx = W.uniform_routing(T, w.E, w.k, seed=T + 1)
    lay = oracle.dispatch_layout(idx.numpy(), w.E, 1)
    g = torch.Generator().manual_seed(T)
    y_perm = torch.randn((T * w.k, w.d), generator=g).to(w.torch_dtype)
    gate = torch.softmax(torch.randn((T, w.k), generator=g), 1)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, dtype=w.torch_dtype)
    y = moe.combine(shape, y_perm.cuda(), torch.from_numpy(lay["slot_row"]).cuda(), gate.cuda())
    ref = oracle.combine(y_perm, lay["slot_row"], gate.double().numpy())
    # fp32 accumulation of k terms, then one rounding to the storage type
    absum = oracle.combine(y_perm.abs(), lay["slot_row"], gate.double().numpy())
    ulp = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -23
    err = np.abs(y.cpu().double().numpy() - ref)
    assert (err <= ulp * np.abs(ref) + 1e-6 * absum + 1e-30).all()
