"""GPU parity of moe_route: the router GEMM and the top-k + gates kernel.

Routing indices are bit-exact against the oracle when both are given the
same fp32 logits (synthetic, drawn on the CPU); gates within 1e-6.  The
router GEMM is compared with the oracle's double logits."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import NEAR_TIE, Case, routing_mismatches

pytestmark = pytest.mark.gpu


def _given_logits(T, E, k, seed, ties):
    g = torch.Generator().manual_seed(seed)
    if ties:
        vals = torch.tensor([-1.5, -0.0, 0.0, 0.25, 0.25, 2.0, 7.0, 1e-30, -1e-30])
        l = vals[torch.randint(0, len(vals), (T, E), generator=g)]
    else:
        l = torch.randn((T, E), generator=g) * 2
    return l.contiguous()


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (1000, 16, 4), (4097, 64, 4), (3001, 64, 2),
                                   (2049, 64, 6), (2500, 128, 8), (777, 256, 16), (300, 33, 5),
                                   (64, 8, 8), (513, 200, 1)])
@pytest.mark.parametrize("ties", [False, True])
def test_topk_given_logits_bit_exact(T, E, k, ties):
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64)
    l = _given_logits(T, E, k, T + E + k, ties)
    ws = moe.workspace(shape)
    _, idx, gate = moe.route(shape, None, None, None, ws, logits=l.cuda())
    ref_idx, ref_gate = oracle.topk(l.double().numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(gate.cpu().double().numpy(), ref_gate, rtol=0, atol=1e-6)
    np.testing.assert_allclose(gate.sum(1).cpu().numpy(), 1.0, atol=1e-6)
    assert moe.get_device_status(ws) == moe.MOE_OK


def test_topk_signed_zero_and_exact_ties():
    shape = moe.Shape(T=3, d=64, E=8, k=3, f=64)
    l = torch.zeros(3, 8)
    l[1, [2, 5, 6]] = 1.0
    l[2] = torch.tensor([-0.0, 0.0, -0.0, 0.0, 1, 1, -1, -1])
    _, idx, gate = moe.route(shape, None, None, None, moe.workspace(shape), logits=l.cuda())
    assert idx.cpu().tolist() == [[0, 1, 2], [2, 5, 6], [4, 5, 0]]
    assert torch.allclose(gate[0].cpu(), torch.full((3,), 1 / 3))


@pytest.mark.parametrize("cfg,T", [(1, 2048), (2, 1531), (3, 700), (5, 389)])
def test_router_logits_and_routing(cfg, T):
    c = Case(cfg, T=T, near_ties=False)
    ws = moe.workspace(c.shape)
    logits, idx, gate = moe.route(c.shape, c.dx, c.packed, c.dbias, ws)
    moe.check_device_status(ws)
    ref = oracle.router_logits(c.x, c.wr, c.bias)
    # fp32 accumulation of K products: bound the error by the magnitude sum
    mag = (c.x.double().abs() @ c.wr.double().abs()).numpy()
    err = np.abs(logits.cpu().double().numpy() - ref)
    assert (err <= 1e-5 * mag + 1e-6).all(), float((err / (mag + 1e-30)).max())
    # routing against the oracle's own routing: differences only at near-ties
    ref_idx, ref_gate = oracle.topk(ref, c.w.k)
    gi = idx.cpu().numpy()
    bad = routing_mismatches(gi, ref_idx)
    m = oracle.margin(ref, c.w.k)
    assert (m[bad] < NEAR_TIE).all()
    ok = np.setdiff1d(np.arange(T), bad)
    # same expert sets; compare the gates expert by expert (two chosen experts
    # closer than fp32 rounding may appear in either slot order)
    og, orf = np.argsort(gi[ok], 1), np.argsort(ref_idx[ok], 1)
    gg = np.take_along_axis(gate.cpu().double().numpy()[ok], og, 1)
    rg = np.take_along_axis(ref_gate[ok], orf, 1)
    np.testing.assert_allclose(gg, rg, atol=1e-5)


def test_route_zero_tokens():
    shape = moe.Shape(T=0, d=256, E=16, k=4, f=256)
    l = torch.empty(0, 16, device="cuda")
    _, idx, gate = moe.route(shape, None, None, None, moe.workspace(shape), logits=l)
    assert idx.numel() == 0


def _bf16_router_case(T, d, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).bfloat16()
    wr = (torch.randn(d, E, generator=g) * 0.05).bfloat16()
    f = 64
    wg = (torch.randn(E, d, f, generator=g) * 0.02).bfloat16()
    shape = moe.Shape(T=T, d=d, E=E, k=k, f=f)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wg.cuda(), wg.transpose(1, 2).contiguous().cuda())
    return x, wr, shape, packed


@pytest.mark.parametrize("T,d,E,k", [(1000, 64, 12, 3), (777, 256, 16, 4), (333, 128, 33, 5),
                                     (1500, 512, 96, 6), (900, 256, 256, 16), (129, 64, 64, 2)])
def test_bf16_router_logit_layouts_and_ragged_tiles(T, d, E, k):
    """The tensor-core router for every way its logits tile leaves the SM
    (TMA tiled stores for E % 32 == 0 -- 2 to 8 boxes --, a coalesced copy
    for E % 4 == 0, per-thread stores otherwise) and a ragged last tile: the
    logits match the oracle's double router within the fp32 accumulation
    bound, and its top-k is bit-exact against the oracle's top-k of the
    same fp32 logits."""
    x, wr, shape, packed = _bf16_router_case(T, d, E, k, seed=T + E)
    ws = moe.workspace(shape)
    logits, idx, gate = moe.route(shape, x.cuda(), packed, None, ws)
    moe.check_device_status(ws)
    ref = oracle.router_logits(x, wr)
    mag = (x.double().abs() @ wr.double().abs()).numpy()
    err = np.abs(logits.cpu().double().numpy() - ref)
    assert (err <= 1e-5 * mag + 1e-6).all()
    ref_idx, ref_gate = oracle.topk(logits.cpu().double().numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(gate.cpu().double().numpy(), ref_gate, rtol=0, atol=1e-6)


@pytest.mark.parametrize("T,d,E,k", [(19205, 256, 64, 4), (19205, 128, 36, 5), (19205, 64, 12, 3),
                                     (20000, 256, 128, 8), (19205, 128, 64, 16),
                                     (19205, 64, 256, 6), (19205, 64, 192, 2), (19205, 128, 192, 4),
                                     (19205, 64, 224, 8)])
def test_bf16_router_more_tiles_than_sms(T, d, E, k):
    """More 128-token tiles than SMs (151 or 157 tiles: two CTAs on some
    SMs, with the ring and the staged logits of each in half the shared
    memory), up to E = 256 experts.  Same checks as above for every way the
    logits leave the SM and for k up to 16."""
    x, wr, shape, packed = _bf16_router_case(T, d, E, k, seed=T + 3 * E)
    ws = moe.workspace(shape)
    logits, idx, gate = moe.route(shape, x.cuda(), packed, None, ws)
    moe.check_device_status(ws)
    ref = oracle.router_logits(x, wr)
    mag = (x.double().abs() @ wr.double().abs()).numpy()
    err = np.abs(logits.cpu().double().numpy() - ref)
    assert (err <= 1e-5 * mag + 1e-6).all()
    ref_idx, ref_gate = oracle.topk(logits.cpu().double().numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(gate.cpu().double().numpy(), ref_gate, rtol=0, atol=1e-6)


def test_bf16_router_unaligned_logits_buffer():
    """A logits buffer that is only 4-byte aligned takes the per-thread
    store path and gives the same bits as an aligned one."""
    import ctypes
    T, d, E, k = 700, 256, 64, 4
    x, wr, shape, packed = _bf16_router_case(T, d, E, k, seed=5)
    ws = moe.workspace(shape)
    dx = x.cuda()
    l0, i0, g0 = moe.route(shape, dx, packed, None, ws)
    base = torch.empty(T * E + 4, dtype=torch.float32, device="cuda")
    l1 = base[1:1 + T * E].view(T, E)
    i1 = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g1 = torch.empty(T, k, dtype=torch.float32, device="cuda")
    s = shape.c
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = moe.lib().moe_route(ctypes.byref(s), p(dx), p(packed), None, p(l1), p(i1), p(g1), p(ws),
                             ws.numel(), None)
    assert st == moe.MOE_OK
    moe.check_device_status(ws)
    assert torch.equal(l1, l0) and torch.equal(i1, i0) and torch.equal(g1, g0)
