"""The whole layer (moe_forward) on seeded random shapes across the
boundary's range, against the oracle: T from 1 to 3000, d and f multiples
of 64 (the fused expert FFN where its shapes apply, the separate GEMMs
with 64- and 128-column gate/up blocks elsewhere, f = 1024 / 1536 for the
down GEMM on CTA pairs), E from 2 to 96 (not only
multiples of 16), k up to min(E, 16), every divisor of E as the EP degree
under contiguous or permuted placement, bf16 and fp32.  Checks: the
dispatch layout bit-exact against the oracle's layout of the GPU's
routing, routing equal to the oracle's away from near-ties, outputs within
2e-2 * max|y| (bf16) or 1e-5 (fp32)."""
import math

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe

from util import check_output, routing_mismatches

pytestmark = pytest.mark.gpu


def _shape(seed):
    g = np.random.default_rng(seed)
    dt = "f32" if g.random() < 0.25 else "bf16"
    E = int(g.choice([2, 3, 5, 8, 12, 16, 24, 33, 48, 64, 96]))
    k = int(g.integers(1, min(E, 16) + 1))
    d = int(g.choice([64, 128, 256, 384, 512, 1024]))
    f = int(g.choice([64, 128, 192, 256, 512]))
    T = int(g.choice([1, 7, 128, 129, 500, 1000, 3000]))
    divs = [p for p in range(1, E + 1) if E % p == 0]
    ep = int(g.choice(divs))
    rmap = None
    if ep > 1 and g.random() < 0.5:
        rmap = [int(v) for v in g.permutation(np.repeat(np.arange(ep), E // ep))]
    return T, d, E, k, f, ep, dt, rmap


def _shape_long_f(seed):
    """Expert widths of 1024 and 1536 on rows that are multiples of 256: the
    down GEMM runs on CTA pairs with ragged groups (bf16), the fp32 path on
    the CUDA cores."""
    g = np.random.default_rng(seed)
    dt = "f32" if g.random() < 0.2 else "bf16"
    E = int(g.choice([2, 5, 8, 12, 24]))
    k = int(g.integers(1, min(E, 3) + 1))
    d = int(g.choice([256, 512]))
    f = int(g.choice([1024, 1536]))
    T = int(g.choice([1, 7, 129, 300]))
    divs = [p for p in range(1, E + 1) if E % p == 0]
    ep = int(g.choice(divs))
    return T, d, E, k, f, ep, dt, None


@pytest.mark.parametrize("seed", range(64))
def test_forward_random_shape(seed):
    _run(seed, _shape(1000 + seed))


@pytest.mark.parametrize("seed", range(12))
def test_forward_random_shape_long_f(seed):
    _run(seed, _shape_long_f(2000 + seed))


def _run(seed, shape_args):
    T, d, E, k, f, ep, dt, rmap = shape_args
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(dtype)
    wr = (torch.randn((d, E), generator=g) * 0.05).to(dtype)
    wg = (torch.randn((E, d, f), generator=g) / math.sqrt(d)).to(dtype)
    wu = (torch.randn((E, d, f), generator=g) / math.sqrt(d)).to(dtype)
    wd = (torch.randn((E, f, d), generator=g) / math.sqrt(f)).to(dtype)
    shape = moe.Shape(T=T, d=d, E=E, k=k, f=f, ep=ep, dtype=dtype)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y = moe.forward(shape, x.cuda(), packed, None, ws, expert_rank=rmap, buffers=buf)
    moe.check_device_status(ws)
    idx = buf.topk_idx.cpu().numpy()
    # the layout, bit for bit, against the oracle's layout of this routing
    lay = oracle.dispatch_layout(idx, E, ep, rmap)
    for name in ("expert_counts", "expert_offsets", "row_token", "slot_row"):
        np.testing.assert_array_equal(buf.layout[name].cpu().numpy(), lay[name], err_msg=name)
    if ep > 1:
        for name in ("rank_counts", "rank_offsets", "slot_send_row"):
            np.testing.assert_array_equal(buf.layout[name].cpu().numpy(), lay[name], err_msg=name)
        n = int(lay["rank_offsets"][-1])
        np.testing.assert_array_equal(buf.layout["send_token"].cpu().numpy()[:n],
                                      lay["send_token"][:n])
    ref = oracle.forward(x, wr, None, wg, wu, wd, k)
    bad = routing_mismatches(idx, ref["idx"])
    assert (oracle.margin(ref["logits"], k)[bad] < 1e-5).all() if k < E else len(bad) == 0
    check_output(y, ref["y"], dt, rows=np.setdiff1d(np.arange(T), bad))
