"""The whole layer (moe_forward) at the edges of its shape range, against
the oracle: no tokens, one token, a handful of tokens over a few experts,
the widest rows the boundary accepts (d = 8192 in bf16 and d = 4096 in
fp32: 16 KB rows), k = E, and top-16 with f = 192 (64-column gate/up
blocks).  Routing is
compared as expert sets (a token whose oracle margin is below 1e-5 may
differ); outputs within 2e-2 * max|y| (bf16) or 1e-5 (fp32)."""
import math

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe

from util import check_output, routing_mismatches

pytestmark = pytest.mark.gpu


def _inputs(T, d, E, f, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(dtype)
    wr = (torch.randn((d, E), generator=g) * 0.02).to(dtype)
    wg = (torch.randn((E, d, f), generator=g) / math.sqrt(d)).to(dtype)
    wu = (torch.randn((E, d, f), generator=g) / math.sqrt(d)).to(dtype)
    wd = (torch.randn((E, f, d), generator=g) / math.sqrt(f)).to(dtype)
    return x, wr, wg, wu, wd


@pytest.mark.parametrize("T,d,E,k,f,dt,ep", [
    (1, 256, 8, 2, 64, "bf16", 1),        # one token
    (3, 128, 4, 2, 128, "bf16", 2),       # fewer tokens than experts, EP 2
    (5, 64, 4, 4, 64, "f32", 1),          # k = E: every expert for every token
    (64, 8192, 8, 2, 128, "bf16", 4),     # widest bf16 rows (16 KB), short down GEMM
    (96, 8192, 8, 2, 1536, "bf16", 1),    # widest bf16 rows, down GEMM on CTA pairs
    (40, 4096, 8, 2, 64, "f32", 1),       # widest fp32 rows (16 KB)
    (129, 2048, 16, 16, 192, "bf16", 8),  # top-16, ragged tiles
])
def test_forward_edge_shapes(T, d, E, k, f, dt, ep):
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    x, wr, wg, wu, wd = _inputs(T, d, E, f, dtype, seed=T * 131 + d)
    shape = moe.Shape(T=T, d=d, E=E, k=k, f=f, ep=ep, dtype=dtype)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y = moe.forward(shape, x.cuda(), packed, None, ws, buffers=buf)
    moe.check_device_status(ws)
    ref = oracle.forward(x, wr, None, wg, wu, wd, k)
    idx = buf.topk_idx.cpu().numpy()
    bad = routing_mismatches(idx, ref["idx"])
    assert (oracle.margin(ref["logits"], k)[bad] < 1e-5).all()
    ok = np.setdiff1d(np.arange(T), bad)
    assert len(ok) >= T - 1
    check_output(y, ref["y"], dt, rows=ok)
    # every token got k distinct experts, gates summing to one
    assert (np.sort(idx, 1)[:, 1:] != np.sort(idx, 1)[:, :-1]).all()
    np.testing.assert_allclose(buf.topk_gate.cpu().double().numpy().sum(1), 1.0, atol=1e-6)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_forward_zero_tokens(dt):
    """T = 0: the call succeeds, launches nothing that writes, and the
    workspace stays usable for the next call."""
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    shape = moe.Shape(T=0, d=256, E=8, k=2, f=64, ep=2, dtype=dtype)
    x0, wr, wg, wu, wd = _inputs(1, 256, 8, 64, dtype, seed=5)
    packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
    ws = moe.workspace(shape, forward=True)
    y = moe.forward(shape, torch.empty((0, 256), dtype=dtype, device="cuda"), packed, None, ws)
    assert y.shape == (0, 256)
    assert moe.get_device_status(ws) == moe.MOE_OK
