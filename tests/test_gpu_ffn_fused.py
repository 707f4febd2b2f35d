"""GPU parity of the fused expert FFN (gate/up GEMM + SwiGLU + down GEMM in
one kernel, H kept on chip), which moe_forward takes for bf16 with f in
{64, 128} and d in {128, 256}.

It must give bit-for-bit the y_perm and output of the separate kernels (the
grouped SwiGLU GEMMs, then moe_combine) on the forward's own routing, and
match the oracle's experts and combine on that routing within the bf16
tolerance.
Cases: both (f, d) sizes, top-1 to top-8, ragged and empty experts, one
expert holding most rows, and the non-gather mode (x larger than the
gathered-operand limit)."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

from util import TOL

pytestmark = pytest.mark.gpu


def _inputs(T, d, E, k, f, seed, skew=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).bfloat16()
    wr = (torch.randn(d, E, generator=g) * 0.02).bfloat16()
    if skew:  # expert 0's router column dominates: most tokens pick it
        wr[:, 0] = (torch.randn(d, generator=g) * 0.2).bfloat16()
    wg = (torch.randn(E, d, f, generator=g) / d ** 0.5).bfloat16()
    wu = (torch.randn(E, d, f, generator=g) / d ** 0.5).bfloat16()
    wd = (torch.randn(E, f, d, generator=g) / d ** 0.5).bfloat16()
    return x, wr, wg, wu, wd


def _fused_and_separate(T, d, E, k, f, seed, skew=False, ep=1):
    x, wr, wg, wu, wd = _inputs(T, d, E, k, f, seed, skew)
    shape = moe.Shape(T=T, d=d, E=E, k=k, f=f, ep=ep)
    dev = "cuda"
    dx = x.to(dev)
    packed = moe.pack_weights(shape, wr.to(dev), wg.to(dev), wu.to(dev), wd.to(dev))
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y = moe.forward(shape, dx, packed, None, ws, buffers=buf)
    moe.check_device_status(ws)
    # the separate kernels on the same routing
    lay = buf.layout
    ws2 = moe.workspace(shape)
    _, y_perm = moe.grouped_swiglu_gather(shape, dx, lay["row_token"], lay["expert_offsets"],
                                          packed, ws2)
    y_sep = moe.combine(shape, y_perm, lay["slot_row"], buf.topk_gate)
    moe.check_device_status(ws2)
    assert torch.equal(buf.y_perm, y_perm)
    return (x, wg, wu, wd), shape, buf, y, y_sep


def _check_oracle(inp, shape, buf, y, tokens):
    """Oracle experts + combine on the GPU's routing, for `tokens`."""
    x, wg, wu, wd = inp
    idx = buf.topk_idx.cpu().numpy()
    gate = buf.topk_gate.cpu().double().numpy()
    ref = oracle.moe_output(x, idx[tokens], gate[tokens], wg, wu, wd, tokens=tokens)
    yg = y.cpu().double().numpy()[tokens]
    scale = np.abs(ref).max()
    assert np.abs(yg - ref).max() <= TOL["bf16"] * scale


@pytest.mark.parametrize("T,d,E,k,f,skew", [
    (2311, 256, 64, 4, 64, False),   # the fine-grained workload's shape
    (777, 128, 16, 2, 64, False),
    (1500, 256, 32, 8, 128, False),
    (900, 128, 8, 1, 128, False),
    (3000, 256, 64, 4, 64, True),    # one expert holds a large share of the rows
    (129, 256, 64, 6, 64, False),    # most experts empty, ragged tails
])
def test_fused_ffn_equals_separate_kernels_and_oracle(T, d, E, k, f, skew):
    inp, shape, buf, y, y_sep = _fused_and_separate(T, d, E, k, f, seed=T + k, skew=skew)
    assert torch.equal(y, y_sep)
    toks = np.arange(T) if T <= 1000 else np.unique(W.sample_tokens(T, 400, seed=1).numpy())
    _check_oracle(inp, shape, buf, y, toks)
    if skew:
        counts = buf.layout["expert_counts"].cpu()
        assert int(counts.max()) > T // 3


def test_fused_ffn_repeatable_and_ep_invariant():
    """Back-to-back calls on one workspace give identical outputs, for any EP
    degree."""
    T, d, E, k, f = 2000, 256, 64, 4, 64
    x, wr, wg, wu, wd = _inputs(T, d, E, k, f, seed=5)
    dx = x.cuda()
    ys = []
    for ep in (1, 8, 1, 64):
        shape = moe.Shape(T=T, d=d, E=E, k=k, f=f, ep=ep)
        packed = moe.pack_weights(shape, wr.cuda(), wg.cuda(), wu.cuda(), wd.cuda())
        ws = moe.workspace(shape, forward=True)
        ys.append(moe.forward(shape, dx, packed, None, ws))
        ys.append(moe.forward(shape, dx, packed, None, ws))
        moe.check_device_status(ws)
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_fused_ffn_without_gather():
    """x beyond the gathered-operand limit (96 MB): the forward permutes in
    token order and the fused kernel loads x_perm tiles by TMA."""
    T, d, E, k, f = 200_000, 256, 64, 4, 64   # x = 102 MB
    inp, shape, buf, y, y_sep = _fused_and_separate(T, d, E, k, f, seed=11)
    assert torch.equal(y, y_sep)
    toks = np.unique(np.concatenate([[0, T - 1], W.sample_tokens(T, 64, seed=2).numpy()]))
    _check_oracle(inp, shape, buf, y, toks)
