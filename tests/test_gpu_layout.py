"""GPU parity of moe_dispatch_layout: bit-exact against the oracle on the
same (CPU-drawn) routing, including ragged and empty inputs, the largest
expert / rank counts, correlated and permuted placements, and the bounded
wait of the decoupled lookback."""
import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

pytestmark = pytest.mark.gpu

KEYS = ("expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
        "rank_offsets", "slot_send_row")


def _check(T, E, k, ep, rmap, idx):
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64, ep=ep)
    ws = moe.workspace(shape)
    out = moe.dispatch_layout(shape, idx.cuda(), ws, expert_rank=rmap)
    assert moe.get_device_status(ws) == moe.MOE_OK
    ref = oracle.dispatch_layout(idx.numpy(), E, ep, rmap)
    for key in KEYS:
        if key.startswith("rank") or key == "slot_send_row":
            if ep == 1:
                continue
        np.testing.assert_array_equal(out[key].cpu().numpy(), ref[key], err_msg=key)
    if ep > 1:
        n = int(ref["stats"]["rows_sent"])
        np.testing.assert_array_equal(out["send_token"][:n].cpu().numpy(), ref["send_token"])
    assert moe.stats_dict(out["stats"]) == ref["stats"]
    return ws, shape


@pytest.mark.parametrize("T,E,k,ep,placement", [
    (1, 16, 4, 1, "contiguous"), (2, 4, 4, 2, "contiguous"), (511, 16, 4, 4, "contiguous"),
    (512, 64, 4, 8, "contiguous"), (513, 64, 4, 8, "permutation"), (2048, 16, 4, 1, "contiguous"),
    (16384, 64, 4, 8, "contiguous"), (16384, 64, 2, 16, "permutation"), (16385, 64, 6, 32, "permutation"),
    (32768, 128, 8, 16, "contiguous"), (5000, 256, 16, 256, "permutation"), (3000, 256, 8, 1, "contiguous"),
    (4099, 256, 3, 64, "permutation"), (1000, 12, 5, 3, "contiguous"),
])
def test_layout_bit_exact(T, E, k, ep, placement):
    idx = W.uniform_routing(T, E, k, seed=T + 7 * E + k)
    rmap = W.contiguous_placement(E, ep) if placement == "contiguous" else \
        W.permutation_placement(E, ep, seed=3)
    _check(T, E, k, ep, rmap, idx)


def test_layout_skewed_and_degenerate_routing():
    # every token on the same k experts (one expert group holds everything)
    T, E, k = 3000, 64, 4
    idx = torch.tensor([[5, 9, 2, 63]] * T, dtype=torch.int32)
    _check(T, E, k, 8, W.contiguous_placement(E, 8), idx)
    # Zipf-like skew: experts drawn with heavy preference, distinct per token
    g = torch.Generator().manual_seed(1)
    p = torch.arange(1, E + 1, dtype=torch.float64).pow(-1.1)
    rows = [torch.multinomial(p, k, replacement=False, generator=g) for _ in range(T)]
    _check(T, E, k, 16, W.permutation_placement(E, 16, seed=9), torch.stack(rows).int())


def test_layout_reuses_workspace_across_calls_and_shapes():
    """The lookback state is left clean: back-to-back calls of different
    sizes on one workspace keep giving exact layouts."""
    big = moe.Shape(T=9000, d=64, E=64, k=6, f=64, ep=32)
    ws = moe.workspace(big)
    for T, k, ep in [(9000, 6, 32), (100, 2, 8), (9000, 6, 32), (4000, 4, 1), (1, 1, 64)]:
        shape = moe.Shape(T=T, d=64, E=64, k=k, f=64, ep=ep)
        idx = W.uniform_routing(T, 64, k, seed=T * k)
        out = moe.dispatch_layout(shape, idx.cuda(), ws)
        ref = oracle.dispatch_layout(idx.numpy(), 64, ep)
        np.testing.assert_array_equal(out["row_token"].cpu().numpy(), ref["row_token"])
        np.testing.assert_array_equal(out["slot_row"].cpu().numpy(), ref["slot_row"])
        if ep > 1:
            np.testing.assert_array_equal(out["slot_send_row"].cpu().numpy(), ref["slot_send_row"])
        assert moe.get_device_status(ws) == moe.MOE_OK


def test_layout_zero_tokens():
    shape = moe.Shape(T=0, d=64, E=16, k=2, f=64, ep=4)
    ws = moe.workspace(shape)
    out = moe.dispatch_layout(shape, torch.empty(0, 2, dtype=torch.int32, device="cuda"), ws)
    assert out["expert_offsets"].cpu().tolist() == [0] * 17
    assert out["rank_offsets"].cpu().tolist() == [0] * 5
    assert moe.stats_dict(out["stats"])["rows_sent"] == 0


def test_layout_bad_expert_index_reported():
    shape = moe.Shape(T=100, d=64, E=16, k=2, f=64, ep=4)
    ws = moe.workspace(shape)
    idx = W.uniform_routing(100, 16, 2, seed=4)
    idx[37, 1] = 16
    moe.dispatch_layout(shape, idx.cuda(), ws)
    assert moe.get_device_status(ws) == moe.MOE_ERR_DEVICE_INDEX
    # the status was reset and the workspace still works
    idx[37, 1] = 3
    out = moe.dispatch_layout(shape, idx.cuda(), ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    ref = oracle.dispatch_layout(idx.numpy(), 16, 4)
    np.testing.assert_array_equal(out["row_token"].cpu().numpy(), ref["row_token"])


def test_lookback_wait_is_bounded():
    """A block that never publishes makes its successors' waits run out
    (50 ms limit here): the call reports MOE_ERR_DEVICE_TIMEOUT and the next
    call on the same workspace is exact again."""
    T, E, k = 4096, 64, 4   # 8 lookback blocks
    shape = moe.Shape(T=T, d=64, E=E, k=k, f=64, ep=8)
    ws = moe.workspace(shape)
    idx = W.uniform_routing(T, E, k, seed=12).cuda()
    moe.debug_dispatch_layout_stall(shape, idx, ws, stall_block=3, wait_limit_ns=50_000_000)
    assert moe.get_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    out = moe.dispatch_layout(shape, idx, ws)
    assert moe.get_device_status(ws) == moe.MOE_OK
    ref = oracle.dispatch_layout(idx.cpu().numpy(), E, 8)
    np.testing.assert_array_equal(out["slot_send_row"].cpu().numpy(), ref["slot_send_row"])


def test_forward_and_standalone_layout_share_a_workspace():
    """The forward's fused router writes per-tile histograms; a standalone
    layout on the same workspace afterwards (and a forward after that) must
    still find its lookback words zeroed."""
    from util import Case
    c = Case(2, T=3000)
    shape = c.shape_ep(8)
    ws = moe.workspace(shape, forward=True)
    buf = moe.ForwardBuffers(shape)
    y0 = moe.forward(shape, c.dx, c.packed, None, ws, buffers=buf)
    idx = W.uniform_routing(3000, 64, 4, seed=21)
    out = moe.dispatch_layout(shape, idx.cuda(), ws)
    ref = oracle.dispatch_layout(idx.numpy(), 64, 8)
    np.testing.assert_array_equal(out["slot_send_row"].cpu().numpy(), ref["slot_send_row"])
    np.testing.assert_array_equal(out["row_token"].cpu().numpy(), ref["row_token"])
    y1 = moe.forward(shape, c.dx, c.packed, None, ws)
    assert torch.equal(y0, y1)
    assert moe.get_device_status(ws) == moe.MOE_OK
