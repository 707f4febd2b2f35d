"""The Python binding rejects arguments of the wrong dtype, size or shape
before anything reaches the library, naming the argument: every array a
kernel indexes by the shape (index arrays, gates, offsets, the packed
weights, a caller's output or buffers) is checked.  No GPU: the checks run
on CPU tensors, ahead of the CUDA-tensor check, which would raise too
(hence each test matches the argument's name in the message)."""
import pytest
import torch

import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import build

S = moe.Shape(T=8, d=64, E=4, k=2, f=64)
R = S.R
i32 = dict(dtype=torch.int32)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def _x():
    return torch.zeros(S.T, S.d, dtype=S.dtype)


def _packed(short=0):
    return torch.zeros(moe.packed_weights_size(S) - short, dtype=torch.uint8)


def _ws():
    return torch.zeros(16, dtype=torch.uint8)


@pytest.mark.parametrize("bad", [torch.zeros(R, dtype=torch.int64), torch.zeros(R - 1, **i32)])
def test_permute_row_token(bad):
    with pytest.raises(ValueError, match="^row_token:"):
        moe.permute(S, _x(), bad)


def test_permute_by_token_slot_row():
    with pytest.raises(ValueError, match="^slot_row:"):
        moe.permute_by_token(S, _x(), torch.zeros(R + 1, **i32))


def test_combine_slot_row_and_gates():
    y_perm = torch.zeros(R, S.d, dtype=S.dtype)
    with pytest.raises(ValueError, match="^slot_row:"):
        moe.combine(S, y_perm, torch.zeros(S.T, **i32))
    with pytest.raises(ValueError, match="^topk_gate:"):
        moe.combine(S, y_perm, torch.zeros(R, **i32), torch.zeros(S.T, S.k, dtype=torch.float64))
    with pytest.raises(ValueError, match="^topk_gate:"):
        moe.combine(S, y_perm, torch.zeros(R, **i32), torch.zeros(S.T, dtype=torch.float32))


def test_grouped_offsets_and_packed():
    x_perm = torch.zeros(R, S.d, dtype=S.dtype)
    with pytest.raises(ValueError, match="^expert_offsets:"):
        moe.grouped_swiglu(S, x_perm, torch.zeros(S.E, **i32), _packed(), _ws())
    with pytest.raises(ValueError, match="^packed:"):
        moe.grouped_swiglu(S, x_perm, torch.zeros(S.E + 1, **i32), _packed(short=1), _ws())
    with pytest.raises(ValueError, match="^packed:"):
        moe.grouped_swiglu(S, x_perm, torch.zeros(S.E + 1, **i32),
                           torch.zeros(moe.packed_weights_size(S), dtype=torch.int8), _ws())


def test_grouped_gather_row_token():
    with pytest.raises(ValueError, match="^row_token:"):
        moe.grouped_swiglu_gather(S, _x(), torch.zeros(R, dtype=torch.int64),
                                  torch.zeros(S.E + 1, **i32), _packed(), _ws())


def test_route_packed_and_bias():
    with pytest.raises(ValueError, match="^packed:"):
        moe.route(S, _x(), None, None, _ws())
    with pytest.raises(ValueError, match="^bias:"):
        moe.route(S, _x(), _packed(), torch.zeros(S.E + 1), _ws())
    with pytest.raises(ValueError, match="^bias:"):
        moe.route(S, _x(), _packed(), torch.zeros(S.E, dtype=torch.float64), _ws())


def test_forward_output_bias_packed_and_buffers():
    x, p = _x(), _packed()
    with pytest.raises(ValueError, match="^y:"):
        moe.forward(S, x, p, None, _ws(), y=torch.zeros(S.T, S.d, dtype=torch.float32))
    with pytest.raises(ValueError, match="^y:"):
        moe.forward(S, x, p, None, _ws(), y=torch.zeros(S.T - 1, S.d, dtype=S.dtype))
    with pytest.raises(ValueError, match="^bias:"):
        moe.forward(S, x, p, torch.zeros(S.E - 1), _ws())
    with pytest.raises(ValueError, match="^packed:"):
        moe.forward(S, x, _packed(short=64), None, _ws())
    other = moe.ForwardBuffers(moe.Shape(T=16, d=64, E=4, k=2, f=64), device="cpu")
    with pytest.raises(ValueError, match="^buffers:"):
        moe.forward(S, x, p, None, _ws(), buffers=other)
    with pytest.raises(ValueError, match="^buffers:"):
        moe.forward_timed(S, x, p, None, _ws(), [], buffers=other)


def test_stall_probe_topk_idx():
    with pytest.raises(ValueError, match="^topk_idx:"):
        moe.debug_dispatch_layout_stall(S, torch.zeros(S.T, S.k + 1, **i32), _ws(), 0, 1000)


def test_matching_buffers_pass_the_checks():
    """Arguments of the right kinds get past the binding's checks (and stop
    at the CUDA-tensor check, since these are CPU tensors)."""
    buf = moe.ForwardBuffers(S, device="cpu")
    with pytest.raises(ValueError, match="CUDA"):
        moe.forward(S, _x(), _packed(), torch.zeros(S.E), _ws(),
                    y=torch.zeros(S.T, S.d, dtype=S.dtype), buffers=buf)
    with pytest.raises(ValueError, match="CUDA"):
        moe.combine(S, torch.zeros(R, S.d, dtype=S.dtype), torch.zeros(S.T, S.k, **i32),
                    torch.zeros(S.T, S.k))


def test_forward_routed_routing_arrays():
    x, p = _x(), _packed()
    with pytest.raises(ValueError, match="^topk_idx:"):
        moe.forward_routed(S, x, p, torch.zeros(S.T, S.k, dtype=torch.int64), None, _ws())
    with pytest.raises(ValueError, match="^topk_idx:"):
        moe.forward_routed(S, x, p, torch.zeros(R, **i32), None, _ws())
    with pytest.raises(ValueError, match="^topk_gate:"):
        moe.forward_routed(S, x, p, torch.zeros(S.T, S.k, **i32),
                           torch.zeros(S.T, S.k, dtype=torch.float64), _ws())
    with pytest.raises(ValueError, match="^packed:"):
        moe.forward_routed(S, x, _packed(short=1), torch.zeros(S.T, S.k, **i32), None, _ws())
    with pytest.raises(ValueError, match="CUDA"):
        moe.forward_routed(S, x, p, torch.zeros(S.T, S.k, **i32), torch.zeros(S.T, S.k), _ws())
