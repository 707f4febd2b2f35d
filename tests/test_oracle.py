"""Pins of the CPU oracle against what the pages and the mathematics fix.

No GPU.  Each test checks the oracle against something other than itself:
brute force on tiny inputs, an independent library routine (numpy / torch
float64), a closed form, an identity the pages' Table I obeys, or a value
worked out by hand.  Each is chosen so that a plausible slip in the oracle
(a dropped term, a wrong sign or index, a swapped operand, an unstable sort)
fails it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from routing_dispatch_experts_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ top-k
def _brute_topk(l, k):
    """Count-of-beaters rule: expert e is chosen iff fewer than k experts beat
    it under (logit desc, index asc); its slot is that count."""
    E = len(l)
    idx = [None] * k
    for e in range(E):
        beaters = sum(1 for q in range(E) if l[q] > l[e] or (l[q] == l[e] and q < e))
        if beaters < k:
            idx[beaters] = e
    return idx


@pytest.mark.parametrize("E", [4, 8, 16, 33])
def test_topk_matches_brute_force_with_ties(oracle_mod, E):
    rng = np.random.default_rng(E)
    # values from a tiny set force many exact ties; include -0.0 and +0.0
    vals = np.array([-1.5, -0.0, 0.0, 0.25, 0.25, 2.0, 7.0])
    for trial in range(40):
        T = 8
        l = rng.choice(vals, size=(T, E))
        for k in sorted({1, 2, min(4, E), E - 1, E}):
            idx, gate = oracle_mod.topk(l, k)
            for t in range(T):
                assert list(idx[t]) == _brute_topk(list(l[t]), k)


def test_topk_exact_ties_take_lowest_index(oracle_mod):
    l = np.zeros((3, 8))
    l[1, [2, 5, 6]] = 1.0
    l[2] = [-0.0, 0.0, -0.0, 0.0, 1, 1, -1, -1]
    idx, _ = oracle_mod.topk(l, 3)
    assert idx[0].tolist() == [0, 1, 2]
    assert idx[1].tolist() == [2, 5, 6]
    assert idx[2].tolist() == [4, 5, 0]  # -0.0 ties +0.0 -> lowest index


def test_gates_equal_full_softmax_renormalised(oracle_mod):
    rng = np.random.default_rng(1)
    l = rng.normal(size=(64, 16)) * 3
    for k in (1, 2, 4, 16):
        idx, gate = oracle_mod.topk(l, k)
        # independent formula: softmax over all E, pick the k, renormalise
        p = np.exp(l - l.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        pk = np.take_along_axis(p, idx.astype(np.int64), axis=1)
        ref = pk / pk.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(gate, ref, rtol=1e-13, atol=0)
        np.testing.assert_allclose(gate.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        assert np.all(np.diff(gate, axis=1) <= 0)
        # k distinct indices in range
        assert all(len(set(r)) == k for r in idx.tolist())
        assert idx.min() >= 0 and idx.max() < 16


def test_margin_hand_examples(oracle_mod):
    l = np.array([[3.0, 1.0, 2.0, 0.0]])
    assert oracle_mod.margin(l, 1)[0] == pytest.approx(1 / 3)
    assert oracle_mod.margin(l, 2)[0] == pytest.approx(1 / 3)
    assert oracle_mod.margin(l, 3)[0] == pytest.approx(1 / 3)
    l2 = np.array([[5.0, 1.0, 4.0, 0.0, 4.5]])
    assert oracle_mod.margin(l2, 1)[0] == pytest.approx(0.5 / 5)
    assert oracle_mod.margin(l2, 2)[0] == pytest.approx(0.5 / 5)
    assert oracle_mod.margin(l2, 3)[0] == pytest.approx(3.0 / 5)
    # exact tie at the boundary -> 0; k == E -> no unchosen expert
    assert oracle_mod.margin(np.array([[1.0, 1.0, 0.0]]), 1)[0] == 0.0
    assert math.isinf(oracle_mod.margin(np.array([[1.0, 2.0]]), 2)[0])


# ---------------------------------------------------------------- router
@pytest.mark.parametrize("cfg", [1, 2, 5])
def test_router_logits_match_float64_matmul(oracle_mod, cfg):
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, 0, T=37)
    wr = W.make_router(w)
    b = W.make_bias(w)
    l = oracle_mod.router_logits(x, wr, b)
    ref = x.double() @ wr.double()
    if b is not None:
        ref += b.double()
    np.testing.assert_allclose(l, ref.numpy(), rtol=1e-12, atol=1e-12)
    tok = np.array([36, 0, 5])
    np.testing.assert_array_equal(oracle_mod.router_logits(x, wr, b, tokens=tok), l[tok])


# -------------------------------------------------------- dispatch layout
def _brute_layout(idx, E, ep, rmap):
    T, k = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")  # rows: by expert, then flat index
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    slot_row = np.empty_like(order)
    slot_row[order] = np.arange(order.size)
    pairs = sorted({(rmap[e], t) for t in range(T) for e in idx[t]})
    send_row = {p: i for i, p in enumerate(pairs)}
    slot_send = np.array([send_row[(rmap[flat[a]], a // k)] for a in range(flat.size)])
    rank_counts = np.bincount([p[0] for p in pairs], minlength=ep)
    return dict(expert_counts=counts, expert_offsets=offsets, row_token=order // k,
                slot_row=slot_row, send_token=np.array([p[1] for p in pairs]),
                slot_send_row=slot_send, rank_counts=rank_counts,
                rank_offsets=np.concatenate([[0], np.cumsum(rank_counts)]),
                rows_sent=len(pairs))


@pytest.mark.parametrize("T,E,k,ep,placement", [
    (1, 4, 1, 2, "contiguous"), (7, 8, 3, 4, "contiguous"), (8, 16, 4, 4, "permutation"),
    (53, 16, 4, 8, "permutation"), (200, 64, 6, 32, "permutation"), (129, 64, 2, 16, "contiguous"),
    (100, 12, 5, 3, "contiguous"), (64, 8, 8, 8, "contiguous"),
])
def test_layout_matches_stable_sort_brute_force(oracle_mod, T, E, k, ep, placement):
    idx = W.uniform_routing(T, E, k, seed=T * 31 + E).numpy()
    rmap = (W.contiguous_placement(E, ep) if placement == "contiguous"
            else W.permutation_placement(E, ep, seed=5))
    got = oracle_mod.dispatch_layout(idx, E, ep, rmap)
    ref = _brute_layout(idx, E, ep, rmap)
    for key in ("expert_counts", "expert_offsets", "row_token", "slot_row", "send_token",
                "slot_send_row", "rank_counts", "rank_offsets"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=key)
    st = got["stats"]
    assert st["rows_sent"] == ref["rows_sent"]
    assert st["dup_removed"] == T * k - ref["rows_sent"]
    # row_token / slot_row are inverse bijections
    assert sorted(got["slot_row"].tolist()) == list(range(T * k))
    assert np.all(got["row_token"][got["slot_row"]] == np.arange(T * k) // k)
    assert got["expert_counts"].sum() == T * k and got["expert_offsets"][-1] == T * k


def test_layout_ep1_has_no_dispatch(oracle_mod):
    idx = W.uniform_routing(50, 16, 4).numpy()
    st = oracle_mod.dispatch_layout(idx, 16, 1)["stats"]
    assert st["rows_sent"] == 0 and st["dup_removed"] == 0
    assert st["tokens_single_rank"] == 50 and st["home_rank_rows"] == 200


def test_dedup_special_cases(oracle_mod):
    T, E, k = 300, 16, 4
    idx = W.uniform_routing(T, E, k, seed=3).numpy()
    # one expert per rank: the k distinct experts hit k distinct ranks
    st = oracle_mod.dispatch_layout(idx, E, E)["stats"]
    assert st["dup_removed"] == 0 and st["rows_sent"] == T * k
    # all experts of every token on one rank: T*k - T rows removed
    idx2 = np.stack([np.arange(k) + 4 * (t % 4) for t in range(T)]).astype(np.int32)
    st2 = oracle_mod.dispatch_layout(idx2, E, 4)["stats"]
    assert st2["dup_removed"] == T * k - T and st2["tokens_single_rank"] == T


def test_layout_rejects_bad_index(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.dispatch_layout(np.array([[0, 16]], np.int32), 16, 1)


def test_table1_identities_hold_on_the_page_and_in_the_oracle(oracle_mod):
    """Table I of Expert Coupling (top-2): with k=2 a token reaches 1 or 2
    GPUs, so Same-GPU = 2 - GPUs and Dedup = 1 - GPUs/k.  The printed rows obey
    both (up to the page's rounding), and so must the oracle's statistics."""
    tab = json.load(open(os.path.join(GOLDEN, "expert_coupling_table1.json")))
    k = tab["k"]
    for ep, plc, same, gpus, dedup, moved, stays in tab["rows"]:
        assert abs(dedup - 100 * (1 - gpus / k)) <= 0.5 + 100 * 0.005 / k
        assert abs(same - 100 * (2 - gpus)) <= 1.0
        # a token that stays home sees its next-layer experts there at 1/EP
        assert abs(stays - 100 / ep) <= 0.5
    for ep in (8, 16):
        for seed in range(3):
            idx = W.uniform_routing(4000, 64, 2, seed=seed).numpy()
            st = oracle_mod.dispatch_layout(idx, 64, ep)["stats"]
            T = 4000
            gp = st["rows_sent"] / T
            assert st["tokens_single_rank"] / T == pytest.approx(2 - gp, abs=1e-12)
            assert st["dup_removed"] / (T * k) == pytest.approx(1 - gp / k, abs=1e-12)


def _expected_ranks(E, k, P):
    per = E // P
    return P * (1 - math.comb(E - per, k) / math.comb(E, k))


@pytest.mark.parametrize("E,k,P", [(64, 2, 8), (64, 2, 16), (64, 4, 8), (64, 6, 32), (128, 8, 16)])
def test_distinct_ranks_closed_form_uniform_routing(oracle_mod, E, k, P):
    """E|R(t)| = P (1 - C(E-E/P, k) / C(E, k)) for k distinct uniform experts
    and contiguous placement; the home-rank share of assignments is 1/P."""
    T = 20000
    idx = W.uniform_routing(T, E, k, seed=E + k + P).numpy()
    st = oracle_mod.dispatch_layout(idx, E, P)["stats"]
    mean = st["rows_sent"] / T
    # per-token |R(t)| lies in [1, k]: std <= (k-1)/2
    bound = 6 * ((k - 1) / 2) / math.sqrt(T)
    assert abs(mean - _expected_ranks(E, k, P)) <= bound
    home = st["home_rank_rows"] / (T * k)
    assert abs(home - 1 / P) <= 6 * math.sqrt((1 / P) / (T * k)) * math.sqrt(k)
    # the closed form reproduces Table I's contiguous rows to their rounding
    if (E, k) == (64, 2):
        assert round(_expected_ranks(64, 2, P), 2) == {8: 1.89, 16: 1.95}[P]


# ----------------------------------------------------------------- experts
def test_swiglu_single_weight_hand_value(oracle_mod):
    d, f = 2, 1
    wg = torch.zeros(1, d, f); wg[0, 0, 0] = 2.0
    wu = torch.zeros(1, d, f); wu[0, 0, 0] = 3.0
    wd = torch.zeros(1, f, d); wd[0, 0, 0] = 5.0
    x = torch.tensor([[1.0, -7.0]])
    y = oracle_mod.moe_output(x, np.zeros((1, 1), np.int32), np.ones((1, 1)), wg, wu, wd)
    sig2 = 1.0 / (1.0 + math.exp(-2.0))
    assert y[0, 0] == pytest.approx(5 * 3 * 2 * sig2, rel=1e-15)
    assert y[0, 1] == 0.0


def test_zero_gate_weights_give_zero_output(oracle_mod):
    w = W.WORKLOADS[1]
    x = W.make_x(w, T=9)
    wg, wu, wd = W.make_experts(w, experts=[0, 1, 2])
    wg.zero_()
    idx = np.array([[0, 1, 2]] * 9, np.int32)
    y = oracle_mod.moe_output(x, idx, np.full((9, 3), 1 / 3), wg, wu, wd)
    assert np.all(y == 0.0)


@pytest.mark.parametrize("cfg", [1, 2])
def test_single_expert_top1_is_dense_swiglu(oracle_mod, cfg):
    """E = 1, k = 1 reduces the layer to one dense SwiGLU FFN."""
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, T=23)
    wg, wu, wd = W.make_experts(w, experts=[3])
    idx = np.zeros((23, 1), np.int32)
    y = oracle_mod.moe_output(x, idx, np.ones((23, 1)), wg, wu, wd)
    xd = x.double()
    ref = (torch.nn.functional.silu(xd @ wg[0].double()) * (xd @ wu[0].double())) @ wd[0].double()
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_grouped_swiglu_rows_match_per_expert_torch(oracle_mod):
    w = W.WORKLOADS[2]
    x = W.make_x(w, T=40)
    wg, wu, wd = W.make_experts(w, experts=range(5))
    off = np.array([0, 7, 7, 20, 33, 40], np.int32)  # expert 1 is empty
    y = oracle_mod.grouped_swiglu(x, off, wg, wu, wd)
    for e in range(5):
        xs = x[off[e]:off[e + 1]].double()
        ref = (torch.nn.functional.silu(xs @ wg[e].double()) * (xs @ wu[e].double())) @ wd[e].double()
        np.testing.assert_allclose(y[off[e]:off[e + 1]], ref.numpy(), rtol=1e-10, atol=1e-12)
    rows = np.array([39, 0, 20])
    np.testing.assert_array_equal(oracle_mod.grouped_swiglu(x, off, wg, wu, wd, rows=rows), y[rows])


# ----------------------------------------------------------------- combine
@pytest.mark.parametrize("cfg", [1, 2])
def test_identity_experts_unit_gates_give_k_times_x(oracle_mod, cfg):
    """Permute then combine with the experts replaced by the identity and
    unit gates reproduces k * x exactly (k*x is exact for k <= 8)."""
    w = W.WORKLOADS[cfg]
    T = 77
    x = W.make_x(w, T=T)
    idx = W.uniform_routing(T, w.E, w.k, seed=2).numpy()
    lay = oracle_mod.dispatch_layout(idx, w.E, 1)
    x_perm = x[torch.from_numpy(lay["row_token"]).long()]
    y = oracle_mod.combine(x_perm, lay["slot_row"], None, k=w.k)
    np.testing.assert_array_equal(y, w.k * x.double().numpy())


def test_combine_weights_each_slot_by_its_own_gate_by_hand(oracle_mod):
    """Non-unit gates worked by hand: two tokens, k = 2, slot rows out of
    order.  y[0] = 0.25 * row 2 + 0.75 * row 0 = [1.75, 0];
    y[1] = 0.5 * row 3 + 0.125 * row 1 = [0, 4.125]."""
    y_perm = np.array([[1.0, 0.0], [0.0, 1.0], [4.0, 0.0], [0.0, 8.0]])
    slot_row = np.array([2, 0, 3, 1], np.int32)
    gate = np.array([[0.25, 0.75], [0.5, 0.125]])
    y = oracle_mod.combine(y_perm, slot_row, gate)
    np.testing.assert_array_equal(y, [[1.75, 0.0], [0.0, 4.125]])


def test_layer_output_weights_experts_by_gates_by_hand(oracle_mod):
    """moe_output with non-unit gates on experts whose outputs are known
    exactly: d = f = 1, W_g = 64 for every expert, so for x in {1, 2} the
    gate projection is 64x and silu(64x) = 64x in double (exp(-64) is below
    half an ulp of 1).  Expert e then gives 64x * (b_e x) * c_e:
    e0 (b=1, c=1), e1 (b=2, c=2), e2 (b=0.5, c=-1).
    Token 0 (x=1), experts (1, 0), gates (0.75, 0.25): 0.75*256 + 0.25*64 = 208.
    Token 1 (x=2), experts (2, 1), gates (0.625, 0.375):
    0.625*(-128) + 0.375*1024 = 304."""
    x = torch.tensor([[1.0], [2.0]])
    wg = torch.full((3, 1, 1), 64.0)
    wu = torch.tensor([1.0, 2.0, 0.5]).reshape(3, 1, 1)
    wd = torch.tensor([1.0, 2.0, -1.0]).reshape(3, 1, 1)
    idx = np.array([[1, 0], [2, 1]], np.int32)
    gate = np.array([[0.75, 0.25], [0.625, 0.375]])
    y = oracle_mod.moe_output(x, idx, gate, wg, wu, wd)
    np.testing.assert_array_equal(y, [[208.0], [304.0]])
    # and the same through the permuted path (layout, grouped experts, combine)
    lay = oracle_mod.dispatch_layout(idx, 3, 1)
    x_perm = x[torch.from_numpy(lay["row_token"]).long()]
    y_perm = oracle_mod.grouped_swiglu(x_perm, lay["expert_offsets"], wg, wu, wd)
    np.testing.assert_array_equal(oracle_mod.combine(y_perm, lay["slot_row"], gate),
                                  [[208.0], [304.0]])


def test_permuted_pipeline_equals_per_token_definition(oracle_mod):
    """layout -> permute -> grouped experts -> combine equals the per-token
    sum of gated expert outputs (same double arithmetic, bit-identical)."""
    w = W.WORKLOADS[2]
    T = 50
    x, wr, b, wg, wu, wd = W.make_all(w, T=T)
    ref = oracle_mod.forward(x, wr, b, wg, wu, wd, w.k)
    lay = oracle_mod.dispatch_layout(ref["idx"], w.E, 8)
    x_perm = x[torch.from_numpy(lay["row_token"]).long()]
    y_perm = oracle_mod.grouped_swiglu(x_perm, lay["expert_offsets"], wg, wu, wd)
    y = oracle_mod.combine(y_perm, lay["slot_row"], ref["gate"])
    np.testing.assert_array_equal(y, ref["y"])


# ------------------------------------------------------ near-ties / nudges
def test_perturbation_flips_only_near_ties(oracle_mod):
    """A perturbation of at most eps per logit can change a routing decision
    only if the token's margin times its spread is below 2*eps ('MoE
    Pretraining: Parallelism Layout ...', Finding 3: the flipped decisions
    are the near-ties).  Planted exact ties, with the perturbation favouring
    the higher index, must flip."""
    rng = np.random.default_rng(11)
    T, E, k, eps = 4000, 16, 4, 1e-6
    l0 = rng.normal(size=(T, E))
    planted = np.arange(0, T, 97)
    for t in planted:
        o = np.argsort(-l0[t], kind="stable")
        lo, hi = sorted((o[k - 1], o[k]))
        l0[t, hi] = l0[t, lo]          # exact tie: lower index is chosen
    delta = rng.uniform(-eps, eps, size=(T, E))
    for t in planted:
        o = np.argsort(-l0[t], kind="stable")
        lo, hi = sorted((o[k - 1], o[k]))
        delta[t, hi], delta[t, lo] = eps, -eps
    l1 = l0 + delta
    i0, _ = oracle_mod.topk(l0, k)
    i1, _ = oracle_mod.topk(l1, k)
    m = oracle_mod.margin(l0, k)
    spread = l0.max(1) - l0.min(1)
    flipped = set(np.where((np.sort(i0, 1) != np.sort(i1, 1)).any(1))[0].tolist())
    assert set(planted.tolist()) <= flipped
    for t in flipped:
        assert m[t] * spread[t] <= 2 * eps


def test_one_ulp_router_nudge_changes_logits_by_at_most_x_ulp(oracle_mod):
    """The 1-ULP nudge of a single router weight moves logit e of token t by
    exactly x[t,i] * (nudged - original) in the oracle's double arithmetic."""
    w = W.WORKLOADS[1]
    x = W.make_x(w, T=256)
    wr = W.make_router(w)
    i, e = 17, 3
    wr2 = wr.clone()
    wr2[i, e] = torch.nextafter(wr[i, e], torch.tensor(1.0))
    ulp = float(wr2[i, e]) - float(wr[i, e])
    d = oracle_mod.router_logits(x, wr2) - oracle_mod.router_logits(x, wr)
    others = np.delete(d, e, axis=1)
    assert np.all(others == 0.0)
    np.testing.assert_allclose(d[:, e], x[:, i].double().numpy() * ulp, rtol=1e-6, atol=1e-15)


# ------------------------------------------------------ correlated placement
def test_correlated_placement_groups_planted_pairs(oracle_mod):
    E, ep, T = 16, 4, 400
    # tokens pick planted pairs (0,9), (1,10), ... -> each pair must share a rank
    pairs = [(e, (e + 9) % E) for e in range(0, E, 2)]
    idx = np.array([pairs[t % len(pairs)] for t in range(T)], np.int32)
    m = oracle_mod.fit_correlated_placement(idx, E, ep)
    assert sorted(m.count(r) for r in range(ep)) == [E // ep] * ep
    for a, b in pairs:
        assert m[a] == m[b]
    # and the dedup rows drop accordingly: each token reaches one rank
    st = oracle_mod.dispatch_layout(idx, E, ep, m)["stats"]
    assert st["tokens_single_rank"] == T and st["dup_removed"] == T
