"""Pins of the oracle's routing variants and router statistics (the CUDA
path does not implement these yet).  Each test checks a property the
definition implies, brute force, or a hand-worked case.  No GPU."""
import numpy as np
import pytest

import oracle


# ------------------------------------------------------------ near-tie share
def test_near_tie_share_counts_planted_ties():
    rng = np.random.default_rng(0)
    T, E, k = 200, 8, 2
    l = rng.normal(size=(T, E)).round(1) * 4          # distinct values at a coarse grid
    l += np.arange(E)[None, :] * 1e-3                  # no accidental exact ties
    planted = rng.choice(T, 37, replace=False)
    for t in planted:                                  # k-th and (k+1)-th equal
        o = np.argsort(-l[t], kind="stable")
        l[t, o[k]] = l[t, o[k - 1]]
    assert oracle.near_tie_share(l, k) == pytest.approx(37 / T)
    # the margin is a ratio of differences: invariant to scaling and shifting
    assert oracle.near_tie_share(3.0 * l - 7.0, k) == pytest.approx(37 / T)
    # k = E has no (k+1)-th score: never a tie
    assert oracle.near_tie_share(l, E) == 0.0


# ---------------------------------------------------------- routing changes
def test_routing_changes_cases():
    a = np.array([[0, 1, 2], [3, 4, 5], [6, 7, 0]])
    assert oracle.routing_changes(a, a) == dict(tokens=0, experts=0, slots=0)
    b = a[:, ::-1].copy()                              # same sets, other slot order
    assert oracle.routing_changes(a, b) == dict(tokens=0, experts=0, slots=6)
    c = a.copy()
    c[1, 2] = 9                                        # one expert swapped in one token
    assert oracle.routing_changes(a, c) == dict(tokens=1, experts=1, slots=1)
    d = a + 10                                         # every expert different
    assert oracle.routing_changes(a, d) == dict(tokens=3, experts=9, slots=9)
    for x, y in ((a, c), (a, d), (b, c)):
        assert oracle.routing_changes(x, y) == oracle.routing_changes(y, x)


# ----------------------------------------------------- selection-only bias
def _dyadic(rng, shape, scale=8):
    """Values on a grid of 1/64: sums of two of them are exact in float32."""
    return rng.integers(-scale * 64, scale * 64, size=shape) / 64.0


def test_selection_bias_zero_is_plain_topk():
    rng = np.random.default_rng(1)
    l = _dyadic(rng, (300, 16))
    i0, g0 = oracle.topk(l, 4)
    i1, g1 = oracle.topk_selection_bias(l, np.zeros(16), 4)
    assert (i0 == i1).all()
    np.testing.assert_allclose(g1, g0, rtol=0, atol=1e-15)


@pytest.mark.parametrize("E,k", [(5, 2), (6, 3), (8, 4)])
def test_selection_bias_brute_force(E, k):
    """Chosen set = the k-subset of the largest keys logit+bias (ties: lower
    index); slots in key order; gates = exp(l) normalised over the set."""
    rng = np.random.default_rng(E * 10 + k)
    l = _dyadic(rng, (60, E), scale=2)                 # coarse: many exact key ties
    b = _dyadic(rng, (E,), scale=2)
    idx, gate = oracle.topk_selection_bias(l, b, k)
    for t in range(len(l)):
        key = (l[t].astype(np.float32) + b.astype(np.float32)).astype(np.float64)
        order = sorted(range(E), key=lambda e: (-key[e], e))
        assert list(idx[t]) == order[:k]
        s = np.array(order[:k])
        ex = np.exp(l[t, s])
        np.testing.assert_allclose(gate[t], ex / ex.sum(), rtol=1e-13, atol=0)
        # every chosen key beats or ties (with a lower index) every unchosen one
        for e in set(range(E)) - set(s.tolist()):
            assert all(key[c] > key[e] or (key[c] == key[e] and c < e) for c in s)


def test_selection_bias_steers_choice_not_weights():
    rng = np.random.default_rng(2)
    l = _dyadic(rng, (400, 16))
    b = _dyadic(rng, (16,), scale=1)
    i1, g1 = oracle.topk_selection_bias(l, b, 4)
    # a constant added to every bias keeps every choice, and gates ignore the bias
    i2, g2 = oracle.topk_selection_bias(l, b + 4.0, 4)
    assert (i1 == i2).all() and (g1 == g2).all()
    # the gates equal plain top-k's gates of the same chosen set
    ref = np.exp(np.take_along_axis(l, i1.astype(np.int64), 1))
    np.testing.assert_allclose(g1, ref / ref.sum(1, keepdims=True), rtol=1e-13)
    # a large bias forces an expert into every token's choice, first slot
    big = np.zeros(16)
    big[11] = 1e6
    i3, g3 = oracle.topk_selection_bias(l, big, 4)
    assert (i3[:, 0] == 11).all()
    np.testing.assert_allclose(g3.sum(1), 1.0, rtol=1e-13)


# --------------------------------------------------------- expert capacity
def test_capacity_formula_cases():
    assert oracle.expert_capacity(16384, 2, 64, 2.0) == 1024   # twice the mean load 512
    assert oracle.expert_capacity(10, 3, 4, 1.0) == 8           # ceil(7.5)
    assert oracle.expert_capacity(0, 2, 8, 2.0) == 0


def test_capacity_first_choices_before_second_choices():
    # expert 0 is the first choice of tokens 2, 3 and the second of 0, 1;
    # expert 1 the reverse; capacity ceil(0.5 * 4 * 2 / 2) = 2 each
    idx = np.array([[1, 0], [1, 0], [0, 1], [0, 1]])
    keep = oracle.capacity_keep(idx, 2, 0.5)
    assert keep.tolist() == [[True, False]] * 4
    # within one choice rank, earlier tokens first
    idx2 = np.array([[0, 1], [0, 2], [0, 3]])
    keep2 = oracle.capacity_keep(idx2, 4, 0.5)                   # capacity ceil(0.5*6/4) = 1
    assert keep2[:, 0].tolist() == [True, False, False]
    assert keep2[:, 1].all()


@pytest.mark.parametrize("cf", [0.25, 0.5, 1.0, 1.25, 2.0])
def test_capacity_invariants(cf):
    rng = np.random.default_rng(int(cf * 100))
    T, E, k = 500, 16, 4
    # skewed loads: a few experts are popular
    p = np.arange(1, E + 1, dtype=float) ** -1.2
    idx = np.stack([rng.choice(E, k, replace=False, p=p / p.sum()) for _ in range(T)])
    keep = oracle.capacity_keep(idx, E, cf)
    cap = oracle.expert_capacity(T, k, E, cf)
    load = np.bincount(idx.ravel(), minlength=E)
    kept = np.bincount(idx[keep], minlength=E)
    # each expert keeps exactly min(load, capacity) rows, whatever the order
    assert (kept == np.minimum(load, cap)).all()
    # more capacity never drops an assignment that less capacity kept
    assert (oracle.capacity_keep(idx, E, cf * 2) >= keep).all()
    # with room for every row nothing is dropped
    assert oracle.capacity_keep(idx, E, E / k + 1).all()
