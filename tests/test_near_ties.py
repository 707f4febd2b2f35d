"""The top-6 workload's near-tie injection (tests/util.py) does what the
parity tests rely on: a seeded 5% of the tokens end with the gap between
their k-th and (k+1)-th router logits below 1e-5 of the token's logit
spread, measured by the oracle in double, and no other token changes.
No GPU."""
import types

import numpy as np

import oracle
from routing_dispatch_experts_b200 import workloads as W

from util import NEAR_TIE, inject_near_ties


def test_injected_tokens_are_near_ties_and_the_rest_untouched():
    w = W.WORKLOADS[4]
    T = 600
    x0 = W.make_x(w, 0, T)
    case = types.SimpleNamespace(w=w, T=T, x=x0.clone(), wr=W.make_router(w), bias=None)
    toks = inject_near_ties(case, seed=0)
    assert len(toks) == round(w.near_tie_frac * T)
    assert len(np.unique(toks)) == len(toks)
    m = oracle.margin(oracle.router_logits(case.x, case.wr), w.k)
    assert (m[toks] < NEAR_TIE).all(), m[toks].max()
    others = np.setdiff1d(np.arange(T), toks)
    assert (case.x[others] == x0[others]).all()
    # the untouched tokens are not near-ties by construction (a random
    # Gaussian workload has few): the injection is what makes them
    m0 = oracle.margin(oracle.router_logits(x0, case.wr), w.k)
    assert (m0[toks] < NEAR_TIE).mean() < 0.2


def test_tokens_that_miss_the_margin_are_replaced_and_left_untouched():
    """With a budget of 8 one-ulp steps most picked tokens miss the margin:
    each is dropped, keeps its x, and another token takes its place, so
    every returned token is a near-tie."""
    w = W.WORKLOADS[4]
    T = 400
    x0 = W.make_x(w, 0, T)
    case = types.SimpleNamespace(w=w, T=T, x=x0.clone(), wr=W.make_router(w), bias=None)
    toks = inject_near_ties(case, seed=0, frac=0.1, max_steps=8)
    first = W.sample_tokens(T, 40, 0 + 101).numpy()
    m = oracle.margin(oracle.router_logits(case.x, case.wr), w.k)
    assert len(toks) == 40
    assert (m[toks] < NEAR_TIE).all()
    missed = np.setdiff1d(first, toks)
    assert len(missed) > 0, "the projection alone reached every picked token"
    changed = np.where((case.x != x0).any(1).numpy())[0]
    assert set(changed.tolist()) <= set(toks.tolist())
    assert not set(missed.tolist()) & set(changed.tolist())
