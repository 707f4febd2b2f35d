"""The seeded synthetic inputs follow the recipe they state, checked through
properties that the recipe implies rather than by re-drawing them: moments
(E|x|^2 = d(1 + sigma^2) for the cluster mixture, d for N(0, 1); the weight
scales), the cluster count (the share of token pairs that point the same
way), the Zipf bias (a distribution whose sorted ratios are rank^-s), the
placements (partitions with E/ep experts per rank), the uniform control
routing and the token samples.  No GPU."""
import math

import numpy as np
import pytest
import torch

from routing_dispatch_experts_b200 import workloads as W


def test_dtypes_and_shapes():
    for cfg, w in W.WORKLOADS.items():
        x = W.make_x(w, 0, 64)
        assert x.shape == (64, w.d) and x.dtype == w.torch_dtype
        assert W.make_router(w).shape == (w.d, w.E)
    assert W.WORKLOADS[1].torch_dtype == torch.float32
    assert all(W.WORKLOADS[c].torch_dtype == torch.bfloat16 for c in (2, 3, 4, 5))


def test_draws_are_reproducible_and_seed_dependent():
    w = W.WORKLOADS[2]
    assert torch.equal(W.make_x(w, 0, 500), W.make_x(w, 0, 500))
    assert not torch.equal(W.make_x(w, 0, 500), W.make_x(w, 1, 500))
    assert torch.equal(W.make_router(w, 3), W.make_router(w, 3))
    # each expert has its own sub-stream: a subset equals the same experts of the whole
    w1 = W.WORKLOADS[1]
    wg, wu, wd = W.make_experts(w1, 0)
    sg, su, sd = W.make_experts(w1, 0, experts=[3, 11])
    assert torch.equal(sg, wg[[3, 11]]) and torch.equal(su, wu[[3, 11]]) and torch.equal(sd, wd[[3, 11]])


@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_second_moment_of_x(cfg):
    """Centres N(0, I) plus sigma N(0, I) noise: E|x|^2 = d (1 + sigma^2);
    plain N(0, 1): E|x|^2 = d.  Mean over 4000 tokens within 3%."""
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, 0, 4000).double()
    want = w.d * (1 + w.sigma_within ** 2) if w.clusters else w.d
    got = float((x * x).sum(1).mean())
    # the mixture's centres are a finite sample: allow for their own spread
    assert abs(got / want - 1) < 0.03, (got, want)


@pytest.mark.parametrize("cfg", [2, 3])
def test_cluster_count_from_aligned_pairs(cfg):
    """Two tokens of one cluster have cosine ~ 1/(1 + sigma^2) = 0.8, two of
    different clusters ~ 0 (+- 1/sqrt(d)); so the share of pairs with cosine
    above 0.5 estimates 1/clusters."""
    w = W.WORKLOADS[cfg]
    x = W.make_x(w, 0, 1500).double()
    xn = x / x.norm(dim=1, keepdim=True)
    c = (xn @ xn.T).numpy()
    iu = np.triu_indices(len(c), 1)
    share = float((c[iu] > 0.5).mean())
    # uniform cluster choice: P(same) = 1/clusters, binomial-ish spread over ~1.1e6 pairs
    assert abs(share * w.clusters - 1) < 0.15, (share, 1 / w.clusters)


def test_weight_scales():
    w = W.WORKLOADS[1]   # fp32: no rounding in the way
    wr = W.make_router(w).double()
    assert abs(float(wr.std()) / 0.02 - 1) < 0.03
    wg, wu, wd = W.make_experts(w)
    for t in (wg, wu, wd):
        assert abs(float(t.double().std()) * math.sqrt(w.d) - 1) < 0.01
        assert abs(float(t.double().mean())) < 3e-3


def test_zipf_bias_is_a_log_distribution_with_power_law_ranks():
    w = W.WORKLOADS[5]
    b = W.make_bias(w).double()
    p = torch.exp(b)
    assert abs(float(p.sum()) - 1) < 1e-6
    ps = torch.sort(p, descending=True).values
    r = torch.arange(1, w.E + 1, dtype=torch.float64)
    # p_(r) / p_(1) = r^-s exactly up to the fp32 storage of the bias
    np.testing.assert_allclose((ps / ps[0]).numpy(), r.pow(-w.zipf).numpy(), rtol=1e-5)
    # which expert gets which rank is a seeded permutation, not the identity
    assert int(torch.argmax(b)) != 0 or int(torch.argmin(b)) != w.E - 1
    assert W.make_bias(W.WORKLOADS[2]) is None


@pytest.mark.parametrize("E,ep", [(16, 1), (64, 8), (64, 16), (64, 32), (128, 16), (256, 256)])
def test_placements_are_partitions(E, ep):
    for m in (W.contiguous_placement(E, ep), W.permutation_placement(E, ep, seed=4)):
        assert len(m) == E and min(m) >= 0 and max(m) < ep
        assert np.bincount(m, minlength=ep).tolist() == [E // ep] * ep
    c = W.contiguous_placement(E, ep)
    assert c == sorted(c)
    assert W.permutation_placement(E, ep, seed=4) == W.permutation_placement(E, ep, seed=4)


def test_permutation_placement_is_not_contiguous():
    assert W.permutation_placement(64, 32, seed=0) != W.contiguous_placement(64, 32)


@pytest.mark.parametrize("T,E,k", [(5000, 64, 2), (5000, 64, 6), (3000, 128, 8), (100, 16, 16)])
def test_uniform_routing(T, E, k):
    idx = W.uniform_routing(T, E, k, seed=9)
    assert idx.dtype == torch.int32 and idx.shape == (T, k)
    a = idx.numpy()
    assert a.min() >= 0 and a.max() < E
    assert all(len(set(row)) == k for row in a)
    # every expert equally likely: counts within 5 sigma of T*k/E
    n = np.bincount(a.ravel(), minlength=E)
    mean = T * k / E
    sd = math.sqrt(mean * (1 - 1 / E))
    assert np.abs(n - mean).max() <= 5 * sd + 1e-9


def test_sample_tokens():
    s = W.sample_tokens(1000, 64, seed=2).numpy()
    assert len(s) == 64 and (np.diff(s) > 0).all() and s.min() >= 0 and s.max() < 1000
    assert len(W.sample_tokens(10, 64)) == 10
    assert (W.sample_tokens(1000, 64, seed=2).numpy() == s).all()
