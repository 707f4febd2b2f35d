"""Seeded synthetic workloads for the MoE-layer forward.

This module only draws random numbers and lays them out in the shapes and
distributions of the five workloads below; it holds none of the layer's own
arithmetic (no router, no top-k, no dispatch, no expert math), so it can feed
both the CUDA path and the CPU oracle.

Every tensor is drawn on the CPU from ``torch.Generator`` streams seeded from
(workload seed, stream id), so the same values come out on every machine and
for any thread count; callers move them to the GPU afterwards.

Workloads (shapes follow the pages):

1. tiny      - T=2048 (4x512), d=256, E=16 SwiGLU experts f=256, top-4, fp32.
               The base MoE of "MoE Pretraining: Parallelism Layout Changes the
               Model, Not Quality", Methodology / Models and Data (16 SwiGLU
               experts of width 256, top-4 routing, fp32 on CPU).
2. fine      - T=16384 (32x512), d=256, E=64, f=64, top-4, bf16; x from a
               32-cluster Gaussian mixture; EP=8 contiguous placement.
               Fine-grained experts of the same page, Finding 4 (64 experts).
3. top2      - T=16384, d=2048, E=64, f=1024, top-2, bf16; 64-cluster mixture
               (sigma 0.5); EP 8 and 16, contiguous vs correlated placement.
               "Expert Coupling in MoE Pretraining", Abstract and Table I.
4. top6      - as 3 with top-6, EP=32, placement from a seeded permutation,
               5% of tokens with injected router near-ties (the injection
               needs router arithmetic and so lives with the tests).
5. large     - T=32768, d=4096, E=128, f=1536, top-8, bf16; x~N(0,1) and a
               Zipf(1.1) expert-popularity bias on the router logits; EP=16
               contiguous.  d=4096 is the model width of Expert Coupling,
               Table II.

Distributions common to all: W_router ~ N(0, 0.02^2) in the "ME" layout
[d, E]; W_gate, W_up ~ N(0, 1/d) in "EMH" [E, d, f]; W_down ~ N(0, 1/d) in
"EHM" [E, f, d] (layout names from "Revisiting MoE and Dense Speed-Accuracy
Comparisons", Table 1).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

# stream ids: each tensor family draws from its own generator
_STREAM = {
    "x": 1, "w_router": 2, "w_gate": 3, "w_up": 4, "w_down": 5,
    "centers": 6, "cluster_id": 7, "bias_perm": 8, "placement": 9,
    "calib": 10, "sample": 11, "near_tie_pick": 12,
}


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    T: int
    d: int
    E: int
    f: int
    k: int
    dtype: str            # "f32" or "bf16"
    clusters: int = 0     # 0 = x ~ N(0,1); else Gaussian mixture
    sigma_within: float = 0.5
    zipf: float = 0.0     # >0: Zipf exponent of the router-logit bias
    eps: tuple = (1,)     # simulated EP degrees exercised
    placements: tuple = ("contiguous",)
    near_tie_frac: float = 0.0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def R(self) -> int:
        return self.T * self.k

    def describe(self) -> str:
        return (f"T={self.T} d={self.d} E={self.E} f={self.f} top-{self.k} "
                f"{self.dtype} EP={'/'.join(map(str, self.eps))} "
                f"{'/'.join(self.placements)}")

    def scaled(self, T: int) -> "Workload":
        """Same workload with a different token count (small parity cases)."""
        return dataclasses.replace(self, T=T)


WORKLOADS = {
    1: Workload(1, "tiny", 2048, 256, 16, 256, 4, "f32", eps=(1,)),
    2: Workload(2, "fine", 16384, 256, 64, 64, 4, "bf16", clusters=32,
                eps=(8,), placements=("contiguous",)),
    3: Workload(3, "top2", 16384, 2048, 64, 1024, 2, "bf16", clusters=64,
                eps=(8, 16), placements=("contiguous", "correlated")),
    4: Workload(4, "top6", 16384, 2048, 64, 1024, 6, "bf16", clusters=64,
                eps=(32,), placements=("permutation",), near_tie_frac=0.05),
    5: Workload(5, "large", 32768, 4096, 128, 1536, 8, "bf16", zipf=1.1,
                eps=(16,), placements=("contiguous",)),
}


def _gen(seed: int, stream: str, sub: int = 0) -> torch.Generator:
    # SplitMix64-style mixing of (seed, stream, sub) into one 63-bit seed
    z = (seed * 0x9E3779B97F4A7C15 + _STREAM[stream] * 0xBF58476D1CE4E5B9
         + sub * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    z ^= z >> 31
    z = (z * 0xD6E8FEB86659FD93) & 0xFFFFFFFFFFFFFFFF
    z ^= z >> 32
    return torch.Generator().manual_seed(z & 0x7FFFFFFFFFFFFFFF)


def _normal(shape, std: float, gen: torch.Generator, dtype) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_x(w: Workload, seed: int = 0, T: Optional[int] = None,
           stream: str = "x") -> torch.Tensor:
    """Token activations x [T, d] in the workload dtype."""
    T = w.T if T is None else T
    g = _gen(seed, stream)
    if w.clusters == 0:
        return _normal((T, w.d), 1.0, g, w.torch_dtype)
    # cluster centres are shared by every batch drawn from this workload
    centers = torch.randn((w.clusters, w.d), generator=_gen(seed, "centers"))
    cid = torch.randint(0, w.clusters, (T,), generator=_gen(seed, "cluster_id", _STREAM[stream]))
    x = torch.randn((T, w.d), generator=g)
    x.mul_(w.sigma_within).add_(centers[cid])
    return x.to(w.torch_dtype)


def make_router(w: Workload, seed: int = 0) -> torch.Tensor:
    """W_router [d, E] ("ME"), N(0, 0.02^2)."""
    return _normal((w.d, w.E), 0.02, _gen(seed, "w_router"), w.torch_dtype)


def make_bias(w: Workload, seed: int = 0) -> Optional[torch.Tensor]:
    """Zipf expert-popularity bias [E] fp32 (None when the workload has none).

    Expert popularity p_e is proportional to rank_e^-s with ranks from a
    seeded permutation; the bias is ln(p_e / sum p).
    """
    if w.zipf <= 0:
        return None
    perm = torch.randperm(w.E, generator=_gen(seed, "bias_perm"))
    rank = perm.to(torch.float64) + 1.0
    p = rank.pow(-w.zipf)
    return torch.log(p / p.sum()).to(torch.float32)


def make_experts(w: Workload, seed: int = 0, experts: Optional[list] = None):
    """W_gate, W_up [E, d, f] ("EMH") and W_down [E, f, d] ("EHM"), N(0, 1/d).

    Each expert is drawn from its own sub-stream, so a subset of experts can
    be produced without drawing the others.
    """
    ids = list(range(w.E)) if experts is None else list(experts)
    std = 1.0 / math.sqrt(w.d)
    dt = w.torch_dtype
    wg = torch.empty((len(ids), w.d, w.f), dtype=dt)
    wu = torch.empty((len(ids), w.d, w.f), dtype=dt)
    wd = torch.empty((len(ids), w.f, w.d), dtype=dt)
    for i, e in enumerate(ids):
        wg[i] = _normal((w.d, w.f), std, _gen(seed, "w_gate", e), dt)
        wu[i] = _normal((w.d, w.f), std, _gen(seed, "w_up", e), dt)
        wd[i] = _normal((w.f, w.d), std, _gen(seed, "w_down", e), dt)
    return wg, wu, wd


def contiguous_placement(E: int, ep: int) -> list:
    """Expert e -> rank e // (E/ep) (Expert Coupling, Fig. 1 contiguous)."""
    per = E // ep
    return [e // per for e in range(E)]


def permutation_placement(E: int, ep: int, seed: int = 0) -> list:
    """map[e] = pi(e) // (E/ep) for a seeded permutation pi."""
    per = E // ep
    pi = torch.randperm(E, generator=_gen(seed, "placement", ep)).tolist()
    return [pi[e] // per for e in range(E)]


def uniform_routing(T: int, E: int, k: int, seed: int = 0) -> torch.Tensor:
    """Control input: each token's k distinct experts uniform at random.

    Used to pin dispatch statistics against their closed form.
    """
    g = _gen(seed, "sample", 7)
    keys = torch.rand((T, E), generator=g)
    return torch.argsort(keys, dim=1)[:, :k].to(torch.int32).contiguous()


def sample_tokens(T: int, n: int, seed: int = 0) -> torch.Tensor:
    """A seeded sorted sample of n distinct token indices in [0, T)."""
    n = min(n, T)
    g = _gen(seed, "sample")
    return torch.sort(torch.randperm(T, generator=g)[:n]).values.to(torch.int64)


def make_all(w: Workload, seed: int = 0, T: Optional[int] = None):
    """x, W_router, bias, W_gate, W_up, W_down for the workload."""
    x = make_x(w, seed, T)
    wr = make_router(w, seed)
    b = make_bias(w, seed)
    wg, wu, wd = make_experts(w, seed)
    return x, wr, b, wg, wu, wd
