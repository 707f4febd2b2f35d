"""Shared helpers of the GPU parity tests: seeded inputs on both sides, the
near-tie injection of the top-6 workload, and tolerance checks.

Inputs are always drawn on the CPU (routing_dispatch_experts_b200.workloads)
and copied to the GPU; expected values come only from the CPU oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W

# max |y_gpu - y_oracle| <= TOL * max |y_oracle|: bf16 storage with fp32
# accumulation (2e-2), and the fp32 workload (1e-5)
TOL = {"bf16": 2e-2, "f32": 1e-5}
# routing decisions whose margin is below this may legitimately differ
NEAR_TIE = 1e-5


def shape_of(w: W.Workload, T=None, ep=1) -> moe.Shape:
    return moe.Shape(T=w.T if T is None else T, d=w.d, E=w.E, k=w.k, f=w.f, ep=ep,
                     dtype=w.torch_dtype)


# weights depend only on (E, d, f, dtype, seed): workloads that share them
# (and cases of one workload at several token counts) draw and pack them once
_WEIGHTS = {}


def _weights(w: W.Workload, seed: int):
    key = (w.E, w.d, w.f, w.dtype, seed)
    if key not in _WEIGHTS:
        wr = W.make_router(w, seed)
        wg, wu, wd = W.make_experts(w, seed)
        dev = "cuda"
        shape = shape_of(w, 0)
        packed = moe.pack_weights(shape, wr.to(dev), wg.to(dev), wu.to(dev), wd.to(dev))
        torch.cuda.synchronize()
        _WEIGHTS.clear()  # keep one set resident (the large workload's is 4.8 GB)
        _WEIGHTS[key] = (wr, wg, wu, wd, packed)
    return _WEIGHTS[key]


class Case:
    """One workload instance: CPU tensors, device tensors and packed weights."""

    def __init__(self, cfg: int, T=None, seed=0, near_ties=None, experts=None):
        self.w = W.WORKLOADS[cfg]
        self.T = self.w.T if T is None else T
        self.x = W.make_x(self.w, seed, self.T)
        self.bias = W.make_bias(self.w, seed)
        self.wr, self.wg, self.wu, self.wd, self.packed = _weights(self.w, seed)
        inject = self.w.near_tie_frac > 0 if near_ties is None else near_ties
        self.near_tie_tokens = inject_near_ties(self, seed) if inject else np.array([], np.int64)
        self.shape = shape_of(self.w, self.T)
        dev = "cuda"
        self.dx = self.x.to(dev)
        self.dbias = None if self.bias is None else self.bias.to(dev)
        torch.cuda.synchronize()

    def shape_ep(self, ep):
        return shape_of(self.w, self.T, ep)


def _bf16_step(v: np.ndarray, up: bool) -> np.ndarray:
    """Next bf16 value above / below (bit patterns as uint16)."""
    neg = (v & 0x8000) != 0
    mag = v & 0x7FFF
    out = v.copy()
    # moving away from zero increments the magnitude
    away = ~neg if up else neg
    out[away] = v[away] + 1
    tow = ~away
    zero = tow & (mag == 0)
    out[tow & ~zero] = v[tow & ~zero] - 1
    out[zero] = 0x0001 if up else 0x8001
    return out


def _nudge_to_tie(row, wr, b, k, target, max_steps):
    """Move one token's bf16 row toward a tie of its k-th and (k+1)-th
    router logits (double).  Returns (row, reached): reached is True once
    the gap is at most `target` times the token's logit spread."""
    # coarse move: project x onto the tie plane of the k-th / (k+1)-th
    # experts in double, then round back to bf16
    xv = torch.from_numpy(row.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    l = xv @ wr + b
    o = np.argsort(-l, kind="stable")
    v = wr[:, o[k - 1]] - wr[:, o[k]]
    xv = xv - (l[o[k - 1]] - l[o[k]]) / (v @ v) * v
    row = torch.from_numpy(xv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    for _ in range(max_steps + 1):
        xv = torch.from_numpy(row.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        l = xv @ wr + b
        o = np.argsort(-l, kind="stable")
        a, c = o[k - 1], o[k]
        spread = l.max() - l.min()
        gap = l[a] - l[c]
        if gap <= target * spread:
            return row, True
        v = wr[:, a] - wr[:, c]
        # every coordinate's one-ulp step up and down, pick the best
        up = _bf16_step(row, True)
        dn = _bf16_step(row, False)
        xu = torch.from_numpy(up.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        xd = torch.from_numpy(dn.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        gu = gap + (xu - xv) * v
        gd = gap + (xd - xv) * v
        gu[~np.isfinite(gu)] = np.inf
        gd[~np.isfinite(gd)] = np.inf
        iu, idn = np.argmin(np.abs(gu)), np.argmin(np.abs(gd))
        if abs(gu[iu]) <= abs(gd[idn]):
            row[iu] = up[iu]
        else:
            row[idn] = dn[idn]
    return row, False


def inject_near_ties(case: Case, seed: int, frac=None, target=5e-6, max_steps=4000):
    """Nudge x of a seeded fraction of tokens, one bf16 ulp at a time, until
    the gap between the k-th and (k+1)-th router logits (in double) is below
    `target` times the token's logit spread.  A token that does not get there
    within `max_steps` keeps its original x and is replaced by the next
    candidate (the seeded sample first, then the other tokens in a seeded
    order), so every returned token is a near-tie.  Returns the tokens
    changed, ascending."""
    w = case.w
    frac = w.near_tie_frac if frac is None else frac
    n = int(round(frac * case.T))
    if n == 0:
        return np.array([], np.int64)
    first = W.sample_tokens(case.T, n, seed + 101).numpy()
    g = torch.Generator().manual_seed(seed + 202)
    picked = set(first.tolist())
    rest = [t for t in torch.randperm(case.T, generator=g).tolist() if t not in picked]
    wr = case.wr.double().numpy()
    b = 0.0 if case.bias is None else case.bias.double().numpy()
    xb = case.x.view(torch.int16).numpy().view(np.uint16)
    done = []
    for t in list(first) + rest:
        if len(done) == n:
            break
        row, reached = _nudge_to_tie(xb[t].copy(), wr, b, w.k, target, max_steps)
        if reached:
            xb[t] = row
            done.append(int(t))
    return np.array(sorted(done), np.int64)


def routing_mismatches(idx_gpu: np.ndarray, idx_ref: np.ndarray) -> np.ndarray:
    """Tokens whose expert sets differ."""
    return np.where((np.sort(idx_gpu, 1) != np.sort(idx_ref, 1)).any(1))[0]


def check_output(y_gpu: torch.Tensor, y_ref: np.ndarray, dtype: str, rows=None):
    yg = y_gpu.float().cpu().double().numpy()
    if rows is not None:
        yg, y_ref = yg[rows], y_ref[rows]
    if yg.size == 0:
        return 0.0
    scale = np.abs(y_ref).max()
    err = np.abs(yg - y_ref).max()
    assert err <= TOL[dtype] * scale, f"max|dy| = {err:.3e} > {TOL[dtype]} * {scale:.3e}"
    return err / scale
