"""CPU oracle of the MoE-layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
binding) never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain loops in double, compiled with
gcc + OpenMP over the outer token/row loop).  This wrapper marshals numpy /
torch CPU arrays and adds the host-side correlated-placement fit of "Expert
Coupling in MoE Pretraining" (Abstract: co-selected experts on one GPU;
Table III: co-selection count W[e,e']).

Every function returns float64 results for floating-point outputs, so a test
rounds them to the compared precision itself.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile liboracle.so next to oracle.c (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64, I32 = ctypes.c_int64, ctypes.c_int32
        _lib.oracle_router_logits.argtypes = [I64, I32, I32, I32, P, P, P, P, I64, P]
        _lib.oracle_topk.argtypes = [I64, I32, I32, P, P, P]
        _lib.oracle_margin.argtypes = [I64, I32, I32, P, P]
        _lib.oracle_dispatch_layout.argtypes = [I64, I32, I32, I32, P, P] + [P] * 9
        _lib.oracle_dispatch_layout.restype = ctypes.c_int
        _lib.oracle_grouped_swiglu.argtypes = [I32, I32, I32, I32, P, P, P, P, P, P, I64, P]
        _lib.oracle_combine.argtypes = [I64, I32, I32, I32, P, P, P, P, P]
        _lib.oracle_moe_output.argtypes = [I64, I32, I32, I32, I32, P, P, P, P, P, P, P, I64, P]
        _lib.oracle_num_threads.restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


# ---------------------------------------------------------------- marshalling
def _typed(a):
    """(contiguous numpy array of the stored bits, dtype code)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), BF16
            if a.dtype == torch.float32:
                return a.numpy(), F32
            raise TypeError(f"unsupported dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"unsupported dtype {a.dtype}")


def _np(a, dtype):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- the steps
def router_logits(x, w_router, bias=None, tokens=None) -> np.ndarray:
    """l[t,e] = sum_i x[t,i] W_r[i,e] + bias[e] in double.  [n, E]."""
    xb, dt = _typed(x)
    wb, dt2 = _typed(w_router)
    assert dt == dt2
    T, d = xb.shape
    E = wb.shape[1]
    b = None if bias is None else _np(bias, np.float32)
    tk = None if tokens is None else _np(tokens, np.int64)
    n = T if tk is None else len(tk)
    out = np.empty((n, E), np.float64)
    _load().oracle_router_logits(T, d, E, dt, _ptr(xb), _ptr(wb), _ptr(b), _ptr(tk), n, _ptr(out))
    return out


def topk(logits, k: int):
    """(idx int32 [n,k], gate float64 [n,k]) from logits (any real dtype)."""
    l = _np(logits, np.float64)
    n, E = l.shape
    idx = np.empty((n, k), np.int32)
    gate = np.empty((n, k), np.float64)
    _load().oracle_topk(n, E, k, _ptr(l), _ptr(idx), _ptr(gate))
    return idx, gate


def margin(logits, k: int) -> np.ndarray:
    """Routing margin (k-th minus (k+1)-th score) / (max - min), per token."""
    l = _np(logits, np.float64)
    n, E = l.shape
    m = np.empty(n, np.float64)
    _load().oracle_margin(n, E, k, _ptr(l), _ptr(m))
    return m


STAT_NAMES = ("rows_sent", "dup_removed", "tokens_single_rank",
              "home_rank_rows", "max_expert_rows", "min_expert_rows")


def dispatch_layout(idx, E: int, ep: int = 1, expert_rank=None) -> dict:
    """Expert-grouped layout + deduplicated send layout (see oracle.c)."""
    ix = _np(idx, np.int32)
    T, k = ix.shape
    R = T * k
    m = (np.arange(E, dtype=np.int32) // (E // ep) if expert_rank is None
         else _np(expert_rank, np.int32))
    out = dict(
        expert_counts=np.zeros(E, np.int32), expert_offsets=np.zeros(E + 1, np.int32),
        row_token=np.zeros(R, np.int32), slot_row=np.zeros(R, np.int32),
        rank_counts=np.zeros(ep, np.int32), rank_offsets=np.zeros(ep + 1, np.int32),
        send_token=np.zeros(R, np.int32), slot_send_row=np.zeros(R, np.int32),
    )
    st = np.zeros(6, np.int64)
    rc = _load().oracle_dispatch_layout(
        T, E, k, ep, _ptr(ix), _ptr(m), *[_ptr(out[n]) for n in (
            "expert_counts", "expert_offsets", "row_token", "slot_row", "rank_counts",
            "rank_offsets", "send_token", "slot_send_row")], _ptr(st))
    if rc != 0:
        raise ValueError("expert index out of range")
    if ep > 1:
        out["send_token"] = out["send_token"][: int(st[0])]
    out["stats"] = dict(zip(STAT_NAMES, (int(v) for v in st)))
    return out


def grouped_swiglu(x_perm, expert_offsets, w_gate, w_up, w_down, rows=None) -> np.ndarray:
    """y_perm[r] = SwiGLU expert of row r applied to x_perm[r], in double."""
    xb, dt = _typed(x_perm)
    g, _ = _typed(w_gate)
    u, _ = _typed(w_up)
    dn, _ = _typed(w_down)
    off = _np(expert_offsets, np.int32)
    E, d, f = g.shape
    rw = None if rows is None else _np(rows, np.int64)
    n = int(off[E]) if rw is None else len(rw)
    out = np.empty((n, d), np.float64)
    _load().oracle_grouped_swiglu(d, E, f, dt, _ptr(xb), _ptr(off), _ptr(g), _ptr(u), _ptr(dn),
                                  _ptr(rw), n, _ptr(out))
    return out


def combine(y_perm, slot_row, gate=None, k: int = None) -> np.ndarray:
    """y[t] = sum_j gate[t,j] y_perm[slot_row[t*k+j]] (j ascending), double."""
    sr = _np(slot_row, np.int32).reshape(-1)
    if isinstance(y_perm, np.ndarray) and y_perm.dtype == np.float64:
        yd, yt, dt = np.ascontiguousarray(y_perm), None, F32
    else:
        yd = None
        yt, dt = _typed(y_perm)
    d = (yd if yd is not None else yt).shape[1]
    g = None if gate is None else _np(gate, np.float64)
    if k is None:
        k = g.shape[1]
    T = sr.size // k
    out = np.empty((T, d), np.float64)
    _load().oracle_combine(T, d, k, dt, _ptr(yt), _ptr(yd), _ptr(sr), _ptr(g), _ptr(out))
    return out


def moe_output(x, idx, gate, w_gate, w_up, w_down, tokens=None) -> np.ndarray:
    """y[t] = sum_j gate[t,j] expert_{idx[t,j]}(x[t]) for listed tokens."""
    xb, dt = _typed(x)
    g, _ = _typed(w_gate)
    u, _ = _typed(w_up)
    dn, _ = _typed(w_down)
    ix = _np(idx, np.int32)
    ga = _np(gate, np.float64)
    T, d = xb.shape
    k = ix.shape[1]
    f = g.shape[2]
    tk = None if tokens is None else _np(tokens, np.int64)
    n = T if tk is None else len(tk)
    assert ix.shape[0] == n and ga.shape == ix.shape
    out = np.empty((n, d), np.float64)
    _load().oracle_moe_output(T, d, k, f, dt, _ptr(xb), _ptr(ix), _ptr(ga), _ptr(g), _ptr(u),
                              _ptr(dn), _ptr(tk), n, _ptr(out))
    return out


def forward(x, w_router, bias, w_gate, w_up, w_down, k: int, tokens=None) -> dict:
    """Whole layer for listed tokens: logits, routing, gates and output."""
    l = router_logits(x, w_router, bias, tokens)
    idx, gate = topk(l, k)
    y = moe_output(x, idx, gate, w_gate, w_up, w_down, tokens)
    return dict(logits=l, idx=idx, gate=gate, y=y)


# ------------------------------------------------ correlated placement (host)
def coselection_counts(idx, E: int) -> np.ndarray:
    """W[e,e'] = number of tokens that select both e and e' (e != e')."""
    ix = _np(idx, np.int64)
    W = np.zeros((E, E), np.int64)
    T, k = ix.shape
    for a in range(k):
        for b in range(k):
            if a != b:
                np.add.at(W, (ix[:, a], ix[:, b]), 1)
    return W


def fit_correlated_placement(idx, E: int, ep: int) -> list:
    """Greedy correlated placement: often co-selected experts share a rank.

    For each rank in order: seed it with the unassigned expert of largest
    row sum of W (ties: lowest index), then repeatedly add the unassigned
    expert with the largest total co-selection with the rank's members (ties:
    lowest index) until the rank holds E/ep experts.
    """
    W = coselection_counts(idx, E)
    per = E // ep
    free = set(range(E))
    rank_of = [-1] * E
    for r in range(ep):
        seed = max(sorted(free), key=lambda e: (int(W[e].sum()), -e))
        members = [seed]
        free.discard(seed)
        while len(members) < per:
            best = max(sorted(free), key=lambda e: (int(W[e, members].sum()), -e))
            members.append(best)
            free.discard(best)
        for e in members:
            rank_of[e] = r
    return rank_of


# ----------------------------------------------------------------------------
# Routing variants and router observability.  Oracle side only so far: the
# CUDA path does not implement these yet.

def near_tie_share(logits, k: int, threshold: float = 1e-5) -> float:
    """Share of tokens whose routing margin is below `threshold`: the router
    statistic that "MoE Pretraining: Parallelism Layout Changes the Model,
    Not Quality" (Practical Implications: monitor the router) recommends
    logging next to the loss.  Margin as in margin(); k = E has no margin
    and counts as no tie."""
    m = margin(logits, k)
    return float(np.mean(m < threshold)) if len(m) else 0.0


def routing_changes(idx_a, idx_b) -> dict:
    """How two routings of the same tokens differ (a run against a recorded
    routing table, same page, Practical Implications):
      tokens   tokens whose set of k experts differs
      experts  sum over tokens of |A(t) minus B(t)|, the experts swapped
      slots    (t, j) whose expert differs, slot order included."""
    a = _np(idx_a, np.int64)
    b = _np(idx_b, np.int64)
    assert a.shape == b.shape
    swapped = np.array([len(set(ra) - set(rb)) for ra, rb in zip(a.tolist(), b.tolist())],
                       np.int64)
    return dict(tokens=int((swapped > 0).sum()), experts=int(swapped.sum()),
                slots=int((a != b).sum()))


def topk_selection_bias(logits, bias, k: int):
    """Top-k with a selection-only expert bias (the auxiliary-loss-free
    router named in "Expert Coupling in MoE Pretraining", Fig. 11; the
    loss-free balancing counts of "MoE Pretraining: Parallelism Layout
    Changes the Model, Not Quality", introduction): the experts are chosen
    on logits + bias under the usual key (value desc, index asc), and the
    gates are the softmax of the chosen experts' logits without the bias,
    in the chosen order.  The sum logits + bias is taken in float32, the
    precision a kernel adding two float32 vectors decides in.
    Returns (idx int32 [n, k], gate float64 [n, k])."""
    l = _np(logits, np.float64)
    b = _np(bias, np.float64)
    key = (l.astype(np.float32) + b.astype(np.float32)[None, :]).astype(np.float64)
    idx, _ = topk(key, k)
    chosen = np.take_along_axis(l, idx.astype(np.int64), 1)
    e = np.exp(chosen - chosen.max(1, keepdims=True))
    return idx, e / e.sum(1, keepdims=True)


def expert_capacity(T: int, k: int, E: int, capacity_factor: float) -> int:
    """Rows an expert may take: ceil(capacity_factor * T * k / E), the factor
    times an expert's mean load ("Revisiting MoE and Dense Speed-Accuracy
    Comparisons", 2.1: expert capacity factor 2 with top-2 routing; the
    formula is the reading taken where the page names only the factor)."""
    return int(math.ceil(capacity_factor * T * k / E))


def capacity_keep(idx, E: int, capacity_factor: float) -> np.ndarray:
    """Which assignments an expert of limited capacity keeps (bool [T, k]).
    Reading taken: every token's first choice is served before any token's
    second choice, and so on (choice rank j ascending), tokens in order
    inside a rank; an assignment is kept while its expert has taken fewer
    than expert_capacity() rows.  A dropped assignment contributes nothing
    to the token's output (its gate is not redistributed)."""
    ix = _np(idx, np.int64)
    T, k = ix.shape
    cap = expert_capacity(T, k, E, capacity_factor)
    taken = [0] * E
    keep = np.zeros((T, k), bool)
    for j in range(k):
        for t in range(T):
            e = int(ix[t, j])
            if taken[e] < cap:
                taken[e] += 1
                keep[t, j] = True
    return keep
