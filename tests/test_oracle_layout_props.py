"""Property-based pins of the oracle's dispatch layout: arbitrary routings
(an expert may repeat within a token, as a caller-supplied routing may),
arbitrary expert->rank partitions, every array and every statistic against
a brute force written from the definitions (stable order by flat index
inside an expert; one send row per distinct (rank, token), ranks ascending,
tokens ascending; home rank floor(t * ep / T)).  No GPU."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


def _brute(idx, E, ep, rmap):
    T, k = idx.shape
    flat = idx.reshape(-1)
    rows = sorted(range(T * k), key=lambda a: (flat[a], a))
    counts = np.bincount(flat, minlength=E)
    out = dict(expert_counts=counts,
               expert_offsets=np.concatenate([[0], np.cumsum(counts)]),
               row_token=np.array([a // k for a in rows], dtype=np.int64))
    slot_row = np.empty(T * k, np.int64)
    for r, a in enumerate(rows):
        slot_row[a] = r
    out["slot_row"] = slot_row
    ranks = [sorted({rmap[e] for e in idx[t]}) for t in range(T)]
    stats = dict(tokens_single_rank=sum(len(r) == 1 for r in ranks),
                 home_rank_rows=sum(rmap[idx[t, j]] == (t * ep) // T
                                    for t in range(T) for j in range(k)),
                 max_expert_rows=int(counts.max()) if T else 0,
                 min_expert_rows=int(counts.min()) if T else 0)
    if ep > 1:
        pairs = sorted((r, t) for t in range(T) for r in ranks[t])
        where = {p: i for i, p in enumerate(pairs)}
        rc = np.bincount([p[0] for p in pairs], minlength=ep)
        out.update(send_token=np.array([p[1] for p in pairs], np.int64),
                   slot_send_row=np.array([where[(rmap[flat[a]], a // k)] for a in range(T * k)],
                                          np.int64),
                   rank_counts=rc, rank_offsets=np.concatenate([[0], np.cumsum(rc)]))
        stats.update(rows_sent=len(pairs), dup_removed=T * k - len(pairs))
    else:
        stats.update(rows_sent=0, dup_removed=0)
    return out, stats


@st.composite
def cases(draw):
    ep = draw(st.sampled_from([1, 2, 3, 4, 8]))
    per = draw(st.integers(1, 4))
    E = ep * per
    k = draw(st.integers(1, min(E, 6)))
    T = draw(st.integers(0, 40))
    idx = np.array(draw(st.lists(st.lists(st.integers(0, E - 1), min_size=k, max_size=k),
                                 min_size=T, max_size=T)), dtype=np.int32).reshape(T, k)
    perm = draw(st.permutations(list(range(E))))
    rmap = [perm[e] // per for e in range(E)]       # any partition with E/ep per rank
    return idx, E, ep, rmap


@settings(max_examples=150, deadline=None)
@given(cases())
def test_layout_and_statistics_match_brute_force(case):
    idx, E, ep, rmap = case
    T, k = idx.shape
    got = oracle.dispatch_layout(idx, E, ep, rmap)
    ref, stats = _brute(idx, E, ep, rmap)
    for key, want in ref.items():
        if key == "send_token":
            n = int(ref["rank_offsets"][-1])
            np.testing.assert_array_equal(got[key][:n], want, err_msg=key)
        else:
            np.testing.assert_array_equal(got[key], want, err_msg=key)
    for key, want in stats.items():
        if T == 0 and key in ("max_expert_rows", "min_expert_rows"):
            continue
        assert got["stats"][key] == want, (key, got["stats"][key], want)
