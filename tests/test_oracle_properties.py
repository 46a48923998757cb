"""Property tests of the oracle's dispatch bookkeeping and top-k (no GPU): random shapes,
both layouts, both drop orders, capacities from tight to dropless, checked against the
definitions restated independently here (counting, sorting, and brute force)."""
import itertools

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import moe_oracle as O


def _topk_rows(rng, T, E, k):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])


@settings(max_examples=300, deadline=None)
@given(T=st.integers(1, 40), E=st.integers(1, 12), kk=st.integers(1, 8),
       cf=st.sampled_from([0.0, 0.2, 0.5, 1.0, 1.25, 3.0]), padded=st.booleans(),
       pick_rank=st.booleans(), seed=st.integers(0, 2**31 - 1))
def test_assignment_invariants(T, E, kk, cf, padded, pick_rank, seed):
    k = min(kk, E)
    rng = np.random.default_rng(seed)
    idx = _topk_rows(rng, T, E, k)
    C = O.capacity(cf, T, k, E)
    if padded and C is None:
        return
    layout = O.LAYOUT_PADDED if padded else O.LAYOUT_COMPACT
    policy = O.DROP_PICK_RANK if pick_rank else O.DROP_TOKEN_ORDER
    a = O.assign(idx, E, C, layout, policy)
    routed = np.bincount(idx.ravel(), minlength=E)
    assert (a["routed"] == routed).all()
    kept = routed if C is None else np.minimum(routed, C)
    assert (a["kept"] == kept).all()
    ar = a["assign_row"]
    assert int((ar >= 0).sum()) == int(kept.sum())
    assert int((ar < 0).sum()) == T * k - int(kept.sum())
    for e in range(E):
        start = e * C if padded else int(kept[:e].sum())
        assert a["offsets"][e] == start
        # the expert's picks in the policy's order; the first C keep slots 0, 1, ...
        picks = [(j, t) if pick_rank else (t, j) for t in range(T) for j in range(k)
                 if idx[t, j] == e]
        picks.sort()
        for slot, p in enumerate(picks):
            t, j = (p[1], p[0]) if pick_rank else p
            if C is not None and slot >= C:
                assert ar[t, j] == -1
            else:
                assert ar[t, j] == start + slot
                assert a["token_of_row"][start + slot] == t
    used = ar[ar >= 0]
    assert len(np.unique(used)) == len(used)             # a row holds one pick
    assert (a["token_of_row"] >= 0).sum() == len(used)   # every other row is unused


@settings(max_examples=300, deadline=None)
@given(T=st.integers(1, 6), E=st.integers(1, 7), kk=st.integers(1, 7),
       seed=st.integers(0, 2**31 - 1), ties=st.booleans())
def test_topk_is_best_subset_in_order(T, E, kk, seed, ties):
    k = min(kk, E)
    rng = np.random.default_rng(seed)
    z = (rng.integers(-3, 4, size=(T, E)) if ties else rng.standard_normal((T, E)))
    z = z.astype(np.float32)
    idx = O.select_topk(z, k)
    for t in range(T):
        # brute force: the k-subset with the largest sorted score vector, ties by index
        order = sorted(range(E), key=lambda e: (-float(z[t, e]), e))
        assert list(idx[t]) == order[:k]
        best = max(itertools.combinations(range(E), k), key=lambda c: sorted(
            (float(z[t, e]) for e in c), reverse=True))
        assert sorted(float(z[t, e]) for e in idx[t]) == sorted(float(z[t, e]) for e in best)


def _prio(v):
    """Larger = kept first: NaN below every number; -0 equals +0."""
    return (0, 0.0) if v != v else (1, float(v))


@settings(max_examples=300, deadline=None)
@given(T=st.integers(1, 40), E=st.integers(1, 12), kk=st.integers(1, 8),
       cf=st.sampled_from([0.0, 0.2, 0.5, 1.0, 1.25, 3.0]), padded=st.booleans(),
       seed=st.integers(0, 2**31 - 1), ties=st.booleans())
def test_score_drop_invariants(T, E, kk, cf, padded, seed, ties):
    """Score priority, checked by exchange: no dropped pick of an expert outranks one of its
    kept picks (higher score, or equal score and lower token); kept picks fill their bucket
    in token order; the counts, and the pick-rank counters, agree with the assignment."""
    k = min(kk, E)
    rng = np.random.default_rng(seed)
    idx = _topk_rows(rng, T, E, k)
    sc = (rng.integers(-2, 3, size=(T, E)) if ties else rng.standard_normal((T, E)))
    sc = sc.astype(np.float32)
    if ties:
        sc[rng.random((T, E)) < 0.1] = np.nan
    C = O.capacity(cf, T, k, E)
    if padded and C is None:
        return
    layout = O.LAYOUT_PADDED if padded else O.LAYOUT_COMPACT
    a = O.assign(idx, E, C, layout, O.DROP_SCORE, scores=sc)
    ar = a["assign_row"]
    routed = np.bincount(idx.ravel(), minlength=E)
    kept = routed if C is None else np.minimum(routed, C)
    assert (a["routed"] == routed).all() and (a["kept"] == kept).all()
    for e in range(E):
        picks = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e]
        kp = [(t, j) for t, j in picks if ar[t, j] >= 0]
        dr = [(t, j) for t, j in picks if ar[t, j] < 0]
        assert len(kp) == kept[e]
        for tk, jk in kp:
            for td, jd in dr:
                pk, pd = _prio(sc[tk, e]), _prio(sc[td, e])
                assert pk > pd or (pk == pd and tk < td)
        start = e * C if padded else int(kept[:e].sum())
        assert [ar[t, j] for t, j in kp] == list(range(start, start + len(kp)))
        assert [a["token_of_row"][ar[t, j]] for t, j in kp] == [t for t, _ in kp]
    if C is None or (routed <= C).all():
        tok = O.assign(idx, E, C, layout, O.DROP_TOKEN_ORDER)
        assert (tok["assign_row"] == ar).all()
    c = O.pick_rank_counts(idx, ar, E)
    assert (c["routed"].sum(axis=0) == routed).all() and (c["routed"].sum(axis=1) == T).all()
    assert (c["kept"].sum(axis=0) == kept).all()
    st_ = O.load_stats(a["routed"], a["kept"], ar, C)
    assert [T - int(c["kept"][j].sum()) for j in range(k)] == st_["dropped_by_rank"][:k]
    assert c["differs"][0] == 0 and all(c["differs"][1:] == T)    # distinct picks
    g = rng.integers(0, 3, size=E)
    cg = O.pick_rank_counts(idx, ar, E, group_of_expert=g)
    for j in range(k):
        assert cg["differs"][j] == sum(1 for t in range(T) if g[idx[t, j]] != g[idx[t, 0]])


@settings(max_examples=150, deadline=None)
@given(parts=st.integers(1, 5), E=st.integers(1, 12), kk=st.integers(1, 4),
       cf=st.sampled_from([0.0, 0.5, 1.0, 2.0]), seed=st.integers(0, 2**31 - 1))
def test_replica_record_invariants(parts, E, kk, cf, seed):
    """The job record adds up the replicas': counts, drops and tokens are sums, the capacity
    is the sum of the capacities, and the percentiles are those of the summed kept counts."""
    k = min(kk, E)
    rng = np.random.default_rng(seed)
    recs, singles = [], []
    for _ in range(parts):
        T = int(rng.integers(1, 30))
        idx = _topk_rows(rng, T, E, k)
        C = O.capacity(cf, T, k, E)
        a = O.assign(idx, E, C)
        recs.append((a["routed"], a["kept"], a["assign_row"], C))
        singles.append(O.load_stats(a["routed"], a["kept"], a["assign_row"], C))
    job = O.replica_load_stats(recs)
    for key in ("active_tokens", "routed_total", "kept_total", "dropped", "tokens_with_drop",
                "tokens_fully_dropped"):
        assert job[key] == sum(s[key] for s in singles), key
    assert job["dropped_by_rank"] == [sum(s["dropped_by_rank"][j] for s in singles)
                                      for j in range(k)]
    caps = [r[3] for r in recs]
    assert job["capacity"] == (-1 if any(c is None for c in caps) else sum(caps))
    kept = np.sum([r[1] for r in recs], axis=0)
    assert job["max"] == float(kept.max())
    assert job["p50"] == pytest.approx(float(np.percentile(kept, 50)))
    if job["capacity"] >= 0:
        assert job["max"] <= job["capacity"]
