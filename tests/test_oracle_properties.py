"""Property tests of the oracle's dispatch bookkeeping and top-k (no GPU): random shapes,
both layouts, both drop orders, capacities from tight to dropless, checked against the
definitions restated independently here (counting, sorting, and brute force)."""
import itertools

import numpy as np
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
