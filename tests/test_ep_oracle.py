"""Pins of the expert-parallel oracle (no GPU): a hand-worked case, layout invariants, and
the identity that drop-before-exchange EP equals the single-GPU layer on each rank's tokens."""
import json
import os

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import ep_oracle as EP
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ep_hand_g2_e4.json")


def test_hand_case_layout_and_stats():
    g = json.load(open(GOLDEN))
    for case in g["cases"]:
        lay = EP.recv_layout(g["kept_by_src"], case["expert_rank"])
        assert lay["base"].tolist() == case["base"]
        assert lay["offsets"] == case["offsets"]
        assert lay["rows"] == case["rows"]
        st = EP.ep_stats(g["kept_by_src"], case["expert_rank"], case["ranks_per_node"],
                         g["row_bytes"])
        for key, want in case["stats"].items():
            got = st[key]
            if isinstance(want, float):
                assert got == pytest.approx(want, rel=1e-12, abs=1e-12), key
            else:
                assert got == want, key


def test_hand_case_with_empty_pairs():
    """Pair percentiles over every ordered pair of different ranks, empty ones included
    (tests/golden/ep_hand_g3_e3_empty_pairs.json, derived by hand)."""
    g = json.load(open(os.path.join(os.path.dirname(GOLDEN), "ep_hand_g3_e3_empty_pairs.json")))
    lay = EP.recv_layout(g["kept_by_src"], g["expert_rank"])
    assert lay["base"].tolist() == g["base"]
    assert lay["offsets"] == g["offsets"] and lay["rows"] == g["rows"]
    st = EP.ep_stats(g["kept_by_src"], g["expert_rank"], g["ranks_per_node"], g["row_bytes"])
    for key, want in g["stats"].items():
        if isinstance(want, float):
            assert st[key] == pytest.approx(want, rel=1e-12, abs=1e-12), key
        else:
            assert st[key] == want, key


def test_contiguous_placement_values():
    # rank g owns the block [g E/world, (g+1) E/world)
    assert EP.contiguous_placement(8, 2).tolist() == [0, 0, 0, 0, 1, 1, 1, 1]
    assert EP.contiguous_placement(6, 3).tolist() == [0, 0, 1, 1, 2, 2]
    assert EP.contiguous_placement(4, 4).tolist() == [0, 1, 2, 3]
    assert EP.contiguous_placement(5, 1).tolist() == [0, 0, 0, 0, 0]
    assert EP.local_experts(EP.contiguous_placement(256, 8), 3).tolist() == list(range(96, 128))
    with pytest.raises(ValueError):
        EP.contiguous_placement(6, 4)


@pytest.mark.parametrize("G,E,seed", [(2, 8, 0), (4, 16, 1), (8, 256, 2), (3, 9, 3)])
def test_layout_invariants(G, E, seed):
    rng = np.random.default_rng(seed)
    kept = rng.integers(0, 7, size=(G, E))
    er = rng.permutation(EP.contiguous_placement(E, G))
    lay = EP.recv_layout(kept, er)
    for g in range(G):
        mine = EP.local_experts(er, g)
        offs = lay["offsets"][g]
        assert offs[0] == 0 and len(offs) == len(mine) + 1
        assert lay["rows"][g] == kept[:, mine].sum()
        for i, e in enumerate(mine):
            assert offs[i + 1] - offs[i] == kept[:, e].sum()
            # inside the bucket, sources in ascending order, back to back
            starts = [lay["base"][s, e] for s in range(G)]
            assert starts[0] == offs[i]
            for s in range(1, G):
                assert starts[s] == starts[s - 1] + kept[s - 1, e]
    st = EP.ep_stats(kept, er, 2, 100)
    assert sum(st["rank_load"]) == st["total_assignments"] == kept.sum()
    assert sum(st["bytes_sent"]) == sum(st["bytes_recv"]) == st["remote_bytes"]
    assert st["remote_bytes"] == (kept.sum() - st["local_assignments"]) * 100
    assert EP.ep_stats(kept, er, G, 100)["cross_node_bytes"] == 0
    assert EP.ep_stats(kept, er, 1, 100)["cross_node_bytes"] == st["remote_bytes"]


@settings(max_examples=200, deadline=None)
@given(G=st.integers(1, 6), per=st.integers(1, 5), rpn=st.integers(1, 4),
       seed=st.integers(0, 2**31 - 1), sparse=st.booleans())
def test_record_invariants_random(G, per, rpn, seed, sparse):
    """Any placement and any kept counts: the pair matrix accounts for every row once, the
    rank and node loads partition the assignments, sent equals received, the percentiles
    lie between the smallest and largest pair message, and ranks on one node exchange no
    cross-node bytes."""
    E = G * per
    rng = np.random.default_rng(seed)
    kept = rng.integers(0, 5, size=(G, E))
    if sparse:
        kept[rng.random((G, E)) < 0.6] = 0
    er = rng.permutation(EP.contiguous_placement(E, G))
    st_ = EP.ep_stats(kept, er, rpn, 7)
    total = int(kept.sum())
    assert st_["total_assignments"] == total == sum(st_["rank_load"]) == sum(st_["node_load"])
    assert st_["rank_load"] == [int(kept[:, er == g].sum()) for g in range(G)]
    local = sum(int(kept[g, er == g].sum()) for g in range(G))
    assert st_["local_assignments"] == local
    assert st_["remote_bytes"] == (total - local) * 7
    assert sum(st_["bytes_sent"]) == sum(st_["bytes_recv"]) == st_["remote_bytes"]
    for g in range(G):
        assert st_["bytes_sent"][g] == int(kept[g, er != g].sum()) * 7
        assert st_["bytes_recv"][g] == int(kept[np.arange(G) != g][:, er == g].sum()) * 7
    pairs = [int(kept[s_, er == g].sum()) * 7 for s_ in range(G) for g in range(G) if s_ != g]
    if pairs:
        assert min(pairs) <= st_["pair_bytes_p50"] <= st_["pair_bytes_p99"] <= max(pairs)
        assert st_["pair_bytes_max"] == max(pairs)
    assert 0 <= st_["cross_node_bytes"] <= st_["remote_bytes"]
    if rpn >= G:
        assert st_["cross_node_bytes"] == 0 and st_["nodes"] == 1
    if rpn == 1:
        assert st_["cross_node_bytes"] == st_["remote_bytes"]
    lay = EP.recv_layout(kept, er)
    assert lay["rows"] == [int(kept[:, er == g].sum()) for g in range(G)]
    # the receive slots of every (source, expert) are disjoint and tile each rank's buffer
    for g in range(G):
        used = np.zeros(lay["rows"][g], dtype=int)
        for e in EP.local_experts(er, g):
            for s_ in range(G):
                b = lay["base"][s_, e]
                used[b:b + kept[s_, e]] += 1
        assert (used == 1).all()


def _ranks(G, T, d, f, E, k, seed):
    rng = np.random.default_rng(seed)
    xs = [rng.standard_normal((T, d)) for _ in range(G)]
    w_router = rng.standard_normal((d, E)) / np.sqrt(d)
    wg = rng.standard_normal((E, f, d)) / np.sqrt(d)
    wu = rng.standard_normal((E, f, d)) / np.sqrt(d)
    wd = rng.standard_normal((E, d, f)) / np.sqrt(f)
    return xs, w_router, wg, wu, wd


@pytest.mark.parametrize("G,E,k,cf,permuted", [(2, 4, 2, 1.0, False), (4, 8, 2, 1.25, True),
                                                (2, 8, 3, 0.0, True), (1, 4, 2, 1.0, False)])
def test_ep_layer_equals_local_layer_per_rank(G, E, k, cf, permuted):
    T, d, f = 24, 16, 12
    xs, w_router, wg, wu, wd = _ranks(G, T, d, f, E, k, seed=G * 100 + E)
    er = EP.contiguous_placement(E, G)
    if permuted:
        er = np.random.default_rng(7).permutation(er)
    ep = EP.ep_layer(xs, w_router, None, wg, wu, wd, k, O.SOFTMAX, cf, er)
    for s in range(G):
        ref = O.moe_layer(xs[s], w_router, None, wg, wu, wd, k, O.SOFTMAX, cf)
        np.testing.assert_allclose(ep["out"][s], ref["out"], rtol=1e-12, atol=1e-12)
        # every kept pick's row in the owner's buffer is the token's x row
        r = ep["routes"][s]
        sr = ep["send_rows"][s]
        for t in range(T):
            for j in range(k):
                if sr[t, j] >= 0:
                    owner = er[r["idx"][t, j]]
                    np.testing.assert_array_equal(ep["recv"][owner][sr[t, j]], xs[s][t])
                else:
                    assert r["assign_row"][t, j] < 0
    if G == 1:
        assert ep["stats"]["local_fraction"] == 1.0 and ep["stats"]["remote_bytes"] == 0
    # each destination receives every kept row for its experts exactly once
    for g in range(G):
        used = np.zeros(ep["layout"]["rows"][g], dtype=int)
        for s in range(G):
            r, sr = ep["routes"][s], ep["send_rows"][s]
            for t in range(T):
                for j in range(k):
                    if sr[t, j] >= 0 and er[r["idx"][t, j]] == g:
                        used[sr[t, j]] += 1
        assert (used == 1).all()


def test_ep_layer_from_given_logits_uses_each_ranks_own():
    """Started from each rank's fp32 logits (the parity protocol), the EP layer equals the
    one that computes them itself."""
    G, E, k, cf, T, d, f = 3, 6, 2, 1.0, 20, 16, 12
    xs, w_router, wg, wu, wd = _ranks(G, T, d, f, E, k, seed=31)
    er = EP.contiguous_placement(E, G)
    z32s = [O.logits_to_fp32(O.router_logits(x, w_router)) for x in xs]
    a = EP.ep_layer(xs, w_router, None, wg, wu, wd, k, O.SOFTMAX, cf, er)
    b = EP.ep_layer(xs, w_router, None, wg, wu, wd, k, O.SOFTMAX, cf, er, z32s=z32s)
    for s in range(G):
        np.testing.assert_array_equal(a["routes"][s]["idx"], b["routes"][s]["idx"])
        np.testing.assert_array_equal(a["out"][s], b["out"][s])
    assert any(not np.array_equal(a["routes"][0]["idx"], a["routes"][s]["idx"])
               for s in range(1, G))


@pytest.mark.parametrize("variant", [
    dict(n_groups=4, topk_groups=2),
    dict(bias_mode=O.BIAS_SELECTION_ONLY),
    dict(drop_policy=O.DROP_PICK_RANK),
    dict(drop_policy=O.DROP_SCORE, bias_mode=O.BIAS_SELECTION_ONLY),
], ids=["groups", "sel_bias", "pick_rank", "score_drops"])
def test_ep_layer_with_routing_variants_equals_local_layer(variant):
    G, E, k, cf, T, d, f = 4, 8, 2, 0.75, 30, 16, 12
    xs, w_router, wg, wu, wd = _ranks(G, T, d, f, E, k, seed=99)
    rng = np.random.default_rng(5)
    biases = [rng.standard_normal((T, E)) * 2.0 for _ in range(G)]
    er = np.random.default_rng(8).permutation(EP.contiguous_placement(E, G))
    ep = EP.ep_layer(xs, w_router, biases, wg, wu, wd, k, O.SIGMOID, cf, er, **variant)
    drops = 0
    for s in range(G):
        ref = O.moe_layer(xs[s], w_router, biases[s], wg, wu, wd, k, O.SIGMOID, cf, **variant)
        np.testing.assert_allclose(ep["out"][s], ref["out"], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(ep["routes"][s]["assign_row"], ref["assign_row"])
        drops += int((ref["assign_row"] < 0).sum())
    assert drops > 0      # the capacity binds, so the drop order matters
