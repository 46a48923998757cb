"""Pins for the CPU oracle (runs without a GPU).

Each test ties one oracle function to something other than itself: a hand-worked case,
brute force, an independent library routine, a closed form, or an invariant.  Together
they are chosen so that a dropped term, a wrong sign, a swapped index or a transposed
operand anywhere in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_warp_b200 import workload as W


def _hand(golden_dir):
    with open(os.path.join(golden_dir, "hand_e4_k2_t8.json")) as f:
        return json.load(f)


# ---------------------------------------------------------------- hand-worked case
def test_hand_case_routing(golden_dir):
    g = _hand(golden_dir)
    z = np.array(g["logits"], dtype=np.float32)
    idx = O.select_topk(z, g["k"])
    assert idx.tolist() == g["topk_idx"]
    C = O.capacity(g["capacity_factor"], g["T"], g["k"], g["E"])
    assert C == g["capacity"]
    for layout, key in ((O.LAYOUT_COMPACT, "compact"), (O.LAYOUT_PADDED, "padded")):
        a = O.assign(idx, g["E"], C, layout)
        assert a["routed"].tolist() == g["routed"]
        assert a["kept"].tolist() == g["kept"]
        assert a["offsets"].tolist() == g[key]["offsets"]
        assert a["assign_row"].tolist() == g[key]["assign_row"]
        assert a["token_of_row"].tolist() == g[key]["token_of_row"]


def test_hand_case_weights(golden_dir):
    g = _hand(golden_dir)
    z = np.array(g["logits"], dtype=np.float32)
    idx = np.array(g["topk_idx"])
    w = O.gate_weights(z, idx, O.SOFTMAX)
    np.testing.assert_allclose(w, np.array(g["softmax_w"]), rtol=0, atol=1e-15)


def test_hand_case_stats(golden_dir):
    g = _hand(golden_dir)
    a = O.assign(np.array(g["topk_idx"]), g["E"], g["capacity"])
    s = O.load_stats(a["routed"], a["kept"], a["assign_row"], g["capacity"])
    for key, v in g["stats"].items():
        if isinstance(v, list):
            assert s[key] == v, key
        else:
            assert s[key] == pytest.approx(v, abs=1e-12), key
    assert s["tokens_per_expert"] == g["kept"]


def test_softmax_weights_of_far_apart_logits():
    # exp(-1000) underflows to 0 in float64, so the exact weights round to (1, 0, 0) and a
    # softmax shifted by anything but the largest pick would overflow to inf / inf
    z = np.array([[500.0, -500.0, 0.0]], dtype=np.float32)
    w = O.gate_weights(z, np.array([[0, 2, 1]]), O.SOFTMAX)
    assert w[0].tolist() == [1.0, math.exp(-500.0), 0.0]


def test_top5pct_share_counts_ceil_of_five_percent():
    """The top-5% share sums the ceil(0.05 E) largest kept counts: 2 experts at E = 32
    (0.05 * 32 = 1.6), 13 at E = 256 (12.8).  Values worked by hand."""
    # E = 32: counts 10, 9 and thirty 1s, 49 kept in all; the two largest hold 19
    kept = [10, 9] + [1] * 30
    rows = np.zeros((49, 1), dtype=np.int64)
    s = O.load_stats(kept, kept, rows, None)
    assert s["top5pct_share"] == pytest.approx(19 / 49, abs=1e-15)
    assert s["max_to_mean"] == pytest.approx(320 / 49, abs=1e-12)   # 10 / (49 / 32)
    # sorted: thirty 1s, 9, 10.  p50: h = 15.5 between two 1s; p95: h = 29.45 between the
    # last 1 and 9 -> 1 + 0.45 * 8; p99: h = 30.69 between 9 and 10 -> 9.69
    assert s["p50"] == pytest.approx(1.0, abs=1e-12)
    assert s["p95"] == pytest.approx(4.6, abs=1e-12)
    assert s["p99"] == pytest.approx(9.69, abs=1e-12)
    # E = 256: thirteen experts with 2, the other 243 with 1: 269 kept, top 13 hold 26
    kept = [2] * 13 + [1] * 243
    s = O.load_stats(kept, kept, np.zeros((269, 1), dtype=np.int64), None)
    assert s["top5pct_share"] == pytest.approx(26 / 269, abs=1e-15)


def test_sigmoid_weights_hand_values():
    # sigma(3) = 0.9525741268224334, sigma(2) = 0.8807970779778823 (tabulated values)
    z = np.array([[3.0, 2.0, -1.0]], dtype=np.float32)
    w = O.gate_weights(z, np.array([[0, 1]]), O.SIGMOID)
    s3, s2 = 0.9525741268224334, 0.8807970779778823
    np.testing.assert_allclose(w[0], [s3 / (s3 + s2), s2 / (s3 + s2)], rtol=0, atol=1e-15)
    # equal logits share the weight equally; the order of picks is respected
    w = O.gate_weights(np.array([[0.5, -2.0, 0.5]], dtype=np.float32), np.array([[2, 1, 0]]),
                       O.SIGMOID)
    assert w[0, 0] == pytest.approx(w[0, 2], abs=1e-15)
    assert w[0, 1] < w[0, 0]


# ---------------------------------------------------------------- brute force top-k
def _brute_topk(zrow, k):
    """Among all k-subsets, the unique one in which every member beats every non-member
    under (larger value, then lower index); ordered the same way."""
    E = len(zrow)
    beats = lambda i, j: zrow[i] > zrow[j] or (zrow[i] == zrow[j] and i < j)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [j for j in range(E) if j not in S]
        if all(beats(i, j) for i in S for j in rest):
            found.append(S)
    assert len(found) == 1
    S = list(found[0])
    # order within the subset: insertion by 'beats'
    ordered = []
    for i in S:
        pos = 0
        while pos < len(ordered) and beats(ordered[pos], i):
            pos += 1
        ordered.insert(pos, i)
    return ordered


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (6, 3), (8, 2), (8, 8), (7, 5)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 100 + k)
    for trial in range(40):
        if trial % 2:
            z = rng.integers(-2, 3, size=(1, E)).astype(np.float32)   # many ties
        else:
            z = rng.standard_normal((1, E)).astype(np.float32)
        idx = O.select_topk(z, k)
        assert idx[0].tolist() == _brute_topk(z[0].tolist(), k)


def test_topk_signed_zero_is_a_tie():
    z = np.array([[-0.0, 0.0, -1.0]], dtype=np.float32)
    assert O.select_topk(z, 2)[0].tolist() == [0, 1]


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,E,k,cf", [(37, 5, 2, 1.0), (64, 8, 2, 1.25), (50, 16, 4, 0.5),
                                      (40, 8, 3, 0.0), (9, 3, 3, 2.0)])
def test_assign_matches_stable_sort_and_bincount(T, E, k, cf):
    rng = np.random.default_rng(T + E)
    z = rng.standard_normal((T, E)).astype(np.float32)
    z[:, 0] += 1.0   # make expert 0 hot so capacity bites
    idx = O.select_topk(z, k)
    C = O.capacity(cf, T, k, E)
    a = O.assign(idx, E, C)
    # counts: bincount
    assert a["routed"].tolist() == np.bincount(idx.ravel(), minlength=E).tolist()
    # permutation: stable sort of the assignment list on key e*T + t
    flat_e = idx.ravel()
    flat_t = np.repeat(np.arange(T), k)
    order = np.argsort(flat_e.astype(np.int64) * T + flat_t, kind="stable")
    slot = np.empty(T * k, dtype=np.int64)
    start = np.concatenate([[0], np.cumsum(np.bincount(flat_e, minlength=E))])
    slot[order] = np.arange(T * k) - start[flat_e[order]]
    assert a["slot"].ravel().tolist() == slot.tolist()
    kept_mask = slot < (C if C is not None else T * k + 1)
    kept = np.bincount(flat_e[kept_mask], minlength=E)
    assert a["kept"].tolist() == kept.tolist()
    # rows of the kept assignments, in stable-sort order, are 0..Σkept-1 (COMPACT)
    kept_order = [i for i in order if kept_mask[i]]
    assert [int(a["assign_row"].ravel()[i]) for i in kept_order] == list(range(int(kept.sum())))
    # invariants
    assert int(a["kept"].sum()) == T * k - int((a["assign_row"] < 0).sum())
    if C is not None:
        assert (a["kept"] <= C).all()
    used = a["token_of_row"]
    assert (used >= 0).all()
    # every kept assignment appears exactly once
    rows = a["assign_row"][a["assign_row"] >= 0]
    assert len(set(rows.tolist())) == len(rows)
    for t in range(T):
        for j in range(k):
            r = a["assign_row"][t, j]
            if r >= 0:
                assert used[r] == t


def test_padded_layout_rows():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((30, 4)).astype(np.float32)
    idx = O.select_topk(z, 2)
    C = O.capacity(1.0, 30, 2, 4)
    a = O.assign(idx, 4, C, O.LAYOUT_PADDED)
    b = O.assign(idx, 4, C, O.LAYOUT_COMPACT)
    assert a["rows"] == 4 * C
    for t in range(30):
        for j in range(2):
            e = idx[t, j]
            if b["assign_row"][t, j] < 0:
                assert a["assign_row"][t, j] == -1
            else:
                assert a["assign_row"][t, j] - e * C == b["assign_row"][t, j] - b["offsets"][e]
    with pytest.raises(ValueError):
        O.assign(idx, 4, None, O.LAYOUT_PADDED)


def test_capacity_values():
    assert O.capacity(1.25, 64, 2, 8) == 20
    assert O.capacity(1.0, 16384, 8, 256) == 512
    assert O.capacity(1.25, 8192, 2, 8) == 2560
    assert O.capacity(1.0, 10, 1, 3) == 4          # 10/3 rounded up
    assert O.capacity(0.01, 10, 1, 3) == 1         # never below one slot
    assert O.capacity(0.0, 10, 1, 3) is None
    assert O.capacity(-1.0, 10, 1, 3) is None


# ---------------------------------------------------------------- weights
def test_softmax_k_equals_E_is_full_softmax():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((20, 6)).astype(np.float32)
    idx = O.select_topk(z, 6)
    w = O.gate_weights(z, idx, O.SOFTMAX)
    full = scipy.special.softmax(z.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, idx.astype(np.int64), 1),
                               rtol=1e-14, atol=0)


def test_weights_sum_to_one_and_follow_rank():
    rng = np.random.default_rng(6)
    z = (rng.standard_normal((50, 16)) * 3).astype(np.float32)
    for gating in (O.SOFTMAX, O.SIGMOID):
        idx = O.select_topk(z, 4)
        w = O.gate_weights(z, idx, gating)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)
        assert (np.diff(w, axis=1) <= 1e-15).all()   # best pick weighs most


def test_sigmoid_matches_scipy_expit():
    rng = np.random.default_rng(8)
    z = (rng.standard_normal((10, 12)) * 4).astype(np.float32)
    idx = O.select_topk(z, 3)
    s = scipy.special.expit(np.take_along_axis(z.astype(np.float64), idx.astype(np.int64), 1))
    np.testing.assert_allclose(O.gate_weights(z, idx, O.SIGMOID), s / s.sum(1, keepdims=True),
                               rtol=1e-14)


# ---------------------------------------------------------------- logits
def test_router_logits_brute_force():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 5))
    wr = rng.standard_normal((5, 4))
    b = rng.standard_normal(4)
    z = O.router_logits(x, wr, b)
    for t in range(3):
        for e in range(4):
            ref = math.fsum(x[t, i] * wr[i, e] for i in range(5)) + b[e]
            assert z[t, e] == pytest.approx(ref, abs=1e-13)
    b2 = rng.standard_normal((3, 4))
    z2 = O.router_logits(x, wr, b2)
    np.testing.assert_allclose(z2 - b2, z - b, atol=1e-13)
    assert O.router_logits(np.eye(5)[:3], wr).tolist() == wr[:3].tolist()


def test_fp32_rounding_of_logits():
    z = np.array([[1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, -(1.0 + 2.0 ** -24)]])
    r = O.logits_to_fp32(z)
    assert r.dtype == np.float32
    assert r[0].tolist() == [1.0, 1.0 + 2.0 ** -22, -1.0]


# ---------------------------------------------------------------- FFN, combine, layer
def _dense_swiglu_torch(x, wg, wu, wd):
    xt = torch.from_numpy(np.asarray(x, dtype=np.float64))
    g = torch.nn.functional.linear(xt, torch.from_numpy(np.asarray(wg, dtype=np.float64)))
    u = torch.nn.functional.linear(xt, torch.from_numpy(np.asarray(wu, dtype=np.float64)))
    h = torch.nn.functional.silu(g) * u
    return torch.nn.functional.linear(h, torch.from_numpy(np.asarray(wd, dtype=np.float64))).numpy()


def test_single_expert_layer_is_dense_swiglu():
    rng = np.random.default_rng(10)
    T, d, f = 11, 16, 24
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((d, 1))
    wg = rng.standard_normal((1, f, d)) / 4
    wu = rng.standard_normal((1, f, d)) / 4
    wd = rng.standard_normal((1, d, f)) / 5
    for gating in (O.SOFTMAX, O.SIGMOID):
        r = O.moe_layer(x, wr, None, wg, wu, wd, k=1, gating=gating, capacity_factor=0.0)
        np.testing.assert_allclose(r["out"], _dense_swiglu_torch(x, wg[0], wu[0], wd[0]),
                                   rtol=1e-12, atol=1e-12)


def test_swiglu_operand_orientation():
    # non-square weights: a transposed operand cannot even be multiplied
    rng = np.random.default_rng(11)
    x = rng.standard_normal((2, 3))
    wg, wu, wd = rng.standard_normal((5, 3)), rng.standard_normal((5, 3)), rng.standard_normal((3, 5))
    h, y = O.swiglu_expert(x, wg, wu, wd)
    assert h.shape == (2, 5) and y.shape == (2, 3)
    # hand value: one input, one hidden unit
    h1, y1 = O.swiglu_expert([[2.0]], [[1.0]], [[3.0]], [[0.5]])
    silu2 = 2.0 / (1.0 + math.exp(-2.0))
    assert h1[0, 0] == pytest.approx(silu2 * 6.0, abs=1e-15)
    assert y1[0, 0] == pytest.approx(silu2 * 3.0, abs=1e-15)


def test_combine_one_hot_reproduces_rows():
    rng = np.random.default_rng(12)
    y = rng.standard_normal((6, 4))
    assign_row = np.array([[3, 1], [0, -1], [-1, -1]])
    w = np.array([[1.0, 0.0], [0.0, 1.0], [0.5, 0.5]])
    out = O.combine(y, assign_row, w)
    np.testing.assert_array_equal(out[0], y[3])
    np.testing.assert_array_equal(out[1], np.zeros(4))   # kept pick has weight 0, dropped pick ignored
    np.testing.assert_array_equal(out[2], np.zeros(4))   # fully dropped token
    w2 = np.array([[0.25, 0.75], [1.0, 0.3], [1.0, 1.0]])
    out2 = O.combine(y, assign_row, w2)
    np.testing.assert_allclose(out2[0], 0.25 * y[3] + 0.75 * y[1], atol=1e-15)
    np.testing.assert_allclose(out2[1], y[0], atol=1e-15)   # no renormalisation over survivors


def test_layer_equals_per_token_sum_of_experts():
    """Whole-layer output equals the per-token definition computed one token at a time."""
    shape = W.reduced(W.TINY_FP32, 24, 32, 48, capacity_factor=1.0)
    inp = W.make_inputs(shape)
    npx = lambda t: t.float().numpy()
    r = O.moe_layer(npx(inp.x), npx(inp.w_router), None, npx(inp.w_gate), npx(inp.w_up),
                    npx(inp.w_down), shape.k, shape.gating, shape.capacity_factor)
    toks = list(range(shape.T))
    o = O.token_outputs(toks, npx(inp.x), r["idx"], r["w"], r["assign_row"] >= 0,
                        lambda e: (npx(inp.w_gate[e]), npx(inp.w_up[e]), npx(inp.w_down[e])))
    np.testing.assert_allclose(r["out"], o, rtol=1e-12, atol=1e-12)
    assert r["stats"]["dropped"] > 0        # capacity 1.0 with a skewed router drops
    # each bucket's hidden rows are silu(x W_g^T) * (x W_u^T) of its tokens (torch's ops)
    for e in range(shape.E):
        lo, n = int(r["offsets"][e]), int(r["kept"][e])
        if n == 0:
            continue
        xt = torch.from_numpy(npx(inp.x)[r["token_of_row"][lo:lo + n]].astype(np.float64))
        g = torch.nn.functional.linear(xt, torch.from_numpy(npx(inp.w_gate[e]).astype(np.float64)))
        u = torch.nn.functional.linear(xt, torch.from_numpy(npx(inp.w_up[e]).astype(np.float64)))
        np.testing.assert_allclose(r["h_perm"][lo:lo + n],
                                   (torch.nn.functional.silu(g) * u).numpy(), rtol=1e-12,
                                   atol=1e-12)


def test_permute_fills_padding_rows_with_zeros():
    x = np.arange(6.0).reshape(3, 2) + 1.0
    xp = O.permute(x, np.array([2, -1, 0, -1]))
    assert xp.tolist() == [[5.0, 6.0], [0.0, 0.0], [1.0, 2.0], [0.0, 0.0]]


def test_routing_decision_is_taken_on_fp32_logits():
    # z64 = (1, 1 + 2^-30): expert 1 is larger in float64, but both round to 1.0f, and the
    # fp32 tie goes to the lower index
    x = np.array([[1.0]])
    wr = np.array([[1.0, 1.0 + 2.0 ** -30]])
    wg, wu, wd = np.ones((2, 1, 1)), np.ones((2, 1, 1)), np.ones((2, 1, 1))
    r = O.moe_layer(x, wr, None, wg, wu, wd, k=1, gating=O.SOFTMAX, capacity_factor=0.0)
    assert r["z32"].tolist() == [[1.0, 1.0]]
    assert r["idx"].tolist() == [[0]]
    assert r["z64"][0, 1] > r["z64"][0, 0]


def test_page_stats_example(golden_dir):
    with open(os.path.join(golden_dir, "page_stats_example.json")) as f:
        g = json.load(f)
    n = g["tokens_per_expert"]
    # the printed list is an excerpt of the layer's experts; max and max/mean over it are
    # what the page's record shows
    s = O.load_stats(n, n, np.zeros((1, 1), dtype=np.int64), None)
    assert s["max"] == g["expert_max"]
    assert round(s["max_to_mean"], g["printed_decimals"]) == g["expert_max_to_mean_printed"]
    assert s["mean"] == pytest.approx(sum(n) / len(n))


def test_percentiles_match_numpy_linear():
    rng = np.random.default_rng(13)
    for n in (1, 2, 4, 7, 256):
        v = rng.integers(0, 1000, size=n)
        for p in (0.5, 0.95, 0.99):
            assert O.percentile_linear(v, p) == pytest.approx(
                float(np.percentile(v, 100 * p, method="linear")), abs=1e-9)


def test_stats_top5_counts_experts():
    kept = list(range(40))          # E = 40 -> ceil(2.0) = 2 experts
    s = O.load_stats(kept, kept, np.zeros((10, 1), dtype=np.int64), None)
    assert s["top5pct_share"] == pytest.approx((39 + 38) / sum(kept))
    kept = [0] * 10
    s = O.load_stats(kept, kept, -np.ones((3, 2), dtype=np.int64), 0)
    assert s["top5pct_share"] == 0.0 and s["max_to_mean"] == 0.0
    assert s["tokens_fully_dropped"] == 3 and s["dropped_by_rank"] == [3, 3]


# ---------------------------------------------------------------- routing variants
def test_group_limited_hand_case():
    # 8 experts in 4 groups of 2: {0,1} {2,3} {4,5} {6,7}
    z = np.array([[5.0, 4.9, 0.0, 0.0, 4.95, 0.0, 4.8, 4.7]], dtype=np.float32)
    assert O.select_topk(z, 2).tolist() == [[0, 4]]                     # no group limit
    assert O.select_topk(z, 2, n_groups=4, topk_groups=1).tolist() == [[0, 1]]
    # groups 0 (5.0) and 2 (4.95) survive; group 3 (4.8) is out
    assert O.select_topk(z, 3, n_groups=4, topk_groups=2).tolist() == [[0, 4, 1]]
    # equal group scores -> lower group index
    z2 = np.array([[1.0, 0.0, 1.0, 0.5, 0.0, 0.0]], dtype=np.float32)
    assert O.select_topk(z2, 2, n_groups=3, topk_groups=1).tolist() == [[0, 1]]
    with pytest.raises(ValueError):
        O.select_topk(z, 3, n_groups=4, topk_groups=1)   # 1 group of 2 cannot hold 3 picks


@pytest.mark.parametrize("E,G,M,k", [(8, 4, 2, 2), (12, 3, 2, 4), (16, 8, 3, 3), (6, 2, 1, 3)])
def test_group_limited_brute_force(E, G, M, k):
    rng = np.random.default_rng(E + G + M + k)
    gs = E // G
    beats = lambda a, b, i, j: a > b or (a == b and i < j)
    for trial in range(30):
        z = (rng.integers(-2, 3, size=E) if trial % 2 else rng.standard_normal(E)).astype(np.float32)
        idx = O.select_topk(z[None], k, G, M)[0].tolist()
        gscore = [max(z[g * gs:(g + 1) * gs]) for g in range(G)]
        # the chosen groups: every chosen group beats every other group
        chosen = [g for g in range(G)
                  if sum(beats(gscore[h], gscore[g], h, g) for h in range(G) if h != g) < M]
        assert len(chosen) == M
        allowed = [e for e in range(E) if e // gs in chosen]
        sub = [float(z[e]) for e in allowed]
        want = [allowed[i] for i in _brute_topk(sub, k)]
        assert idx == want


def test_selection_only_bias_hand_case():
    z = np.array([[1.0, 2.0, 3.0]], dtype=np.float32)
    b = np.array([3.0, 0.0, 0.0], dtype=np.float32)
    r = O.route(z, 2, O.SOFTMAX, 0.0, bias=b, bias_mode=O.BIAS_SELECTION_ONLY)
    assert r["idx"].tolist() == [[0, 2]]          # scores 4, 2, 3
    e1, e3 = math.exp(1.0), math.exp(3.0)        # weights from the unbiased logits 1 and 3
    np.testing.assert_allclose(r["w"][0], [e1 / (e1 + e3), e3 / (e1 + e3)], rtol=0, atol=1e-15)
    # in the default mode the bias is already inside the logits: nothing added again
    r0 = O.route(z, 2, O.SOFTMAX, 0.0, bias=b, bias_mode=O.BIAS_SCORE_AND_WEIGHT)
    assert r0["idx"].tolist() == [[2, 1]]


def test_selection_only_bias_is_one_fp32_addition():
    z = np.array([[1.0, 1.0 + 2.0 ** -23]], dtype=np.float32)
    b = np.array([2.0 ** -24, 0.0], dtype=np.float32)    # 1 + 2^-24 rounds back to 1 in fp32
    s = O.selection_scores(z, b, O.BIAS_SELECTION_ONLY)
    assert s.dtype == np.float32 and s[0].tolist() == [1.0, 1.0 + 2.0 ** -23]
    assert O.select_topk(s, 1).tolist() == [[1]]


def test_pick_rank_drop_order_hand_case():
    idx = np.array([[0, 1], [1, 0], [0, 1]])
    tok = O.assign(idx, 2, 2, drop_policy=O.DROP_TOKEN_ORDER)
    rank = O.assign(idx, 2, 2, drop_policy=O.DROP_PICK_RANK)
    # expert 0 slots, token order: t0.j0, t1.j1, t2.j0 -> t2's first pick dropped
    assert tok["assign_row"].tolist() == [[0, 2], [3, 1], [-1, -1]]
    # pick rank: first picks t0->e0 s0, t1->e1 s0, t2->e0 s1; then second picks
    # t0->e1 s1, t1->e0 s2 (dropped), t2->e1 s2 (dropped); rows = offset (0 or 2) + slot
    assert rank["assign_row"].tolist() == [[0, 3], [2, -1], [1, -1]]
    assert rank["kept"].tolist() == [2, 2] and rank["routed"].tolist() == [3, 3]


@pytest.mark.parametrize("T,E,k,cf", [(60, 6, 2, 0.8), (45, 8, 3, 1.0), (30, 4, 4, 0.5)])
def test_pick_rank_slots_match_stable_sort(T, E, k, cf):
    rng = np.random.default_rng(T * k)
    z = rng.standard_normal((T, E)).astype(np.float32)
    z[:, 1] += 1.5
    idx = O.select_topk(z, k)
    C = O.capacity(cf, T, k, E)
    a = O.assign(idx, E, C, drop_policy=O.DROP_PICK_RANK)
    flat_e = idx.ravel().astype(np.int64)
    flat_t = np.repeat(np.arange(T), k)
    flat_j = np.tile(np.arange(k), T)
    order = np.argsort(flat_e * (k * T) + flat_j * T + flat_t, kind="stable")
    start = np.concatenate([[0], np.cumsum(np.bincount(flat_e, minlength=E))])
    slot = np.empty(T * k, dtype=np.int64)
    slot[order] = np.arange(T * k) - start[flat_e[order]]
    assert a["slot"].ravel().tolist() == slot.tolist()
    # no later pick is kept while an earlier-ranked pick to the same expert was dropped
    for e in range(E):
        for j in range(1, k):
            later_kept = ((idx[:, j] == e) & (a["assign_row"][:, j] >= 0)).any()
            earlier_dropped = ((idx[:, :j] == e) & (a["assign_row"][:, :j] < 0)).any()
            assert not (later_kept and earlier_dropped)


def test_score_drop_order_hand_case():
    # scores consistent with the picks: each row's picks are its top-2
    idx = np.array([[0, 1], [1, 0], [0, 1]])
    sc = np.array([[0.5, 0.2], [0.7, 0.9], [0.9, 0.1]], dtype=np.float32)
    a = O.assign(idx, 2, 2, drop_policy=O.DROP_SCORE, scores=sc)
    # expert 0 holds t0 (0.5), t1 (0.7), t2 (0.9): keeps t2 and t1, drops t0's first pick;
    # expert 1 holds t0 (0.2), t1 (0.9), t2 (0.1): keeps t1 and t0, drops t2's second pick.
    # Kept picks take rows in token order: e0 rows 0, 1 = t1, t2; e1 rows 2, 3 = t0, t1.
    assert a["assign_row"].tolist() == [[-1, 2], [3, 0], [1, -1]]
    assert a["token_of_row"].tolist() == [1, 2, 0, 1]
    assert a["kept"].tolist() == [2, 2] and a["routed"].tolist() == [3, 3]
    # dropless: every policy gives the token-order rows
    free = O.assign(idx, 2, None, drop_policy=O.DROP_SCORE, scores=sc)
    assert free["assign_row"].tolist() == O.assign(idx, 2, None)["assign_row"].tolist()
    # the second-choice counters of the same case
    c = O.pick_rank_counts(idx, a["assign_row"], 2)
    assert c["routed"].tolist() == [[2, 1], [1, 2]]
    assert c["kept"].tolist() == [[1, 1], [1, 1]]
    assert c["differs"].tolist() == [0, 3]
    assert c["dropped_share"] == [1 / 3, 1 / 3]
    assert c["differs_share"] == [0.0, 1.0]
    same = O.pick_rank_counts(idx, a["assign_row"], 2, group_of_expert=[0, 0])
    assert same["differs"].tolist() == [0, 0]


def test_score_drop_ties_signed_zero_and_nan():
    one = np.zeros((3, 1), dtype=np.int64)          # three tokens, one expert, k = 1
    def kept(scores, C):
        a = O.assign(one, 1, C, drop_policy=O.DROP_SCORE,
                     scores=np.array(scores, dtype=np.float32).reshape(3, 1))
        return [int(r >= 0) for r in a["assign_row"][:, 0]]
    assert kept([0.0, -0.0, 0.0], 1) == [1, 0, 0]          # -0 ties +0: lower token wins
    assert kept([-0.0, 0.0, 0.0], 2) == [1, 1, 0]
    assert kept([np.nan, 1.0, 1.0], 2) == [0, 1, 1]        # NaN ranks below every number
    assert kept([np.nan, -np.inf, np.nan], 2) == [1, 1, 0]
    assert kept([1.0, 2.0, 3.0], 0) == [0, 0, 0]


def test_score_drop_uses_selection_scores():
    # three tokens all pick expert 0 (C = ceil(0.5 * 3 * 1 / 2) = 1); with the
    # selection-only bias the priority is z + b: t0 (1 + 5) beats t2 (3 - 1) and t1 (2)
    z = np.array([[1.0, 0.0], [2.0, 0.0], [3.0, 0.0]], dtype=np.float32)
    b = np.array([[5.0, 0.0], [0.0, 0.0], [-1.0, 0.0]], dtype=np.float32)
    r = O.route(z, 1, O.SOFTMAX, 0.5, bias=b, bias_mode=O.BIAS_SELECTION_ONLY,
                drop_policy=O.DROP_SCORE)
    assert r["C"] == 1 and r["idx"][:, 0].tolist() == [0, 0, 0]
    assert r["assign_row"][:, 0].tolist() == [0, -1, -1]
    # the same logits without the bias keep the highest logit, t2
    r = O.route(z, 1, O.SOFTMAX, 0.5, drop_policy=O.DROP_SCORE)
    assert r["assign_row"][:, 0].tolist() == [-1, -1, 0]


def test_replica_stats_hand_case():
    # replica A: 3 tokens, both picks of token 2 over capacity 2; replica B: 1 token, C = 1
    a = (np.array([3, 3]), np.array([2, 2]), np.array([[0, 2], [1, 3], [-1, -1]]), 2)
    b = (np.array([1, 1]), np.array([1, 1]), np.array([[1, 0]]), 1)
    s = O.replica_load_stats([a, b])
    assert (s["active_tokens"], s["capacity"], s["routed_total"], s["kept_total"]) == (4, 3, 8, 6)
    assert (s["dropped"], s["tokens_with_drop"], s["tokens_fully_dropped"]) == (2, 1, 1)
    assert s["dropped_by_rank"] == [1, 1]
    assert (s["p50"], s["max"], s["mean"], s["max_to_mean"]) == (3.0, 3.0, 3.0, 1.0)
    assert (s["routed_max"], s["routed_max_to_mean"], s["top5pct_share"]) == (4.0, 1.0, 0.5)
    assert O.replica_load_stats([a, (b[0], b[1], b[2], None)])["capacity"] == -1


@pytest.mark.parametrize("parts", [1, 2, 5])
def test_replica_stats_of_a_dropless_split_equal_the_whole_batch(parts):
    rng = np.random.default_rng(parts)
    T, E, k = 103, 16, 4
    z = rng.standard_normal((T, E)).astype(np.float32)
    z[:, 3] += 1.0
    idx = O.select_topk(z, k)
    whole = O.assign(idx, E, None)
    cuts = np.linspace(0, T, parts + 1).astype(int)
    recs = []
    for lo, hi in zip(cuts, cuts[1:]):
        a = O.assign(idx[lo:hi], E, None)
        recs.append((a["routed"], a["kept"], a["assign_row"], None))
    got = O.replica_load_stats(recs)
    want = O.load_stats(whole["routed"], whole["kept"], whole["assign_row"], None)
    for key, val in want.items():
        assert got[key] == val, key


def test_hand_case_score_drops_and_counters(golden_dir):
    g = _hand(golden_dir)
    with open(os.path.join(golden_dir, "hand_e4_k2_t8_score_drops.json")) as f:
        want = json.load(f)
    z = np.array(g["logits"], dtype=np.float32)
    r = O.route(z, g["k"], O.SOFTMAX, g["capacity_factor"], drop_policy=O.DROP_SCORE)
    assert r["idx"].tolist() == want["idx"]
    assert r["assign_row"].tolist() == want["assign_row"]
    assert r["token_of_row"].tolist() == want["token_of_row"]
    assert r["kept"].tolist() == want["kept"]
    c = O.pick_rank_counts(r["idx"], r["assign_row"], g["E"])
    assert c["routed"].tolist() == want["routed_by_rank"]
    assert c["kept"].tolist() == want["kept_by_rank"]
    assert c["differs"].tolist() == want["differs_by_rank"]
    assert c["dropped_share"] == want["dropped_share_by_rank"]
