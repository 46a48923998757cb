"""Planted mistakes in the oracle, on the CPU: every mutant must fail the pin named beside it.

Each row below is a plausible slip in one line of `oracle/moe_oracle.py` or
`oracle/ep_oracle.py`: a dropped term, a flipped sign, a wrong index or axis, a transposed
operand, a changed rounding, tie or drop rule.  The test builds the mutant module from the
oracle's source with that one edit, points the pin's test module at it, runs the pin and
requires it to fail; the real oracle is never modified.  So the claim that the pins catch
any plausible mistake is checked, row by row, not just asserted.

Rewrites that cannot change a result are not rows: the padded layout's row count written as
offsets[E] (it equals E * C), and the selection score z + b added in float64 and then
rounded to float32 (fp32 addition is the correctly rounded exact sum).
"""
import contextlib
import os
import types

import pytest

import test_ep_oracle as TE
import test_oracle as TO
import test_oracle_properties as TP
from oracle import ep_oracle, moe_oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")
M, P = moe_oracle.__file__, ep_oracle.__file__
G = {"golden_dir": GOLDEN}

# (file, exact text, replacement, pin module, pin name, pin arguments, what the slip is)
ROWS = [
    # router scoring
    (M, "z = z + (b[None, :] if b.ndim == 1 else b)", "z = z",
     TO, "test_router_logits_brute_force", {}, "bias dropped"),
    (M, "z = z + (b[None, :] if b.ndim == 1 else b)", "z = z - (b[None, :] if b.ndim == 1 else b)",
     TO, "test_router_logits_brute_force", {}, "bias subtracted"),
    (M, "z = z + (b[None, :] if b.ndim == 1 else b)", "z = z + (b[None, :] if b.ndim == 1 else b.T)",
     TO, "test_router_logits_brute_force", {}, "per-token bias transposed"),
    (M, "z = x64 @ w64", "z = x64 @ (w64 * (1 + 1e-7))",
     TO, "test_router_logits_brute_force", {}, "logits scaled by 1 + 1e-7"),
    (M, "return np.asarray(z64, dtype=np.float64).astype(np.float32)",
     "return np.asarray(z64, dtype=np.float64).astype(np.float16).astype(np.float32)",
     TO, "test_fp32_rounding_of_logits", {}, "logits rounded through fp16"),
    (M, "        z32 = logits_to_fp32(z64)", "        z32 = np.asarray(z64, dtype=np.float64)",
     TO, "test_routing_decision_is_taken_on_fp32_logits", {}, "routing on unrounded logits"),
    # top-k
    (M, "order = np.lexsort((experts, -zt, ~eligible))", "order = np.lexsort((experts, zt, ~eligible))",
     TO, "test_hand_case_routing", G, "smallest scores picked"),
    (M, "order = np.lexsort((experts, -zt, ~eligible))", "order = np.lexsort((-experts, -zt, ~eligible))",
     TO, "test_hand_case_routing", G, "ties to the higher expert"),
    (M, "order = np.lexsort((experts, -zt, ~eligible))", "order = np.lexsort((experts, -zt))",
     TO, "test_group_limited_hand_case", {}, "group limit ignored"),
    (M, "gscore = zt.reshape(n_groups, gsize).max(axis=1)",
     "gscore = zt.reshape(n_groups, gsize).sum(axis=1)",
     TO, "test_group_limited_hand_case", {}, "group score summed"),
    (M, "gscore = zt.reshape(n_groups, gsize).max(axis=1)",
     "gscore = zt.reshape(gsize, n_groups).max(axis=0)",
     TO, "test_group_limited_hand_case", {}, "groups strided instead of contiguous"),
    (M, "gorder = np.lexsort((np.arange(n_groups), -gscore))",
     "gorder = np.lexsort((-np.arange(n_groups), -gscore))",
     TO, "test_group_limited_hand_case", {}, "group ties to the higher group"),
    (M, "for g in gorder[:topk_groups]:", "for g in gorder[:max(1, topk_groups - 1)]:",
     TO, "test_group_limited_hand_case", {}, "one group too few"),
    (M, "eligible[g * gsize:(g + 1) * gsize] = True", "eligible[g:g + gsize] = True",
     TO, "test_group_limited_hand_case", {}, "group slice offset"),
    # gate weights
    (M, "s = 1.0 / (1.0 + np.exp(-sel))", "s = 1.0 / (1.0 + np.exp(sel))",
     TO, "test_sigmoid_weights_hand_values", {}, "sigmoid sign"),
    (M, "return s / s.sum(axis=1, keepdims=True)", "return s",
     TO, "test_sigmoid_weights_hand_values", {}, "sigmoid not renormalised"),
    (M, "return e / e.sum(axis=1, keepdims=True)", "return e / e.sum(axis=0, keepdims=True)",
     TO, "test_hand_case_weights", G, "softmax over tokens"),
    (M, "e = np.exp(sel - m)", "e = np.exp(-(sel - m))",
     TO, "test_hand_case_weights", G, "softmax sign"),
    (M, "m = sel.max(axis=1, keepdims=True)", "m = sel.min(axis=1, keepdims=True)",
     TO, "test_softmax_weights_of_far_apart_logits", {}, "softmax shifted by the smallest pick"),
    (M, "sel = np.take_along_axis(z, np.asarray(idx, dtype=np.int64), axis=1)",
     "sel = -np.sort(-z, axis=1)[:, :np.asarray(idx).shape[1]]",
     TO, "test_sigmoid_weights_hand_values", {}, "weights of the largest logits, not the picks"),
    # capacity
    (M, "return int(math.ceil(float(capacity_factor) * T * k / E))",
     "return int(math.floor(float(capacity_factor) * T * k / E))",
     TO, "test_capacity_values", {}, "capacity floored"),
    (M, "return int(math.ceil(float(capacity_factor) * T * k / E))",
     "return int(math.ceil(float(capacity_factor) * T / E))",
     TO, "test_hand_case_routing", G, "capacity without k"),
    (M, "if capacity_factor <= 0:", "if capacity_factor < 0:",
     TO, "test_capacity_values", {}, "cf = 0 not dropless"),
    (M, "    C = capacity(capacity_factor, T, k, E)", "    C = capacity(capacity_factor, T, k, E + 1)",
     TO, "test_hand_case_score_drops_and_counters", G, "capacity over E + 1 experts"),
    # assignment, drops, layout
    (M, "walk = [(t, j) for j in range(k) for t in range(T)]",
     "walk = [(t, j) for t in range(T) for j in range(k)]",
     TO, "test_pick_rank_drop_order_hand_case", {}, "pick-rank policy walks tokens"),
    (M, "kept = routed.copy() if C is None else np.minimum(routed, C)",
     "kept = routed.copy() if C is None else np.minimum(routed, C - 1)",
     TO, "test_hand_case_routing", G, "one row fewer than C kept"),
    (M, "return (1 if v != v else 0, -v if v == v else 0.0, tj[0])",
     "return (1 if v != v else 0, v if v == v else 0.0, tj[0])",
     TO, "test_score_drop_order_hand_case", {}, "lowest scores kept"),
    (M, "return (1 if v != v else 0, -v if v == v else 0.0, tj[0])",
     "return (1 if v != v else 0, -v if v == v else 0.0, -tj[0])",
     TO, "test_score_drop_ties_signed_zero_and_nan", {}, "score ties to the higher token"),
    (M, "return (1 if v != v else 0, -v if v == v else 0.0, tj[0])",
     "return (0, -v if v == v else 0.0, tj[0])",
     TO, "test_score_drop_ties_signed_zero_and_nan", {}, "NaN not ranked lowest"),
    (M, "is_kept = (pos < C) if C is not None", "is_kept = (pos <= C) if C is not None",
     TO, "test_score_drop_order_hand_case", {}, "C + 1 kept under score drops"),
    (M, "                    pos[t, j] = next_slot[e]\n                    next_slot[e] += 1",
     "                    pass",
     TO, "test_score_drop_order_hand_case", {}, "kept picks keep their priority rank as row"),
    (M, "offsets[e] = e * C", "offsets[e] = e * (C + 1)",
     TO, "test_hand_case_routing", G, "padded bucket stride"),
    (M, "                token_of_row[r] = t", "                token_of_row[r] = j",
     TO, "test_hand_case_routing", G, "token_of_row holds the pick rank"),
    (M, "                r = offsets[e] + pos[t, j]",
     "                r = offsets[e] + pos[t, j] + (1 if pos[t, j] > 0 and e == 0 else 0)",
     TO, "test_hand_case_routing", G, "row off by one in bucket 0"),
    # permute, expert FFN, combine
    (M, "out[used] = x64[token_of_row[used]]",
     "out[used] = x64[np.nonzero(used)[0] % x64.shape[0]]",
     TO, "test_layer_equals_per_token_sum_of_experts", {}, "rows not permuted"),
    (M, "    out = np.zeros((len(token_of_row), x64.shape[1]), dtype=np.float64)",
     "    out = np.ones((len(token_of_row), x64.shape[1]), dtype=np.float64)",
     TO, "test_permute_fills_padding_rows_with_zeros", {}, "padding rows not zero"),
    (M, "return u / (1.0 + np.exp(-u))", "return u / (1.0 + np.exp(u))",
     TO, "test_single_expert_layer_is_dense_swiglu", {}, "silu sign"),
    (M, "return u / (1.0 + np.exp(-u))", "return 1.0 / (1.0 + np.exp(-u))",
     TO, "test_single_expert_layer_is_dense_swiglu", {}, "sigmoid in place of silu"),
    (M, "h = silu(g) * u", "h = silu(u) * g",
     TO, "test_single_expert_layer_is_dense_swiglu", {}, "gate and up swapped"),
    (M, "h = silu(g) * u", "h = g * u",
     TO, "test_single_expert_layer_is_dense_swiglu", {}, "no activation"),
    (M, "y = h @ np.asarray(w_down_e, dtype=np.float64).T",
     "y = (h @ np.asarray(w_down_e, dtype=np.float64).T) * 1.0001",
     TO, "test_single_expert_layer_is_dense_swiglu", {}, "down projection scaled"),
    (M, "h, y = swiglu_expert(x_perm[s:s + n], wg, wu, wd)",
     "h, y = swiglu_expert(x_perm[s:s + n], *expert_weights(max(e - 1, 0)))",
     TO, "test_layer_equals_per_token_sum_of_experts", {}, "bucket run with the previous expert"),
    (M, "        h_perm[s:s + n] = h\n",
     "        h_perm[s:s + n] = h + (1e-3 if e == 1 else 0)\n",
     TO, "test_layer_equals_per_token_sum_of_experts", {}, "hidden rows of one expert off"),
    (M, "out[t] += weights[t, j] * y[r]", "out[t] += weights[t, 0] * y[r]",
     TO, "test_combine_one_hot_reproduces_rows", {}, "combine uses the first weight"),
    (M, "            if r >= 0:\n                out[t] += weights[t, j] * y[r]",
     "            out[t] += weights[t, j] * y[r]",
     TO, "test_combine_one_hot_reproduces_rows", {}, "dropped picks combined"),
    (M, "term = w_rows[i, j] * y[0]", "term = w_rows[i, 0] * y[0]",
     TO, "test_layer_equals_per_token_sum_of_experts", {}, "per-token output uses one weight"),
    (M, "            if not kept_rows[i, j]:\n                continue", "            pass",
     TO, "test_layer_equals_per_token_sum_of_experts", {}, "per-token output keeps drops"),
    # load statistics
    (M, "h = (n - 1) * p", "h = n * p if n * p < n - 1 else (n - 1) * p",
     TO, "test_hand_case_stats", G, "percentile position n p"),
    (M, "return s[lo] + (h - lo) * (s[hi] - s[lo])", "return s[lo]",
     TO, "test_hand_case_stats", G, "percentile not interpolated"),
    (M, "n_top = int(math.ceil(0.05 * E))", "n_top = max(1, int(0.05 * E))",
     TO, "test_top5pct_share_counts_ceil_of_five_percent", {}, "top-5% count floored"),
    (M, "tokens_fully_dropped=int((drops_per_token == k).sum())",
     "tokens_fully_dropped=int((drops_per_token >= 1).sum())",
     TO, "test_hand_case_stats", G, "fully dropped = any drop"),
    (M, "tokens_with_drop=int((drops_per_token > 0).sum())",
     "tokens_with_drop=int((drops_per_token > 1).sum())",
     TO, "test_hand_case_stats", G, "tokens with a drop need two"),
    (M, "p99=percentile_linear(kept, 0.99)", "p99=percentile_linear(kept, 0.95)",
     TO, "test_hand_case_stats", G, "p99 is p95"),
    (M, "max_to_mean=(mx / mean) if mean > 0 else 0.0",
     "max_to_mean=(mx / (sum(routed) / E)) if mean > 0 else 0.0",
     TO, "test_hand_case_stats", G, "max/mean over routed counts"),
    (M, "dropped_by_rank = [int((assign_row[:, j] < 0).sum()) for j in range(k)]",
     "dropped_by_rank = [int((assign_row[:, k - 1 - j] < 0).sum()) for j in range(k)]",
     TO, "test_hand_case_stats", G, "drops by pick rank reversed"),
    (M, "routed_max_to_mean=(max(routed) / routed_mean)",
     "routed_max_to_mean=(max(kept) / routed_mean)",
     TO, "test_hand_case_stats", G, "routed max from kept counts"),
    (M, "capacity=-1 if C is None else int(C)", "capacity=0 if C is None else int(C)",
     TO, "test_replica_stats_hand_case", {}, "dropless capacity recorded as 0"),
    (M, "active_tokens=T,", "active_tokens=T * k,",
     TO, "test_replica_stats_hand_case", {}, "active tokens counts picks"),
    (M, "C = None if any(c is None for c in caps) else int(sum(caps))",
     "C = None if any(c is None for c in caps) else int(max(caps))",
     TO, "test_replica_stats_hand_case", {}, "job capacity = largest replica's"),
    (M, "C = None if any(c is None for c in caps) else int(sum(caps))",
     "C = None if all(c is None for c in caps) else int(sum(c or 0 for c in caps))",
     TO, "test_replica_stats_hand_case", {}, "job dropless only if all replicas are"),
    (M, "    rows = np.vstack([np.asarray(p[2]) for p in parts])",
     "    rows = np.asarray(parts[0][2])",
     TO, "test_replica_stats_hand_case", {}, "job record from the first replica's picks"),
    # routing variants and the second-choice counters
    (M, "    return (z32 + (b[None, :] if b.ndim == 1 else b)).astype(np.float32)",
     "    return (z32 - (b[None, :] if b.ndim == 1 else b)).astype(np.float32)",
     TO, "test_selection_only_bias_hand_case", {}, "selection bias subtracted"),
    (M, "w = gate_weights(z32, idx, gating)", "w = gate_weights(sel, idx, gating)",
     TO, "test_selection_only_bias_hand_case", {}, "weights from the biased scores"),
    (M, "z64 = router_logits(x, w_router, None if sel_only else logit_bias)",
     "z64 = router_logits(x, w_router, logit_bias)",
     TE, "test_ep_layer_with_routing_variants_equals_local_layer",
     {"variant": dict(bias_mode=moe_oracle.BIAS_SELECTION_ONLY)},
     "selection-only bias added to the logits"),
    (M, "if grp[e] != grp[int(idx[t, 0])]:", "if grp[e] != grp[int(idx[t, max(j - 1, 0)])]:",
     TP, "test_score_drop_invariants", {}, "differs compared with the previous pick"),
    (M, "if ar[t, j] >= 0:\n                kept[j, e] += 1", "if ar[t, j] > 0:\n                kept[j, e] += 1",
     TO, "test_score_drop_order_hand_case", {}, "row 0 not counted as kept"),
    (M, "dropped_share=[share(T - int(kept[j].sum())) for j in range(k)]",
     "dropped_share=[share(T - int(routed[j].sum())) for j in range(k)]",
     TO, "test_score_drop_order_hand_case", {}, "dropped share from routed counts"),
    (M, "differs_share=[share(int(n)) for n in differs]",
     "differs_share=[share(int(n)) for n in differs[::-1]]",
     TO, "test_score_drop_order_hand_case", {}, "differs share reversed"),
    # expert parallelism
    (P, "return np.arange(E) // per", "return np.arange(E) % (E // per)",
     TE, "test_contiguous_placement_values", {}, "round-robin placement"),
    (P, "    return np.nonzero(np.asarray(expert_rank) == g)[0]",
     "    return np.nonzero(np.asarray(expert_rank) == g)[0][::-1]",
     TE, "test_hand_case_layout_and_stats", {}, "local experts descending"),
    (P, "            for s in range(G):\n                base[s, e] = pos",
     "            for s in reversed(range(G)):\n                base[s, e] = pos",
     TE, "test_hand_case_layout_and_stats", {}, "sources descending in a bucket"),
    (P, "out[t, j] = b[e] + (a[t, j] - off[e])", "out[t, j] = b[e] + a[t, j]",
     TE, "test_ep_layer_equals_local_layer_per_rank",
     dict(G=2, E=4, k=2, cf=1.0, permuted=False), "send row without the bucket offset"),
    (P, "            e = mine[i]", "            e = int(mine[0]) + i",
     TE, "test_ep_layer_equals_local_layer_per_rank",
     dict(G=4, E=8, k=2, cf=1.25, permuted=True), "local expert i taken as a block index"),
    (P, "recv[er[r[\"idx\"][t, j]]][sr[t, j]] = x64[t]",
     "recv[er[r[\"idx\"][t, j]]][sr[t, j]] = x64[min(t + (1 if s == 1 else 0), T - 1)]",
     TE, "test_ep_layer_equals_local_layer_per_rank",
     dict(G=2, E=4, k=2, cf=1.0, permuted=False), "a rank sends the next token's row"),
    (P, "acc = acc + r[\"w\"][t, j] * y_recv[er[r[\"idx\"][t, j]]][sr[t, j]]",
     "acc = acc + r[\"w\"][t, 0] * y_recv[er[r[\"idx\"][t, j]]][sr[t, j]]",
     TE, "test_ep_layer_equals_local_layer_per_rank",
     dict(G=2, E=4, k=2, cf=1.0, permuted=False), "EP combine uses the first weight"),
    (P, "if z32s is None else np.asarray(z32s[s], dtype=np.float32))",
     "if z32s is None else np.asarray(z32s[0], dtype=np.float32))",
     TE, "test_ep_layer_from_given_logits_uses_each_ranks_own", {}, "rank 0's logits for all"),
    (P, "pair_rows[s, er[e]] += kept[s, e]", "pair_rows[er[e], s] += kept[s, e]",
     TE, "test_hand_case_layout_and_stats", {}, "pair matrix transposed"),
    (P, "local = int(np.trace(pair_rows))", "local = 0",
     TE, "test_hand_case_layout_and_stats", {}, "local assignments not counted"),
    (P, "cross = sum(int(pair_bytes[s, g]) for s in range(G) for g in range(G)\n"
        "                if s != g and node[s] != node[g])",
     "cross = sum(int(pair_bytes[s, g]) for s in range(G) for g in range(G)\n"
     "                if s != g)",
     TE, "test_hand_case_layout_and_stats", {}, "every remote byte counted as crossing"),
    (P, "off_diag = [int(pair_bytes[s, g]) for s in range(G) for g in range(G) if s != g]",
     "off_diag = [int(pair_bytes[s, g]) for s in range(G) for g in range(G)"
     " if s != g and pair_bytes[s, g] > 0]",
     TE, "test_hand_case_with_empty_pairs", {}, "empty pairs left out of the percentiles"),
    (P, "node = [r // ranks_per_node for r in range(G)]", "node = [r % ranks_per_node for r in range(G)]",
     TE, "test_hand_case_layout_and_stats", {}, "node of a rank by modulo"),
    (P, "    n_nodes = (G + ranks_per_node - 1) // ranks_per_node",
     "    n_nodes = max(1, G // ranks_per_node)",
     TE, "test_hand_case_with_empty_pairs", {}, "partial node not counted"),
    (P, "rank_load_max_minus_mean=max(rank_load) - mean_load",
     "rank_load_max_minus_mean=max(rank_load) - min(rank_load)",
     TE, "test_hand_case_layout_and_stats", {}, "busiest minus least busy rank"),
    (P, "node_load_max_to_mean=(max(node_load) / mean_node) if mean_node else 0.0,",
     "node_load_max_to_mean=(max(node_load) / mean_load) if mean_node else 0.0,",
     TE, "test_hand_case_layout_and_stats", {}, "node max over the rank mean"),
    (P, "pair_bytes_p99=O.percentile_linear(off_diag, 0.99) if off_diag else 0.0,",
     "pair_bytes_p99=O.percentile_linear(off_diag, 0.95) if off_diag else 0.0,",
     TE, "test_hand_case_layout_and_stats", {}, "pair p99 is p95"),
    (P, "bytes_recv=[int(pair_bytes[:, g].sum() - pair_bytes[g, g]) for g in range(G)]",
     "bytes_recv=[int(pair_bytes[g, :].sum() - pair_bytes[g, g]) for g in range(G)]",
     TE, "test_hand_case_layout_and_stats", {}, "received bytes read as sent"),
]


def _module(name, path, src):
    mod = types.ModuleType(name)
    mod.__file__ = path
    exec(compile(src, path, "exec"), mod.__dict__)
    return mod


@contextlib.contextmanager
def _mutant(path, old, new):
    srcs = {}
    for p in (M, P):
        with open(p) as f:
            srcs[p] = f.read()
    n = srcs[path].count(old)
    assert n == 1, f"the mutated text occurs {n} times in {os.path.basename(path)}"
    srcs[path] = srcs[path].replace(old, new)
    mo = _module("oracle.moe_oracle", M, srcs[M])
    ep = _module("oracle.ep_oracle", P, srcs[P])
    ep.O = mo                          # the EP oracle calls the (mutant) single-GPU oracle
    saved = (TO.O, TP.O, TE.O, TE.EP)
    TO.O = TP.O = TE.O = mo
    TE.EP = ep
    try:
        yield
    finally:
        TO.O, TP.O, TE.O, TE.EP = saved


@pytest.mark.filterwarnings("ignore::RuntimeWarning")   # some mutants overflow on purpose
@pytest.mark.parametrize("row", ROWS, ids=[r[-1].replace(" ", "_") for r in ROWS])
def test_pin_catches_planted_mistake(row):
    path, old, new, mod, name, kwargs, _what = row
    pin = getattr(mod, name)
    with _mutant(path, old, new):
        with pytest.raises(Exception):
            pin(**kwargs)


def test_unmutated_oracle_passes_every_named_pin():
    """The same harness with no edit: each pin passes, so a failure above is the mutant's."""
    seen = set()
    for path, old, _new, mod, name, kwargs, _what in ROWS:
        key = (mod.__name__, name, repr(sorted(kwargs.items())))
        if key in seen:
            continue
        seen.add(key)
        with _mutant(path, old, old):
            getattr(mod, name)(**kwargs)
