"""CPU oracle for one Mixture-of-Experts layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this module.  The product path (the C-ABI library and its Python binding) never
imports, links or calls it, and it imports nothing from the product.

What it computes is the plain definition of the layer, in float64, step by step, in the
order the pages describe it:

  router scores -> top-k experts per token -> gate weights renormalised over the k picks
  -> per-expert capacity with overflow dropped (or padded) -> dispatch into expert-major
  buckets -> per-expert SwiGLU FFN -> gate-weighted combine back to token order
  -> per-layer load statistics.

Sources (page title, section):
  [EP-serving]  "Expert Parallelism for MoE Serving" (aiunderstanding.org), sections
                "Deep dive" (router picks top-k, often 1 or 2, per token; dispatch and
                combine all-to-alls) and "Technical insight" (capacity factors, expert
                buffers, dropping or padding tokens to keep GEMM shapes uniform); FAQ
                (capacity = max tokens per expert, pad or drop past it).
  [EP-checks]   "MoE expert parallelism needs measurements before launch" (airouter.kz),
                sections "Mean expert load proves almost nothing" (mu = sum n_e / E; the
                per-layer record tokens_per_expert, expert_p50, expert_p95, expert_max,
                expert_max_to_mean, top_5_percent_expert_share, dropped_tokens),
                "Capacity factor changes quality, memory and the latency tail" (top-1
                capacity = mean tokens per expert x factor, rounding engine-specific;
                overflow dropped; drop_tokens=false = unlimited capacity; drop rate per
                layer and per route top-1/top-2), "Profile all-to-all separately from
                compute" (router -> pack/permute -> dispatch -> expert -> combine ->
                unpack; EP=1 keeps experts local with no all-to-all).

Readings taken where the pages are silent (each one is listed in the design notes):
  * capacity C = ceil(cf * T * k / E) for cf > 0 (mean assignments per expert times the
    factor, rounded up); cf <= 0 means dropless (no limit);
  * top-k orders experts by the fp32 logit, descending, equal logits -> lower expert index;
  * the logit bias is added before selection and before the gate weights;
  * softmax gate: exp(z_j - z_max) / sum over the k picks; sigmoid gate: s(z_j) / sum of s
    over the k picks;
  * overflow: within each expert, assignments are kept in token order (lower token index
    first); the first C are kept, the rest dropped;
  * COMPACT layout: expert buckets packed back to back; PADDED: bucket e starts at e*C;
  * combine sums the kept picks in pick order; a dropped pick contributes 0 and the
    remaining weights are NOT renormalised;
  * tokens_per_expert = kept counts; percentiles = linear interpolation (type 7) over all
    E experts including empty ones; top-5% share = sum of the ceil(0.05 E) largest kept
    counts over the total; dropped_tokens counts dropped (token, expert) assignments.
  Routing variants ([EP-serving] "Real-world implementation": node-limited routing;
  "Future": loss-free balancing; [EP-checks] "Top-2 does not insure against hot experts"):
  * group-limited: experts form n_groups equal contiguous groups, a group's score is its
    best selection score, a token keeps the topk_groups best groups (equal scores -> lower
    group index) and picks its k experts among them;
  * selection-only bias: selection on fp32(z + b), gate weights from the unbiased z;
  * pick-rank drop order: within an expert, all first picks (token order), then all second
    picks, and so on;
  * score drop order: an expert keeps the C picks with the highest fp32 selection score
    (equal scores -> lower token; NaN below every number); its kept picks take slots in
    token order;
  * second-choice counters ([EP-checks] "Top-2 does not insure against hot experts"): per
    pick rank and expert the assignments and the kept assignments, and per pick rank the
    tokens whose pick lies in another group than their first pick, a group being any
    caller-given map of experts (the experts themselves, routing groups, owner ranks or
    nodes).

Every function below is pinned by tests in tests/test_oracle.py against hand-worked
cases, brute force, closed forms or independent textbook routines.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional, Tuple

import numpy as np

SOFTMAX = 0
SIGMOID = 1
LAYOUT_COMPACT = 0
LAYOUT_PADDED = 1
BIAS_SCORE_AND_WEIGHT = 0
BIAS_SELECTION_ONLY = 1
DROP_TOKEN_ORDER = 0
DROP_PICK_RANK = 1
DROP_SCORE = 2


# --------------------------------------------------------------------------------------
# Router scoring  [EP-serving, "Deep dive": a router scores every expert for each token]
# --------------------------------------------------------------------------------------
def router_logits(x, w_router, logit_bias=None) -> np.ndarray:
    """z64[t, e] = sum_i x[t, i] * W_r[i, e] + b[t, e], in float64.

    x: [T, d]; w_router: [d, E]; logit_bias: None, [E] (same for every token) or [T, E].
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    z = x64 @ w64
    if logit_bias is not None:
        b = np.asarray(logit_bias, dtype=np.float64)
        z = z + (b[None, :] if b.ndim == 1 else b)
    return z


def logits_to_fp32(z64) -> np.ndarray:
    """Round the float64 logits to float32 (round to nearest even): the precision in
    which the routing decision is taken."""
    return np.asarray(z64, dtype=np.float64).astype(np.float32)


# --------------------------------------------------------------------------------------
# Top-k selection  [EP-serving, "Deep dive": router picks the top-k experts per token]
# --------------------------------------------------------------------------------------
def select_topk(z32, k: int, n_groups: int = 0, topk_groups: int = 0) -> np.ndarray:
    """idx[t, 0..k-1]: the k experts with the largest fp32 score, best first; equal
    scores rank the lower expert index first.  With n_groups > 1, only the experts of the
    token's topk_groups best groups (group score = best score in the group, equal group
    scores -> lower group index) are eligible."""
    z = np.asarray(z32, dtype=np.float32)
    T, E = z.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    grouped = n_groups > 1
    if grouped:
        if E % n_groups or not (1 <= topk_groups <= n_groups) or topk_groups * (E // n_groups) < k:
            raise ValueError("bad group configuration")
        gsize = E // n_groups
    idx = np.empty((T, k), dtype=np.int32)
    experts = np.arange(E)
    for t in range(T):
        zt = z[t].astype(np.float64)
        eligible = np.ones(E, dtype=bool)
        if grouped:
            gscore = zt.reshape(n_groups, gsize).max(axis=1)
            gorder = np.lexsort((np.arange(n_groups), -gscore))
            eligible[:] = False
            for g in gorder[:topk_groups]:
                eligible[g * gsize:(g + 1) * gsize] = True
        # lexsort: last key is primary -> eligible first, then by -z, then by expert index
        order = np.lexsort((experts, -zt, ~eligible))
        idx[t] = order[:k]
    return idx


def gate_weights(z32, idx, gating: int) -> np.ndarray:
    """Gate weight of each pick, renormalised over the k picks, float64 from the fp32
    logits.  Softmax: exp(z_j - m) / sum_i exp(z_i - m) with m the largest picked logit.
    Sigmoid: s(z_j) / sum_i s(z_i), s(u) = 1 / (1 + exp(-u))."""
    z = np.asarray(z32, dtype=np.float32).astype(np.float64)
    sel = np.take_along_axis(z, np.asarray(idx, dtype=np.int64), axis=1)
    if gating == SOFTMAX:
        m = sel.max(axis=1, keepdims=True)
        e = np.exp(sel - m)
        return e / e.sum(axis=1, keepdims=True)
    if gating == SIGMOID:
        s = 1.0 / (1.0 + np.exp(-sel))
        return s / s.sum(axis=1, keepdims=True)
    raise ValueError("unknown gating")


# --------------------------------------------------------------------------------------
# Capacity  [EP-checks, "Capacity factor ...": capacity = mean tokens/expert x factor;
#            drop_tokens=false = unlimited]
# --------------------------------------------------------------------------------------
def capacity(capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
    """C = ceil(cf * T * k / E) for cf > 0; None (no limit) for cf <= 0."""
    if capacity_factor <= 0:
        return None
    return int(math.ceil(float(capacity_factor) * T * k / E))


# --------------------------------------------------------------------------------------
# Dispatch bookkeeping  [EP-serving, "Technical insight": expert buffers, drop or pad;
#                        EP-checks, "Profile all-to-all ...": pack/permute before dispatch]
# --------------------------------------------------------------------------------------
def assign(idx, E: int, C: Optional[int], layout: int = LAYOUT_COMPACT,
           drop_policy: int = DROP_TOKEN_ORDER, scores=None) -> Dict[str, np.ndarray]:
    """Walk the assignments in (expert ascending, token ascending) order, which for a
    top-k (distinct experts per token) is the same as walking tokens in order and giving
    each pick the next free slot of its expert.  With drop_policy = DROP_PICK_RANK the walk
    goes pick rank by pick rank (all first picks in token order, then all second picks...).
    Slot pos < C is kept, the rest dropped.
    With drop_policy = DROP_SCORE the walk only decides which picks are kept: each
    expert keeps the C picks with the highest fp32 selection score scores[t, e] (equal
    scores: lower token first; a NaN score below every number), and its kept picks then
    take slots 0, 1, ... in token order, so that without overflow the rows are those of
    the token-order policy.

    Returns routed[E], kept[E], offsets[E+1] (bucket starts), assign_row[T, k]
    (-1 = dropped), token_of_row[rows] (-1 = unused padding row) and rows.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    if layout == LAYOUT_PADDED and C is None:
        raise ValueError("PADDED layout needs a finite capacity")
    pos = np.full((T, k), -1, dtype=np.int64)
    next_slot = [0] * E
    if drop_policy == DROP_PICK_RANK:
        walk = [(t, j) for j in range(k) for t in range(T)]
    elif drop_policy == DROP_SCORE:
        if scores is None:
            raise ValueError("DROP_SCORE needs the selection scores")
        sc = np.asarray(scores, dtype=np.float32)

        def order(tj):
            v = float(sc[tj[0], idx[tj[0], tj[1]]])
            return (1 if v != v else 0, -v if v == v else 0.0, tj[0])

        walk = sorted(((t, j) for t in range(T) for j in range(k)), key=order)
    else:
        walk = [(t, j) for t in range(T) for j in range(k)]
    for t, j in walk:
        e = int(idx[t, j])
        pos[t, j] = next_slot[e]
        next_slot[e] += 1
    routed = np.array(next_slot, dtype=np.int64)
    kept = routed.copy() if C is None else np.minimum(routed, C)
    if drop_policy == DROP_SCORE:
        # priority rank -> kept or not; kept picks re-slotted in token order (a dropped
        # pick keeps its priority rank, >= C)
        is_kept = (pos < C) if C is not None else np.ones_like(pos, dtype=bool)
        next_slot = [0] * E
        for t in range(T):
            for j in range(k):
                if is_kept[t, j]:
                    e = int(idx[t, j])
                    pos[t, j] = next_slot[e]
                    next_slot[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    if layout == LAYOUT_COMPACT:
        for e in range(E):
            offsets[e + 1] = offsets[e] + kept[e]
        rows = int(offsets[E])
    else:
        for e in range(E + 1):
            offsets[e] = e * C
        rows = E * C
    assign_row = np.full((T, k), -1, dtype=np.int64)
    token_of_row = np.full(rows, -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if C is None or pos[t, j] < C:
                r = offsets[e] + pos[t, j]
                assign_row[t, j] = r
                token_of_row[r] = t
    return dict(routed=routed, kept=kept, offsets=offsets, assign_row=assign_row,
                token_of_row=token_of_row, rows=rows, slot=pos)


def permute(x, token_of_row) -> np.ndarray:
    """x_perm[r] = x[token_of_row[r]] for used rows; padding rows are zero."""
    x64 = np.asarray(x, dtype=np.float64)
    out = np.zeros((len(token_of_row), x64.shape[1]), dtype=np.float64)
    used = token_of_row >= 0
    out[used] = x64[token_of_row[used]]
    return out


# --------------------------------------------------------------------------------------
# Expert FFN  [EP-checks: "expert MLP"; SwiGLU experts of Mixtral / DeepSeek-V3]
# --------------------------------------------------------------------------------------
def silu(u):
    return u / (1.0 + np.exp(-u))


def swiglu_expert(x_rows, w_gate_e, w_up_e, w_down_e) -> Tuple[np.ndarray, np.ndarray]:
    """h = silu(x W_g^T) * (x W_u^T), y = h W_d^T, all float64.  Weights are stored
    out x in: W_g, W_u [f, d]; W_d [d, f].  Returns (h, y)."""
    xr = np.asarray(x_rows, dtype=np.float64)
    g = xr @ np.asarray(w_gate_e, dtype=np.float64).T
    u = xr @ np.asarray(w_up_e, dtype=np.float64).T
    h = silu(g) * u
    y = h @ np.asarray(w_down_e, dtype=np.float64).T
    return h, y


def expert_ffn(x_perm, offsets, kept, expert_weights: Callable[[int], tuple]):
    """Run every expert on its bucket rows [offsets[e], offsets[e] + kept[e]).
    expert_weights(e) -> (W_g[e], W_u[e], W_d[e]).  Returns (h_perm, y_perm); rows outside
    every bucket stay zero."""
    x_perm = np.asarray(x_perm, dtype=np.float64)
    E = len(kept)
    h_perm = None
    y_perm = np.zeros_like(x_perm)
    for e in range(E):
        n = int(kept[e])
        if n == 0:
            continue
        s = int(offsets[e])
        wg, wu, wd = expert_weights(e)
        h, y = swiglu_expert(x_perm[s:s + n], wg, wu, wd)
        if h_perm is None:
            h_perm = np.zeros((x_perm.shape[0], h.shape[1]), dtype=np.float64)
        h_perm[s:s + n] = h
        y_perm[s:s + n] = y
    return h_perm, y_perm


# --------------------------------------------------------------------------------------
# Combine  [EP-serving, "Deep dive": results shuffled back; EP-checks: combine + unpack]
# --------------------------------------------------------------------------------------
def combine(y_perm, assign_row, weights) -> np.ndarray:
    """out[t] = sum over kept picks j (in pick order) of w[t, j] * y_perm[assign_row[t, j]]."""
    y = np.asarray(y_perm, dtype=np.float64)
    T, k = assign_row.shape
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            r = int(assign_row[t, j])
            if r >= 0:
                out[t] += weights[t, j] * y[r]
    return out


# --------------------------------------------------------------------------------------
# Load statistics  [EP-checks, "Mean expert load proves almost nothing"; "Capacity
#                   factor ...": drop rate per layer and per route]
# --------------------------------------------------------------------------------------
def percentile_linear(values, p: float) -> float:
    """Linear-interpolation percentile (type 7): sort ascending, h = (n-1) p,
    v = s[floor h] + (h - floor h) (s[floor h + 1] - s[floor h])."""
    s = sorted(float(v) for v in values)
    n = len(s)
    h = (n - 1) * p
    lo = int(math.floor(h))
    hi = min(lo + 1, n - 1)
    return s[lo] + (h - lo) * (s[hi] - s[lo])


def load_stats(routed, kept, assign_row, C: Optional[int]) -> dict:
    routed = [int(v) for v in routed]
    kept = [int(v) for v in kept]
    E = len(kept)
    T, k = assign_row.shape
    total_kept = sum(kept)
    mean = total_kept / E
    mx = max(kept)
    routed_mean = sum(routed) / E
    n_top = int(math.ceil(0.05 * E))
    top = sorted(kept, reverse=True)[:n_top]
    dropped_by_rank = [int((assign_row[:, j] < 0).sum()) for j in range(k)]
    drops_per_token = (assign_row < 0).sum(axis=1)
    return dict(
        E=E, k=k, active_tokens=T,
        capacity=-1 if C is None else int(C),
        routed_total=sum(routed), kept_total=total_kept,
        dropped=T * k - total_kept,
        tokens_with_drop=int((drops_per_token > 0).sum()),
        tokens_fully_dropped=int((drops_per_token == k).sum()),
        p50=percentile_linear(kept, 0.50), p95=percentile_linear(kept, 0.95),
        p99=percentile_linear(kept, 0.99),
        max=float(mx), mean=mean,
        max_to_mean=(mx / mean) if mean > 0 else 0.0,
        routed_max=float(max(routed)),
        routed_max_to_mean=(max(routed) / routed_mean) if routed_mean > 0 else 0.0,
        top5pct_share=(sum(top) / total_kept) if total_kept > 0 else 0.0,
        dropped_by_rank=dropped_by_rank,
        tokens_per_expert=kept, routed_per_expert=routed,
    )


def replica_load_stats(parts) -> dict:
    """The job's record over data-parallel replicas ([EP-checks] "Mean expert load proves
    almost nothing": one record per layer for the job).  parts: per replica (routed, kept,
    assign_row, C).  The job record is load_stats of the union of the replicas' picks: counts
    added per expert, the replicas' assign_row stacked (only kept / dropped matters), and an
    expert's capacity the sum of the replicas' capacities (dropless if any replica is)."""
    routed = np.sum([np.asarray(p[0], dtype=np.int64) for p in parts], axis=0)
    kept = np.sum([np.asarray(p[1], dtype=np.int64) for p in parts], axis=0)
    rows = np.vstack([np.asarray(p[2]) for p in parts])
    caps = [p[3] for p in parts]
    C = None if any(c is None for c in caps) else int(sum(caps))
    return load_stats(routed, kept, rows, C)


# --------------------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------------------
def selection_scores(z32, bias=None, bias_mode: int = BIAS_SCORE_AND_WEIGHT) -> np.ndarray:
    """The fp32 scores the top-k is taken on.  In the default mode the bias is already part
    of the logits z32; in selection-only mode the score is fp32(z32 + b), one fp32 addition."""
    z32 = np.asarray(z32, dtype=np.float32)
    if bias_mode != BIAS_SELECTION_ONLY or bias is None:
        return z32
    b = np.asarray(bias, dtype=np.float32)
    return (z32 + (b[None, :] if b.ndim == 1 else b)).astype(np.float32)


def route(z32, k: int, gating: int, capacity_factor: float, layout: int = LAYOUT_COMPACT,
          n_groups: int = 0, topk_groups: int = 0, bias=None,
          bias_mode: int = BIAS_SCORE_AND_WEIGHT, drop_policy: int = DROP_TOKEN_ORDER):
    """Everything that follows from the fp32 logits z32: picks (on the selection scores),
    weights (on z32) and bookkeeping."""
    z32 = np.asarray(z32, dtype=np.float32)
    T, E = z32.shape
    sel = selection_scores(z32, bias, bias_mode)
    idx = select_topk(sel, k, n_groups, topk_groups)
    w = gate_weights(z32, idx, gating)
    C = capacity(capacity_factor, T, k, E)
    a = assign(idx, E, C, layout, drop_policy, scores=sel)
    return dict(idx=idx, w=w, C=C, **a)


def pick_rank_counts(idx, assign_row, E: int, group_of_expert=None) -> dict:
    """The three second-choice counters of [EP-checks] "Top-2 does not insure against hot
    experts", kept for every pick rank j:
      routed[j][e]  picks of rank j that chose expert e (where the second choices go),
      kept[j][e]    those of them that reached the expert FFN (the rest were dropped),
      differs[j]    tokens whose pick j lies in another group than their pick 0, with
                    group = group_of_expert[e] (default: the expert itself).
    Shares (each over the T tokens): differs / T and 1 - sum_e kept[j][e] / T."""
    idx = np.asarray(idx)
    ar = np.asarray(assign_row)
    T, k = idx.shape
    grp = np.arange(E) if group_of_expert is None else np.asarray(group_of_expert)
    routed = np.zeros((k, E), dtype=np.int64)
    kept = np.zeros((k, E), dtype=np.int64)
    differs = np.zeros(k, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            routed[j, e] += 1
            if ar[t, j] >= 0:
                kept[j, e] += 1
            if grp[e] != grp[int(idx[t, 0])]:
                differs[j] += 1
    share = (lambda n: n / T) if T else (lambda n: 0.0)
    return dict(routed=routed, kept=kept, differs=differs,
                differs_share=[share(int(n)) for n in differs],
                dropped_share=[share(T - int(kept[j].sum())) for j in range(k)])


def moe_layer(x, w_router, logit_bias, w_gate, w_up, w_down, k: int, gating: int,
              capacity_factor: float, layout: int = LAYOUT_COMPACT, z32=None,
              n_groups: int = 0, topk_groups: int = 0, bias_mode: int = BIAS_SCORE_AND_WEIGHT,
              drop_policy: int = DROP_TOKEN_ORDER) -> dict:
    """The whole forward on small inputs.  If z32 is given, routing starts from those fp32
    logits (the parity protocol); otherwise from fp32(z64).  In selection-only bias mode
    the logits carry no bias and the bias only shifts the selection scores."""
    sel_only = bias_mode == BIAS_SELECTION_ONLY
    z64 = router_logits(x, w_router, None if sel_only else logit_bias)
    if z32 is None:
        z32 = logits_to_fp32(z64)
    r = route(z32, k, gating, capacity_factor, layout, n_groups, topk_groups,
              logit_bias if sel_only else None, bias_mode, drop_policy)
    x_perm = permute(x, r["token_of_row"])

    def weights_of(e):
        return w_gate[e], w_up[e], w_down[e]

    h_perm, y_perm = expert_ffn(x_perm, r["offsets"], r["kept"], weights_of)
    out = combine(y_perm, r["assign_row"], r["w"])
    stats = load_stats(r["routed"], r["kept"], r["assign_row"], r["C"])
    return dict(z64=z64, z32=z32, x_perm=x_perm, h_perm=h_perm, y_perm=y_perm, out=out,
                stats=stats, **r)


def token_outputs(tokens, x_rows, idx_rows, w_rows, kept_rows, expert_weights) -> np.ndarray:
    """Layer output for a few tokens only, one by one: out[t] = sum over kept picks j of
    w[t, j] * FFN_{idx[t, j]}(x[t]).  Used at full size, where the whole layer is too
    large for the CPU.  kept_rows[i, j] says whether pick j of token i survived capacity."""
    outs = []
    for i, _t in enumerate(tokens):
        acc = None
        for j in range(idx_rows.shape[1]):
            if not kept_rows[i, j]:
                continue
            wg, wu, wd = expert_weights(int(idx_rows[i, j]))
            _, y = swiglu_expert(np.asarray(x_rows[i:i + 1], dtype=np.float64), wg, wu, wd)
            term = w_rows[i, j] * y[0]
            acc = term if acc is None else acc + term
        if acc is None:
            acc = np.zeros(np.asarray(x_rows).shape[1], dtype=np.float64)
        outs.append(acc)
    return np.stack(outs)
