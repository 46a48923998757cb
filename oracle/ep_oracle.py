"""CPU oracle for the expert-parallel (EP) layer across `world` ranks -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import this
module.  It imports nothing from the product.

What it computes, in float64 and in the order the pages give it:

  every rank routes its own tokens and applies the capacity limit (overflow is dropped
  before the exchange) -> the dispatch all-to-all sends each kept (token, expert) row to the
  rank that owns the expert -> each rank runs the SwiGLU FFN of its own experts over the rows
  it received -> the combine all-to-all returns every result row to the token's rank ->
  the gate-weighted sum in pick order -> per-layer expert, rank and node load records.

Sources (page title, section):
  [EP-serving] "Expert Parallelism for MoE Serving" (aiunderstanding.org), "Deep dive" and
               "Technical insight": experts live on different GPUs; dispatch and combine
               are the two all-to-alls of every MoE layer.
  [EP-checks]  "MoE expert parallelism needs measurements before launch" (airouter.kz):
               "Capacity factor changes quality, memory and the latency tail" (tokens past
               the capacity are dropped before the exchange); "Expert and GPU can be
               balanced differently" (expert_load, rank_load = the assignments of all
               experts a rank owns, node_load; per layer: the share of local assignments,
               bytes sent and received by each rank, p50 and p99 of the message size
               between rank pairs, the gap between the busiest and the mean rank, the
               share of traffic crossing a node boundary; placement need not be in order).

Readings taken where the pages are silent (each one is listed in the design notes):
  * placement: expert_rank[e] gives the owner of expert e (default: contiguous blocks of
    E / world experts); a rank's local experts are its experts in ascending index;
  * capacity is applied per source rank with that rank's own T (drop before exchange), so
    each rank's result equals the single-GPU layer on its own tokens;
  * receive layout of rank g: its experts in ascending order; inside an expert, source
    ranks in ascending order; inside a source, that source's slot order;
  * a message is the rows one rank sends another in one dispatch (the combine returns the
    same bytes); local assignments send nothing; pair statistics run over all ordered pairs
    s != g, empty ones included, with the type-7 percentile of the single-GPU statistics;
  * the node-crossing share is the part of the inter-rank bytes whose two ranks sit on
    different nodes (rank r is on node r // ranks_per_node).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np

from oracle import moe_oracle as O


def contiguous_placement(E: int, world: int) -> np.ndarray:
    """expert_rank[e] = e // (E / world): rank g owns experts [g E/world, (g+1) E/world)."""
    if world < 1 or E % world:
        raise ValueError("E must be a multiple of world")
    per = E // world
    return np.arange(E) // per


def local_experts(expert_rank, g: int) -> np.ndarray:
    """The experts rank g owns, in ascending index (its local expert order)."""
    return np.nonzero(np.asarray(expert_rank) == g)[0]


def recv_layout(kept_by_src, expert_rank) -> dict:
    """Where every source's kept rows land on their owner.

    kept_by_src[s][e]: rows source rank s keeps for expert e.  Returns
      base[s][e]      first row, in the owner's receive buffer, of source s's rows for e;
      offsets[g]      bucket starts of rank g's local experts (len = local experts + 1);
      rows[g]         rows rank g receives.
    Rank g's buffer: its experts ascending; inside an expert, sources ascending."""
    kept = np.asarray(kept_by_src, dtype=np.int64)
    G, E = kept.shape
    er = np.asarray(expert_rank)
    base = np.full((G, E), -1, dtype=np.int64)
    offsets: List[List[int]] = []
    rows = []
    for g in range(G):
        pos = 0
        offs = [0]
        for e in local_experts(er, g):
            for s in range(G):
                base[s, e] = pos
                pos += int(kept[s, e])
            offs.append(pos)
        offsets.append(offs)
        rows.append(pos)
    return dict(base=base, offsets=offsets, rows=rows)


def send_rows(assign_row, idx, offsets, base_of_src) -> np.ndarray:
    """Row of pick (t, j) in its owner's receive buffer: base[s][e] + the pick's slot inside
    expert e on the source (assign_row - offsets[e]); -1 for a dropped pick."""
    a = np.asarray(assign_row, dtype=np.int64)
    ix = np.asarray(idx, dtype=np.int64)
    off = np.asarray(offsets, dtype=np.int64)
    b = np.asarray(base_of_src, dtype=np.int64)
    out = np.full(a.shape, -1, dtype=np.int64)
    T, k = a.shape
    for t in range(T):
        for j in range(k):
            if a[t, j] >= 0:
                e = ix[t, j]
                out[t, j] = b[e] + (a[t, j] - off[e])
    return out


def ep_stats(kept_by_src, expert_rank, ranks_per_node: int, row_bytes: int) -> dict:
    """The per-layer EP record of [EP-checks] "Expert and GPU can be balanced differently"
    from the kept-count matrix kept_by_src[s][e]."""
    kept = np.asarray(kept_by_src, dtype=np.int64)
    G, E = kept.shape
    er = np.asarray(expert_rank)
    if ranks_per_node < 1:
        raise ValueError("ranks_per_node must be >= 1")
    n_nodes = (G + ranks_per_node - 1) // ranks_per_node
    node = [r // ranks_per_node for r in range(G)]
    expert_load = kept.sum(axis=0)
    rank_load = [int(expert_load[er == g].sum()) for g in range(G)]
    node_load = [sum(rank_load[g] for g in range(G) if node[g] == n) for n in range(n_nodes)]
    pair_rows = np.zeros((G, G), dtype=np.int64)   # [source, destination]
    for s in range(G):
        for e in range(E):
            pair_rows[s, er[e]] += kept[s, e]
    total = int(kept.sum())
    local = int(np.trace(pair_rows))
    pair_bytes = pair_rows * row_bytes
    off_diag = [int(pair_bytes[s, g]) for s in range(G) for g in range(G) if s != g]
    remote_bytes = sum(off_diag)
    cross = sum(int(pair_bytes[s, g]) for s in range(G) for g in range(G)
                if s != g and node[s] != node[g])
    mean_load = total / G
    mean_node = total / n_nodes
    return dict(
        world=G, ranks_per_node=ranks_per_node, nodes=n_nodes,
        total_assignments=total, local_assignments=local,
        local_fraction=(local / total) if total else 0.0,
        remote_bytes=remote_bytes,
        cross_node_bytes=cross,
        cross_node_fraction=(cross / remote_bytes) if remote_bytes else 0.0,
        pair_bytes_p50=O.percentile_linear(off_diag, 0.50) if off_diag else 0.0,
        pair_bytes_p99=O.percentile_linear(off_diag, 0.99) if off_diag else 0.0,
        pair_bytes_max=float(max(off_diag)) if off_diag else 0.0,
        rank_load=rank_load,
        rank_load_max=float(max(rank_load)), rank_load_mean=mean_load,
        rank_load_max_minus_mean=max(rank_load) - mean_load,
        rank_load_max_to_mean=(max(rank_load) / mean_load) if mean_load else 0.0,
        node_load=node_load,
        node_load_max_to_mean=(max(node_load) / mean_node) if mean_node else 0.0,
        bytes_sent=[int(pair_bytes[s].sum() - pair_bytes[s, s]) for s in range(G)],
        bytes_recv=[int(pair_bytes[:, g].sum() - pair_bytes[g, g]) for g in range(G)],
    )


def ep_layer(xs: Sequence, w_router, biases: Optional[Sequence], w_gate, w_up, w_down, k: int,
             gating: int, capacity_factor: float, expert_rank, z32s: Optional[Sequence] = None,
             ranks_per_node: int = 1, row_bytes: int = 0, n_groups: int = 0,
             topk_groups: int = 0, bias_mode: int = O.BIAS_SCORE_AND_WEIGHT,
             drop_policy: int = O.DROP_TOKEN_ORDER) -> dict:
    """The EP layer over len(xs) ranks, steps in the pages' order.  xs[s]: rank s's tokens;
    biases[s]: its logit bias (or None); z32s[s]: its fp32 logits when routing is to start
    from given logits (the parity protocol).  The routing variants apply on every rank, before
    the exchange, exactly as on one GPU."""
    G = len(xs)
    E = np.asarray(w_router).shape[1]
    er = np.asarray(expert_rank)
    # 1. route and drop locally
    routes = []
    sel_only = bias_mode == O.BIAS_SELECTION_ONLY
    for s in range(G):
        b = None if biases is None else biases[s]
        z32 = (O.logits_to_fp32(O.router_logits(xs[s], w_router, None if sel_only else b))
               if z32s is None else np.asarray(z32s[s], dtype=np.float32))
        routes.append(O.route(z32, k, gating, capacity_factor, O.LAYOUT_COMPACT, n_groups,
                              topk_groups, b if sel_only else None, bias_mode, drop_policy))
    kept = np.stack([r["kept"] for r in routes])
    lay = recv_layout(kept, er)
    # 2. dispatch all-to-all: every kept row goes to its owner's buffer
    d = np.asarray(xs[0]).shape[1]
    recv = [np.zeros((lay["rows"][g], d)) for g in range(G)]
    sends = []
    for s in range(G):
        r = routes[s]
        sr = send_rows(r["assign_row"], r["idx"], r["offsets"], lay["base"][s])
        sends.append(sr)
        x64 = np.asarray(xs[s], dtype=np.float64)
        T = x64.shape[0]
        for t in range(T):
            for j in range(k):
                if sr[t, j] >= 0:
                    recv[er[r["idx"][t, j]]][sr[t, j]] = x64[t]
    # 3. expert FFN of each rank over its own buckets
    y_recv = []
    for g in range(G):
        mine = local_experts(er, g)
        offs = lay["offsets"][g]
        counts = [offs[i + 1] - offs[i] for i in range(len(mine))]

        def weights_of(i, mine=mine):
            e = mine[i]
            return w_gate[e], w_up[e], w_down[e]

        _, y = O.expert_ffn(recv[g], offs[:-1], counts, weights_of)
        y_recv.append(y)
    # 4. combine all-to-all back to the token's rank, then the weighted sum in pick order
    outs = []
    for s in range(G):
        r = routes[s]
        sr = sends[s]
        T = sr.shape[0]
        out = np.zeros((T, d))
        for t in range(T):
            acc = np.zeros(d)
            for j in range(k):
                if sr[t, j] >= 0:
                    acc = acc + r["w"][t, j] * y_recv[er[r["idx"][t, j]]][sr[t, j]]
            out[t] = acc
        outs.append(out)
    stats = ep_stats(kept, er, ranks_per_node, row_bytes or d * 8)
    return dict(routes=routes, kept_by_src=kept, layout=lay, send_rows=sends, recv=recv,
                y_recv=y_recv, out=outs, stats=stats)
