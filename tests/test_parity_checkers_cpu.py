"""The GPU parity checks, run on the CPU against results the oracle made.

`moe_parity`'s checks compare what the kernels wrote with the oracle.  Here each check is
handed a stand-in run whose buffers hold the oracle's own answer, rounded to the layer's
storage types as the kernels store it.  The check must accept it, and it must reject the
same answer with one planted error in any single field: one logit, pick, gate weight, count,
offset, row, permuted element, hidden or output row, or statistic.  So a green GPU run
means what it says.
"""
import copy
import math
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import moe_parity as MP
from oracle import moe_oracle as O
from routing_dispatch_expert_warp_b200 import workload as W

SHAPES = {
    "bf16_E256_k8_drops": W.reduced(W.DSV3_PREFILL_ZIPF, 64, 64, 32, capacity_factor=0.6),
    "fp32_E8_k2_drops": W.reduced(W.TINY_FP32, 48, 32, 24, capacity_factor=0.75),
    "bf16_E8_k2_padded": W.reduced(W.MIXTRAL_8X22B_MIXED, 40, 64, 48, capacity_factor=0.8,
                                   layout=W.LAYOUT_PADDED),
}


def _max_rows(s, C):
    A = s.T * s.k
    if s.layout == W.LAYOUT_PADDED:
        return s.E * C
    return A if C is None else min(A, s.E * C)


def _oracle_run(shape):
    """A stand-in for a GPU run: the oracle's result in the buffers the kernels fill."""
    inp = W.make_inputs(shape)
    npx = lambda t: None if t is None else t.double().numpy()
    sel_only = shape.bias_mode == O.BIAS_SELECTION_ONLY
    z64 = O.router_logits(npx(inp.x), npx(inp.w_router),
                          None if sel_only else npx(inp.logit_bias))
    z32 = O.logits_to_fp32(z64)
    sel_bias = npx(inp.logit_bias).astype(np.float32) if sel_only else None
    r = O.route(z32, shape.k, shape.gating, MP.cf32(shape), shape.layout, shape.n_groups,
                shape.topk_groups, sel_bias, shape.bias_mode, shape.drop_policy)
    dt = torch.bfloat16 if shape.dtype == W.BF16 else torch.float32
    rows = _max_rows(shape, r["C"])
    tor = np.full(rows, -1, dtype=np.int64)
    tor[:r["rows"]] = r["token_of_row"]
    x_perm = torch.zeros(rows, shape.d_model, dtype=dt)
    used = np.nonzero(tor >= 0)[0]
    x_perm[torch.from_numpy(used)] = inp.x[torch.from_numpy(tor[used])]

    def weights_of(e):
        return npx(inp.w_gate[e]), npx(inp.w_up[e]), npx(inp.w_down[e])

    h64, y64 = O.expert_ffn(x_perm.double().numpy(), r["offsets"], r["kept"], weights_of)
    h = torch.from_numpy(h64).to(dt)
    y_perm = torch.from_numpy(y64).to(dt)
    out = torch.from_numpy(O.combine(y_perm.double().numpy(), r["assign_row"], r["w"])).to(dt)
    i32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.int64)).to(torch.int32)
    b = SimpleNamespace(
        logits=torch.from_numpy(z32.copy()), topk_idx=i32(r["idx"]),
        topk_w=torch.from_numpy(r["w"].astype(np.float32)),
        routed_counts=i32(r["routed"]), kept_counts=i32(r["kept"]),
        expert_offsets=i32(r["offsets"]), assign_row=i32(r["assign_row"]),
        token_of_row=i32(tor), x_perm=x_perm, h=h, y_perm=y_perm, out=out)
    run = SimpleNamespace(shape=shape, inp=inp, b=b)
    stats = O.load_stats(r["routed"], r["kept"], r["assign_row"], r["C"])
    return run, stats


def _all_checks(run, stats):
    n = len(MP.LAYER_REPORT)
    try:
        r = MP.check_routing(run)
        MP.check_stats(stats, r)
        MP.check_permute(run, r)
        MP.check_ffn_rows(run, r)
        MP.check_combine(run, r)
        MP.check_layer_output(run, run.b.out, r, label="oracle-made stand-in")
    finally:
        del MP.LAYER_REPORT[n:]     # stand-ins stay out of the session's report of GPU errors


@pytest.fixture(scope="module", params=sorted(SHAPES))
def made(request):
    run, stats = _oracle_run(SHAPES[request.param])
    assert stats["dropped"] > 0          # the capacity binds, so drops are checked too
    return run, stats


def test_checks_accept_the_oracles_answer(made):
    run, stats = made
    _all_checks(run, stats)


def _first_kept(run):
    ar = run.b.assign_row.numpy()
    t, j = np.argwhere(ar >= 0)[0]
    return int(t), int(j), int(ar[t, j])


def _first_dropped(run):
    t, j = np.argwhere(run.b.assign_row.numpy() < 0)[0]
    return int(t), int(j)


def _plant_logit(run, stats):
    run.b.logits[3, 5] += 1e-3 * (1.0 + abs(float(run.b.logits[3, 5])))


def _plant_pick_swap(run, stats):
    run.b.topk_idx[2, [0, 1]] = run.b.topk_idx[2, [1, 0]].clone()


def _plant_weight(run, stats):
    run.b.topk_w[1, 0] += 3e-6


def _plant_routed(run, stats):
    run.b.routed_counts[0] += 1


def _plant_kept(run, stats):
    e = int(torch.argmax(run.b.kept_counts))
    run.b.kept_counts[e] -= 1


def _plant_offset(run, stats):
    run.b.expert_offsets[1] += 1


def _plant_row_swap(run, stats):
    ar = run.b.assign_row
    kept = np.argwhere(ar.numpy() >= 0)
    (t0, j0), (t1, j1) = kept[0], kept[1]
    ar[t0, j0], ar[t1, j1] = int(ar[t1, j1]), int(ar[t0, j0])


def _plant_dropped_kept(run, stats):
    t, j = _first_dropped(run)
    run.b.assign_row[t, j] = 0


def _plant_token_of_row(run, stats):
    tor = run.b.token_of_row
    r = int(np.nonzero(tor.numpy() >= 0)[0][-1])
    tor[r] = (int(tor[r]) + 1) % run.shape.T


def _plant_unused_row(run, stats):
    tor = run.b.token_of_row.numpy()
    unused = np.nonzero(tor < 0)[0]
    run.b.token_of_row[int(unused[-1])] = 0


def _plant_x_perm(run, stats):
    _, _, row = _first_kept(run)
    v = run.b.x_perm[row, 7]
    run.b.x_perm[row, 7] = torch.nextafter(v, v + 1)


def _plant_h(run, stats):
    _, _, row = _first_kept(run)
    run.b.h[row] = 0


def _plant_y(run, stats):
    _, _, row = _first_kept(run)
    run.b.y_perm[row] = -run.b.y_perm[row]


def _plant_out(run, stats):
    t, _, _ = _first_kept(run)
    run.b.out[t] = run.b.out[t] * 1.5


def _plant_stat(run, stats):
    stats["p95"] += 1e-9


def _plant_drop_stat(run, stats):
    stats["tokens_with_drop"] += 1


PLANTS = {f.__name__[len("_plant_"):]: f for f in (
    _plant_logit, _plant_pick_swap, _plant_weight, _plant_routed, _plant_kept, _plant_offset,
    _plant_row_swap, _plant_dropped_kept, _plant_token_of_row, _plant_unused_row,
    _plant_x_perm, _plant_h, _plant_y, _plant_out, _plant_stat, _plant_drop_stat)}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_checks_reject_one_planted_error(made, plant):
    run0, stats0 = made
    if plant == "unused_row" and (run0.b.token_of_row.numpy() >= 0).all():
        pytest.skip("every row is used")
    b = SimpleNamespace(**{k: v.clone() for k, v in vars(run0.b).items()})
    run = SimpleNamespace(shape=run0.shape, inp=run0.inp, b=b)
    stats = copy.deepcopy(stats0)
    PLANTS[plant](run, stats)
    with pytest.raises(AssertionError):
        _all_checks(run, stats)
