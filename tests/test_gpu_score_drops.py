"""Score-priority drops and the second-choice counters through the C ABI, against the oracle
("MoE expert parallelism needs measurements before launch", "Top-2 does not insure against
hot experts").  Bookkeeping is compared bit for bit: the drop decision is taken on the same
fp32 scores on both sides (the GPU's logits, plus the selection-only bias in one fp32
addition), so every kept/dropped pick, row and count must agree exactly."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import workload as W

from moe_parity import (GpuRun, check_combine, check_ffn_rows, check_layer_output,
                        check_permute, check_routing, check_stats, i64,
                        router_launches)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


SCORE_SHAPES = [
    # group-limited top-8 of 256 with the selection-only bias; tensor-core router
    W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256, n_groups=8, topk_groups=4, bias_mode=1,
              drop_policy=2),
    # heavy drops through the fp32 router, bias inside the logits
    W.reduced(W.DSV3_PREFILL_ZIPF, 700, 256, 128, capacity_factor=0.6, drop_policy=2),
    # padded buckets, chunk bias in score and weights
    W.reduced(W.MIXTRAL_8X22B_MIXED, 900, 256, 384, n_decode_tokens=8, layout=W.LAYOUT_PADDED,
              drop_policy=2),
    # fp32 layer, chunk bias for selection only
    W.reduced(W.TINY_FP32, 200, 64, 96, bias="chunks", bias_mode=1, capacity_factor=0.9,
              drop_policy=2),
    # dropless: the rows must be those of the token-order policy
    W.reduced(W.MIXTRAL_8X7B, 600, 256, 384, drop_policy=2),
]


@pytest.mark.parametrize("shape", SCORE_SHAPES,
                         ids=lambda s: f"{s.name}_cf{s.capacity_factor}_l{s.layout}_b{s.bias_mode}")
def test_score_drops_match_oracle(shape):
    run = GpuRun(shape)
    st = run.all_stages()
    r = check_routing(run)              # routes with DROP_SCORE on the GPU's fp32 logits
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)
    check_layer_output(run, run.b.out, r)
    if shape.capacity_factor <= 0:
        tok = O.assign(r["idx"], shape.E, None, shape.layout, O.DROP_TOKEN_ORDER)
        np.testing.assert_array_equal(i64(run.b.assign_row), tok["assign_row"])


def _dispatch_scored(cfg, idx, logits, bias=None, x=None, x_perm=None):
    """Bookkeeping (and the permute when x_perm is given) from hand-made picks and scores."""
    T, k, E = cfg.T, cfg.k, cfg.E
    dev = "cuda"
    out = dict(routed=torch.empty(E, dtype=torch.int32, device=dev),
               kept=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               assign_row=torch.empty((T, k), dtype=torch.int32, device=dev),
               token_of_row=torch.empty(max(M.max_rows(cfg), 1), dtype=torch.int32, device=dev))
    ws = M.alloc_workspace(cfg)
    M.moe_dispatch_scored(cfg, x, idx, logits, bias, out["routed"], out["kept"], out["offsets"],
                          out["assign_row"], out["token_of_row"], x_perm, ws)
    M.moe_check_device_error(ws)
    torch.cuda.synchronize()
    return {key: i64(v) for key, v in out.items()}


def _check_against_assign(got, idx, scores, E, C, layout):
    a = O.assign(idx, E, C, layout, O.DROP_SCORE, scores=scores)
    np.testing.assert_array_equal(got["routed"], a["routed"])
    np.testing.assert_array_equal(got["kept"], a["kept"])
    np.testing.assert_array_equal(got["offsets"], a["offsets"])
    np.testing.assert_array_equal(got["assign_row"], a["assign_row"])
    R = a["rows"]
    np.testing.assert_array_equal(got["token_of_row"][:R], a["token_of_row"])
    assert (got["token_of_row"][R:] == -1).all()
    return a


def _picks(rng, T, E, k, hot=None):
    """k distinct experts per token; with `hot`, every token's first pick is expert hot."""
    idx = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        if hot is None:
            idx[t] = rng.choice(E, size=k, replace=False)
        else:
            rest = rng.choice(np.delete(np.arange(E), hot), size=k - 1, replace=False)
            idx[t] = np.concatenate([[hot], rest])
    return idx


TIE_VALUES = np.array([-1.0, -0.0, 0.0, 1.0, np.nan, np.inf, -np.inf, 2.5], dtype=np.float32)


@pytest.mark.parametrize("T,E,k,cf,layout,hot,ties", [
    (20000, 16, 2, 1.0, W.LAYOUT_COMPACT, 0, True),      # one expert holds every token
    (20000, 16, 2, 1.0, W.LAYOUT_PADDED, 3, False),
    (777, 8, 3, 0.5, W.LAYOUT_COMPACT, None, True),      # ragged tail, ties, NaN, +-0, inf
    (4097, 256, 8, 1.25, W.LAYOUT_COMPACT, None, False),
    (300, 4, 4, 0.01, W.LAYOUT_PADDED, None, True),      # capacity 3: almost all dropped
    (1, 8, 2, 0.1, W.LAYOUT_COMPACT, None, False),       # one token
])
def test_hand_made_scores(T, E, k, cf, layout, hot, ties):
    rng = np.random.default_rng(T * 31 + E)
    idx = _picks(rng, T, E, k, hot)
    z = (rng.choice(TIE_VALUES, size=(T, E)) if ties
         else rng.standard_normal((T, E))).astype(np.float32)
    cfg = M.make_config(T, 64, 64, E, k, capacity_factor=cf, layout=layout,
                        drop_policy=M.DROP_SCORE)
    C = O.capacity(float(np.float32(cf)), T, k, E)
    got = _dispatch_scored(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(z).cuda())
    a = _check_against_assign(got, idx, z, E, C, layout)
    if hot is not None:
        assert a["kept"][hot] == C and a["routed"][hot] == T


@pytest.mark.parametrize("stride", [0, 8, 11])
def test_selection_only_bias_decides_drops(stride):
    """Scores = fp32(logit + bias) with a per-token bias (row stride >= E) or one [E]
    vector; a bias that reorders the picks must reorder the drops the same way."""
    T, E, k, cf = 1500, 8, 2, 0.75
    rng = np.random.default_rng(stride + 5)
    idx = _picks(rng, T, E, k)
    z = rng.standard_normal((T, E)).astype(np.float32)
    if stride == 0:
        b = rng.standard_normal(E).astype(np.float32)
        bfull = np.broadcast_to(b, (T, E))
    else:
        b = rng.standard_normal((T, stride)).astype(np.float32) * 3
        bfull = b[:, :E]
    scores = (z + bfull).astype(np.float32)
    C = O.capacity(float(np.float32(cf)), T, k, E)
    cfg = M.make_config(T, 64, 64, E, k, capacity_factor=cf, bias_mode=M.BIAS_SELECTION_ONLY,
                        drop_policy=M.DROP_SCORE)
    got = _dispatch_scored(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(z).cuda(),
                           torch.from_numpy(np.ascontiguousarray(b)).cuda())
    _check_against_assign(got, idx, scores, E, C, W.LAYOUT_COMPACT)
    # with the bias in the logits (score-and-weight mode) the bias is not read again
    cfg2 = M.make_config(T, 64, 64, E, k, capacity_factor=cf, drop_policy=M.DROP_SCORE)
    got2 = _dispatch_scored(cfg2, torch.from_numpy(idx).cuda(), torch.from_numpy(z).cuda(),
                            torch.from_numpy(np.ascontiguousarray(b)).cuda())
    _check_against_assign(got2, idx, z, E, C, W.LAYOUT_COMPACT)


def test_scored_permute_rows():
    shape = W.reduced(W.DSV3_PREFILL_ZIPF, 600, 256, 128, capacity_factor=0.8)
    inp = W.make_inputs(shape, device="cuda")
    T, E, k = shape.T, shape.E, shape.k
    rng = np.random.default_rng(2)
    idx = _picks(rng, T, E, k, hot=7)
    z = rng.standard_normal((T, E)).astype(np.float32)
    cfg = M.make_config(T, shape.d_model, shape.d_ff, E, k, capacity_factor=0.8,
                        drop_policy=M.DROP_SCORE)
    xp = torch.zeros((M.max_rows(cfg), shape.d_model), dtype=torch.bfloat16, device="cuda")
    got = _dispatch_scored(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(z).cuda(),
                           x=inp.x, x_perm=xp)
    tor = got["token_of_row"]
    used = np.nonzero(tor >= 0)[0]
    assert torch.equal(xp[torch.from_numpy(used).cuda()],
                       inp.x[torch.from_numpy(tor[used]).cuda()])


@pytest.mark.parametrize("T", [400, 9600], ids=["k_split_router", "epilogue_topk_router"])
def test_layer_forward_with_workspace_logits(T):
    """moe_layer_forward reads the scores from the caller's logits or, when the logits
    pointer is NULL, from the workspace copy moe_route wrote: same result either way, with
    the tensor-core router's K split over blocks (few tiles; the top-k kernel writes z) and
    with its GEMM epilogue taking the top-k (75 tiles)."""
    shape = W.reduced(W.DSV3_PREFILL_ZIPF, T, 256, 128, capacity_factor=0.7, bias_mode=1,
                      drop_policy=2)
    inp = W.make_inputs(shape, device="cuda")
    cfg = M.config_from_shape(shape)
    a = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    out_a = a(inp.x).clone()
    b = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    b._structs.logits = None
    c0 = M.kernel_launch_count()
    out_b = b(inp.x)
    launched = M.kernel_launch_count() - c0
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    assert torch.equal(a.bufs.assign_row, b.bufs.assign_row)
    # router (the tensor-core GEMM on the split W_r MoELayer made once, and the top-k unless it
    # rides in the GEMM's epilogue), 5 ranking kernels, permute, 2 FFN, combine, stats
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    stats = 2 if T * shape.k > 32768 else 1   # above 32768 picks: the drop count of its own
    assert launched == router_launches(shape, True, sms) + 5 + 1 + 2 + 1 + stats


# ------------------------------------------------------------------ second-choice counters
COUNT_SHAPES = [
    W.reduced(W.DSV3_PREFILL_ZIPF, 5000, 256, 128, capacity_factor=0.8, drop_policy=1),
    W.reduced(W.MIXTRAL_8X22B_MIXED, 1111, 256, 256, n_decode_tokens=8),
    W.reduced(W.DSV3_DECODE, 64, 256, 128, capacity_factor=0.5, drop_policy=2),
    W.reduced(W.TINY_FP32, 100, 64, 96, capacity_factor=0.6).replace(k=1),
]


@pytest.mark.parametrize("shape", COUNT_SHAPES, ids=lambda s: f"{s.name}_k{s.k}_d{s.drop_policy}")
def test_pick_rank_counts_match_oracle(shape):
    run = GpuRun(shape)
    run.all_stages()
    idx = i64(run.b.topk_idx)
    ar = i64(run.b.assign_row)
    E = shape.E
    rng = np.random.default_rng(4)
    maps = [None, (np.arange(E) // max(E // 8, 1)).astype(np.int32),
            rng.integers(0, 3, size=E).astype(np.int32)]
    for g in maps:
        gt = None if g is None else torch.from_numpy(g).cuda()
        routed, kept, differs = M.moe_pick_rank_counts(run.cfg, run.b.topk_idx, run.b.assign_row,
                                                       run.ws, gt)
        M.moe_check_device_error(run.ws)
        torch.cuda.synchronize()
        want = O.pick_rank_counts(idx, ar, E, g)
        np.testing.assert_array_equal(i64(routed), want["routed"])
        np.testing.assert_array_equal(i64(kept), want["kept"])
        np.testing.assert_array_equal(i64(differs), want["differs"])
    # the per-rank drops agree with the layer statistics
    st = run.stats()
    for j in range(shape.k):
        assert shape.T - int(i64(kept)[j].sum()) == st["dropped_by_rank"][j]


def test_pick_rank_counts_bad_expert_reported():
    shape = W.reduced(W.MIXTRAL_8X7B, 300, 128, 128)
    run = GpuRun(shape)
    run.all_stages()
    run.b.topk_idx[5, 1] = 4096
    M.moe_pick_rank_counts(run.cfg, run.b.topk_idx, run.b.assign_row, run.ws)
    with pytest.raises(M.MoEError) as ei:
        M.moe_check_device_error(run.ws)
    assert ei.value.status == 6


def test_hand_case_from_golden_fixture(golden_dir):
    """The hand-worked score-drop case and its counters, on the GPU, against the fixture's
    values (derived by hand, not by the oracle)."""
    import json
    import os
    with open(os.path.join(golden_dir, "hand_e4_k2_t8.json")) as f:
        g = json.load(f)
    with open(os.path.join(golden_dir, "hand_e4_k2_t8_score_drops.json")) as f:
        want = json.load(f)
    cfg = M.make_config(g["T"], 64, 64, g["E"], g["k"], capacity_factor=g["capacity_factor"],
                        drop_policy=M.DROP_SCORE)
    idx = torch.tensor(want["idx"], dtype=torch.int32, device="cuda")
    z = torch.tensor(g["logits"], dtype=torch.float32, device="cuda")
    got = _dispatch_scored(cfg, idx, z)
    assert got["assign_row"].tolist() == want["assign_row"]
    assert got["token_of_row"][:len(want["token_of_row"])].tolist() == want["token_of_row"]
    assert got["kept"].tolist() == want["kept"]
    ws = M.alloc_workspace(cfg)
    ar = torch.tensor(want["assign_row"], dtype=torch.int32, device="cuda")
    routed, kept, differs = M.moe_pick_rank_counts(cfg, idx, ar, ws)
    M.moe_check_device_error(ws)
    assert routed.cpu().tolist() == want["routed_by_rank"]
    assert kept.cpu().tolist() == want["kept_by_rank"]
    assert differs.cpu().tolist() == want["differs_by_rank"]
