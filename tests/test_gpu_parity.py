"""GPU vs oracle parity through the C ABI, stage by stage and end to end.

Reduced workloads keep each routing regime of the five named layers (E, k, gating, capacity
factor, dtype, bias kind) at sizes the oracle finishes in seconds, while still spanning
several GEMM tiles and ragged tails.  The full-size workloads are checked on sampled rows
and tokens plus properties that hold at any size.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import workload as W

from moe_parity import (GpuRun, check_combine, check_ffn_rows, check_layer_output,
                        check_permute, check_routing, check_stats, f64, i64, rel_fro,
                        router_launches)

pytestmark = pytest.mark.gpu

REDUCED = [
    W.TINY_FP32,
    W.reduced(W.TINY_FP32, 300, 96, 160, capacity_factor=1.0),
    W.reduced(W.MIXTRAL_8X7B, 1000, 512, 768),
    W.reduced(W.DSV3_DECODE, 128, 512, 256),
    W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256),
    W.reduced(W.MIXTRAL_8X22B_MIXED, 1200, 384, 640, n_decode_tokens=16),
    W.reduced(W.MIXTRAL_8X7B, 700, 256, 384, layout=W.LAYOUT_PADDED, capacity_factor=1.1),
]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


@pytest.mark.parametrize("shape", REDUCED, ids=lambda s: s.name)
def test_stages_match_oracle(shape):
    run = GpuRun(shape)
    st = run.all_stages()
    r = check_routing(run)
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)
    check_layer_output(run, run.b.out, r)


@pytest.mark.parametrize("shape", REDUCED[:3] + REDUCED[4:6], ids=lambda s: s.name)
def test_layer_forward_matches_stages_and_is_deterministic(shape):
    run = GpuRun(shape)
    run.all_stages()
    layer, out1 = run.layer_forward()
    out1 = out1.clone()
    assert torch.equal(out1, run.b.out), "moe_layer_forward differs from the staged calls"
    out2 = layer(run.inp.x)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2), "two runs differ bitwise"
    st = layer.bufs.stats_dict()
    r = check_routing(run)
    check_stats(st, r)


# ------------------------------------------------------------------ edge cases
def _edge(T, d, f, E, k, gating=W.SOFTMAX, cf=0.0, dtype=W.BF16, layout=W.LAYOUT_COMPACT,
          seed=7):
    return W.MoEShape(f"edge_T{T}_d{d}_f{f}_E{E}_k{k}_cf{cf}_dt{dtype}_l{layout}", T, d, f, E, k,
                      gating, cf, dtype, layout=layout, seed=seed)


EDGES = [
    _edge(1, 128, 128, 8, 2),                    # a single token
    _edge(1, 64, 64, 4, 4, cf=1.0, dtype=W.F32),  # k = E, capacity 1
    _edge(33, 64, 128, 8, 8, gating=W.SIGMOID),  # k = E, sigmoid
    _edge(65, 128, 192, 1, 1),                   # one expert: a dense FFN
    _edge(200, 64, 64, 16, 1, cf=0.05),          # capacity 1 with top-1
    _edge(129, 128, 128, 32, 3, gating=W.SIGMOID, dtype=W.F32),
    _edge(300, 256, 128, 200, 6, cf=1.0),         # E not a power of two, > 32
    _edge(600, 256, 128, 200, 4, gating=W.SIGMOID, cf=1.5),   # tensor-core router, ragged E
    _edge(520, 128, 128, 64, 8, gating=W.SIGMOID),            # tensor-core router, E = 64
    _edge(300, 2048, 128, 32, 4),       # E = 32 with a long d
    _edge(150, 7168, 64, 8, 2, gating=W.SIGMOID),             # E = 8 at the DeepSeek d
    _edge(77, 6144, 64, 8, 2),          # E = 8 at the Mixtral-8x22B d
]


@pytest.mark.parametrize("shape", EDGES, ids=lambda s: s.name)
def test_edge_shapes(shape):
    run = GpuRun(shape)
    st = run.all_stages()
    r = check_routing(run)
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)
    check_layer_output(run, run.b.out, r)


def test_all_tokens_to_one_expert_with_drops():
    shape = _edge(500, 128, 128, 8, 2, cf=1.0)
    inp = W.make_inputs(shape, device="cuda")
    bias = torch.zeros(8, device="cuda")
    bias[5] = 100.0          # every token picks expert 5 first
    inp.logit_bias = bias
    run = GpuRun(shape.replace(bias="none"), inp)
    st = run.all_stages()
    r = check_routing(run)
    C = O.capacity(1.0, 500, 2, 8)
    assert int(r["kept"][5]) == C and st["dropped"] >= 500 - C
    assert st["dropped_by_rank"][0] == 500 - C
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)


def test_capacity_exactly_hit_keeps_everything():
    # T*k/E with cf = 1 and a uniform assignment: every expert gets exactly C
    T, E, k = 64, 8, 1
    shape = _edge(T, 64, 64, E, k, cf=1.0)
    inp = W.make_inputs(shape, device="cuda")
    bias = torch.full((T, E), -50.0, device="cuda")
    bias[torch.arange(T), torch.arange(T) % E] = 50.0
    inp.logit_bias = bias.contiguous()
    run = GpuRun(shape, inp)
    st = run.all_stages()
    r = check_routing(run)
    assert (r["kept"] == T // E).all() and st["dropped"] == 0
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)


@pytest.mark.parametrize("counts,d,f", [
    ((129, 176, 177, 256), 256, 384),     # tails 1, 48 (folded into the last tile), 49, 0
    ((16, 17, 300, 140), 384, 256),       # buckets below one tile; tails 44 and 12; d not /256
    ((170, 208, 131, 175), 128, 640),     # tails 42, 80, 3, 47
])
def test_bucket_tails_of_every_size(counts, d, f):
    """Exact per-expert bucket sizes (top-1 picks forced by a [T, E] bias) so that the grouped
    GEMM meets tails that ride along with the last full tile, tails that get a tile of their
    own, buckets smaller than a tile and buckets of whole tiles."""
    E, k = len(counts), 1
    T = sum(counts)
    shape = _edge(T, d, f, E, k)
    inp = W.make_inputs(shape, device="cuda")
    owner = torch.cat([torch.full((c,), e, dtype=torch.long) for e, c in enumerate(counts)])
    owner = owner[torch.randperm(T, generator=torch.Generator().manual_seed(5))].cuda()
    bias = torch.full((T, E), -40.0, device="cuda")
    bias[torch.arange(T, device="cuda"), owner] = 40.0
    inp.logit_bias = bias.contiguous()
    run = GpuRun(shape, inp)
    st = run.all_stages()
    r = check_routing(run)
    assert tuple(int(c) for c in r["kept"]) == counts
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)
    check_layer_output(run, run.b.out, r)


def _forced_buckets(counts, d, f, seed=5):
    """A top-1 layer whose bucket sizes are exactly `counts` (a [T, E] bias forces the picks)."""
    E, T = len(counts), sum(counts)
    shape = _edge(T, d, f, E, 1)
    inp = W.make_inputs(shape, device="cuda")
    owner = torch.cat([torch.full((c,), e, dtype=torch.long) for e, c in enumerate(counts)])
    owner = owner[torch.randperm(T, generator=torch.Generator().manual_seed(seed))].cuda()
    bias = torch.full((T, E), -40.0, device="cuda")
    bias[torch.arange(T, device="cuda"), owner] = 40.0
    inp.logit_bias = bias.contiguous()
    return shape, inp


@pytest.mark.parametrize("counts,d,f", [
    # 256-row pair tiles: tails of 1, 127, 128 (the second CTA of the pair has no rows),
    # 129, 255, whole tiles, 257, and an empty expert
    ((1, 127, 128, 129, 255, 256, 257, 0, 511, 513, 15, 16, 17, 33), 256, 384),
    ((300, 0, 5, 700), 512, 256),          # d = 512 (two 256-column down blocks)
    ((64, 200, 384), 192, 320),            # d and d_ff not multiples of 256 / 128
])
def test_ffn_kernels_equal_each_other_and_oracle(counts, d, f):
    """The three expert FFN kernels -- token-N (weight rows as M, tails rounded to 16 tokens),
    token-major (128 x 256 tiles) and CTA pairs (256 x 256 tiles, one MMA over two SMs) --
    each match the oracle, and they compute the same sums in the same K order, so h and
    y_perm agree bitwise."""
    shape, inp = _forced_buckets(counts, d, f)
    run = GpuRun(shape, inp)
    try:
        M.set_ffn_kernel("token_n")
        st = run.all_stages()
        r = check_routing(run)
        assert tuple(int(c) for c in r["kept"]) == counts
        check_ffn_rows(run, r)
        check_layer_output(run, run.b.out, r)
        check_stats(st, r)
        used = int(run.b.expert_offsets[-1])
        h1, y1 = run.b.h[:used].clone(), run.b.y_perm[:used].clone()
        for kind in ("token_major", "pairs"):
            M.set_ffn_kernel(kind)
            run.b.h.zero_(), run.b.y_perm.zero_()
            run.ffn()
            M.moe_check_device_error(run.ws)
            torch.cuda.synchronize()
            check_ffn_rows(run, r)
            assert torch.equal(run.b.h[:used], h1), f"h differs: {kind} vs token_n"
            assert torch.equal(run.b.y_perm[:used], y1), f"y_perm differs: {kind} vs token_n"
    finally:
        M.set_ffn_kernel("token_major")


def test_tied_logits_pick_lower_index():
    shape = _edge(40, 64, 64, 16, 4, gating=W.SIGMOID)
    inp = W.make_inputs(shape, device="cuda")
    inp.x.zero_()                                      # every logit equals its bias
    bias = torch.zeros(16, device="cuda")
    bias[[3, 7, 9, 12]] = 1.0                          # four tied winners
    inp.logit_bias = bias
    run = GpuRun(shape, inp)
    run.all_stages()
    r = check_routing(run)
    assert (r["idx"] == np.array([3, 7, 9, 12])).all()
    assert np.allclose(f64(run.b.topk_w), 0.25)


@pytest.mark.parametrize("k", [1, 8])
def test_tensor_core_router_ties_across_expert_halves(k):
    """The tensor-core router (E = 256, T = 600 >= 512: two 128-expert halves per token, their
    lists merged) with every logit equal to its bias and twelve experts tied on both sides of
    the half boundary: the picks are the k lowest tied experts in index order, as the oracle's
    order (equal scores -> lower index) demands."""
    shape = _edge(600, 128, 64, 256, k, gating=W.SIGMOID)
    inp = W.make_inputs(shape, device="cuda")
    inp.x.zero_()                                      # z = x . W_r = 0 exactly
    tied = [255, 131, 3, 200, 129, 60, 127, 140, 250, 10, 128, 90]
    bias = torch.full((256,), -2.0, device="cuda")
    bias[tied] = 1.0
    inp.logit_bias = bias
    run = GpuRun(shape, inp)
    run.all_stages()
    r = check_routing(run)
    want = np.array(sorted(tied)[:k])
    assert (r["idx"] == want).all()
    assert np.allclose(f64(run.b.topk_w), 1.0 / k)


def test_empty_experts_and_padded_layout():
    shape = _edge(256, 128, 128, 64, 2, cf=2.0, layout=W.LAYOUT_PADDED)
    inp = W.make_inputs(shape, device="cuda")
    bias = torch.full((64,), -30.0, device="cuda")
    bias[:5] = 0.0                                     # only 5 of 64 experts ever picked
    inp.logit_bias = bias
    run = GpuRun(shape, inp)
    st = run.all_stages()
    r = check_routing(run)
    assert (r["kept"][5:] == 0).all()
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)


# ------------------------------------------------------------------ routing variants
VARIANTS = [
    # group-limited top-8 of 256 (8 groups, 4 kept), bias for selection only, pick-rank drops;
    # 1024 tokens: tensor-core router
    W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256, n_groups=8, topk_groups=4, bias_mode=1,
              drop_policy=1),
    # the same regime at 300 tokens (the router's K split over blocks) and token-order drops
    W.reduced(W.DSV3_PREFILL_ZIPF, 300, 256, 128, n_groups=16, topk_groups=2, bias_mode=1),
    # E = 8 with groups (general top-k path), pick-rank drops, chunk bias in score and weight
    W.reduced(W.MIXTRAL_8X22B_MIXED, 900, 256, 384, n_decode_tokens=8, n_groups=4,
              topk_groups=2, drop_policy=1),
    # tensor-core router with the top-k in its epilogue: selection-only bias, E not a
    # multiple of 32 (masked expert columns), a per-token bias, T with a 64-row tail tile
    W.reduced(W.DSV3_PREFILL_ZIPF, 1000, 256, 128, E=200, bias="chunks", bias_mode=1,
              n_decode_tokens=8),
    W.reduced(W.DSV3_PREFILL_ZIPF, 1088, 320, 128, E=96, k=6, gating=W.SOFTMAX),
    # E = 8 fused router with selection-only bias; fp32 layer
    W.reduced(W.TINY_FP32, 200, 64, 96, bias="chunks", bias_mode=1, drop_policy=1,
              capacity_factor=0.9),
]


@pytest.mark.parametrize("shape", VARIANTS, ids=lambda s: s.name + f"_g{s.n_groups}_b{s.bias_mode}_d{s.drop_policy}")
def test_routing_variants_match_oracle(shape):
    run = GpuRun(shape)
    st = run.all_stages()
    r = check_routing(run)
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)
    check_layer_output(run, run.b.out, r)
    if shape.n_groups > 1:   # every token's experts lie in at most topk_groups groups
        gsize = shape.E // shape.n_groups
        spans = [len(set(int(e) // gsize for e in row)) for row in r["idx"]]
        assert max(spans) <= shape.topk_groups


# ------------------------------------------------------------------ errors without faults
@pytest.mark.parametrize("shape", [W.reduced(W.DSV3_PREFILL_ZIPF, 700, 256, 128),
                                   W.reduced(W.DSV3_PREFILL_ZIPF, 640, 256, 128, bias_mode=1)],
                         ids=["bias_in_logits", "selection_only_bias"])
def test_tensor_core_router_without_logits_buffer(shape):
    """moe_route on the tensor-core router (top-k in the GEMM's epilogue) with no logits
    buffer -- z then goes to the workspace -- picks and weights exactly as with one."""
    assert shape.dtype == W.BF16 and shape.E > 32 and shape.T >= 512
    run = GpuRun(shape)
    run.route()
    idx, w = run.b.topk_idx.clone(), run.b.topk_w.clone()
    b, i = run.b, run.inp
    b.topk_idx.fill_(-7), b.topk_w.fill_(-7.0)
    M.moe_route(run.cfg, i.x, i.w_router, i.logit_bias, None, b.topk_idx, b.topk_w, run.ws)
    M.moe_check_device_error(run.ws)
    torch.cuda.synchronize()
    assert torch.equal(b.topk_idx, idx) and torch.equal(b.topk_w, w)
    run.dispatch()
    r = check_routing(run)   # and the picks against the oracle from the returned logits
    assert r["idx"].shape == (shape.T, shape.k)


@pytest.mark.parametrize("shape", [
    W.reduced(W.DSV3_PREFILL_ZIPF, 1000, 256, 128),                        # tensor-core router
    W.reduced(W.DSV3_PREFILL_ZIPF, 1088, 320, 128, E=200, bias="chunks", bias_mode=1,
              n_decode_tokens=8),                                          # masked experts
    W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256, n_groups=8, topk_groups=4),  # + top-k kernel
    W.reduced(W.DSV3_PREFILL_ZIPF, 300, 256, 128),                         # fp32 router: ignored
], ids=["tc", "tc_E200_selbias", "tc_groups", "fp32_T300"])
def test_presplit_router_weight_equals_split_per_call(shape):
    """moe_route_ex given the split W_r of moe_router_split: logits, picks and weights bitwise
    those of moe_route (which splits W_r at every call), with one launch fewer where the
    tensor-core router runs; and the split itself is [hi(W_r^T) | lo(W_r^T)] in bf16."""
    run = GpuRun(shape)
    run.route()
    b, i = run.b, run.inp
    z, idx, w = b.logits.clone(), b.topk_idx.clone(), b.topk_w.clone()
    split = M.router_split(run.cfg, i.w_router)
    assert split is not None and split.numel() == 2 * shape.E * shape.d_model * 2
    wt = i.w_router.t().contiguous()                          # [E, d] fp32
    hi = wt.to(torch.bfloat16)
    lo = (wt - hi.float()).to(torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(split.view(torch.bfloat16).view(shape.E, 2 * shape.d_model),
                       torch.cat([hi, lo], dim=1))
    b.logits.fill_(-7.0), b.topk_idx.fill_(-7), b.topk_w.fill_(-7.0)
    c0 = M.kernel_launch_count()
    M.moe_route_ex(run.cfg, i.x, i.w_router, split, i.logit_bias, b.logits, b.topk_idx,
                   b.topk_w, run.ws)
    launched = M.kernel_launch_count() - c0
    M.moe_check_device_error(run.ws)
    torch.cuda.synchronize()
    assert torch.equal(b.logits, z) and torch.equal(b.topk_idx, idx) and torch.equal(b.topk_w, w)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert launched == router_launches(shape, True, sms)
    run.dispatch()
    check_routing(run)


@pytest.mark.parametrize("shape", [
    W.reduced(W.DSV3_PREFILL_ZIPF, 12000, 256, 64),                   # 94 tiles, 8 K steps
    W.reduced(W.DSV3_PREFILL_ZIPF, 9472, 128, 64),                    # 74 tiles: halves
    W.reduced(W.DSV3_PREFILL_ZIPF, 10000, 192, 64, E=200, bias="chunks", bias_mode=1,
              n_decode_tokens=8),                                     # masked experts
], ids=["T12000_d256", "T9472_d128", "T10000_E200_selbias"])
def test_tensor_core_router_at_many_tiles(shape):
    """The tensor-core router over 74-94 token tiles, each starting its K loop at its own
    chunk of the split weight: logits, picks and weights against the oracle, and bitwise the
    same on a second call."""
    run = GpuRun(shape)
    run.route()
    b, i = run.b, run.inp
    z, idx, w = b.logits.clone(), b.topk_idx.clone(), b.topk_w.clone()
    b.logits.fill_(-7.0), b.topk_idx.fill_(-7), b.topk_w.fill_(-7.0)
    run.route()
    M.moe_check_device_error(run.ws)
    torch.cuda.synchronize()
    assert torch.equal(b.logits, z) and torch.equal(b.topk_idx, idx) and torch.equal(b.topk_w, w)
    run.dispatch()
    check_routing(run)


def test_bad_expert_index_is_reported_not_faulted():
    shape = _edge(50, 64, 64, 8, 2)
    run = GpuRun(shape)
    run.route()
    run.b.topk_idx[3, 1] = 999
    run.dispatch()
    with pytest.raises(M.MoEError) as ei:
        M.moe_check_device_error(run.ws)
    assert ei.value.status == 6
    M.moe_check_device_error(run.ws)   # cleared
    run.route()
    run.dispatch()
    M.moe_check_device_error(run.ws)


def test_bounded_wait_runs_out_and_context_survives():
    cfg = M.make_config(8, 64, 64, 4, 2)
    ws = M.alloc_workspace(cfg)
    M.set_wait_limit_ns(20_000_000)    # 20 ms
    try:
        M.moe_selftest_bounded_wait(ws)
        with pytest.raises(M.MoEError) as ei:
            M.moe_check_device_error(ws)
        assert ei.value.status == 5
    finally:
        M.set_wait_limit_ns(0)
    # the context still works: a normal layer forward afterwards
    run = GpuRun(_edge(64, 128, 128, 8, 2))
    st = run.all_stages()
    r = check_routing(run)
    check_stats(st, r)


# ------------------------------------------------------------------ E <= 8 router, wide d
SMALL_E_WIDE = [
    W.reduced(W.MIXTRAL_8X7B, 1000, 2304, 128),                                  # 9 chunks
    W.reduced(W.MIXTRAL_8X7B, 500, 1024, 128).replace(E=4, k=2),                 # E < 8
    W.reduced(W.MIXTRAL_8X7B, 300, 768, 64).replace(E=6, k=3, gating=W.SIGMOID),
    W.reduced(W.TINY_FP32, 333, 1024, 64),                                       # fp32 x
    W.reduced(W.MIXTRAL_8X22B_MIXED, 777, 768, 128, n_decode_tokens=8, bias_mode=1),
    W.reduced(W.MIXTRAL_8X7B, 1, 512, 64),                                       # one token
    W.reduced(W.MIXTRAL_8X7B, 70, 16384, 64),                                    # 64 chunks
    W.reduced(W.MIXTRAL_8X7B, 70, 16640, 64),                                    # 65 chunks
]


@pytest.mark.parametrize("shape", SMALL_E_WIDE,
                         ids=lambda s: f"{s.name}_E{s.E}_k{s.k}_b{s.bias_mode}")
def test_small_e_router_wide_d(shape):
    """E <= 8 with d over many 256-element chunks, E below the lane group, fp32 x, a chunk
    bias for selection only, one token: logits within the fp32 tolerance, everything
    downstream bit-exact from them."""
    run = GpuRun(shape)
    run.all_stages()
    r = check_routing(run)
    check_layer_output(run, run.b.out, r)


# ------------------------------------------------------------------ launch accounting
@pytest.mark.parametrize("shape,stats_kernels", [
    (W.reduced(W.MIXTRAL_8X7B, 1000, 512, 768), 1),          # lane-ordered W_r + fused router
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256), 1),     # W_r split + GEMM split along K + top-k
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256, n_groups=8, topk_groups=4), 1),  # + top-k
    (W.reduced(W.DSV3_DECODE, 128, 512, 256), 1),            # one tile, K split over blocks
    (W.reduced(W.DSV3_PREFILL_ZIPF, 12000, 256, 64), 2),     # 94 tiles: top-k in the epilogue
    (W.reduced(W.DSV3_PREFILL_ZIPF, 4200, 256, 128), 2),     # 33600 picks: spread drop count
])
def test_kernel_launch_count_per_layer(shape, stats_kernels):
    """One staged layer forward launches the router's kernels (the W_r split, the tensor-core
    GEMM and, when K is split or the picks are group-limited, the top-k; or the E <= 32
    router's two), count + rank + permute, the two grouped GEMMs, combine and the statistics
    (above 32768 picks the drops are counted by a kernel of their own) -- and the library's
    own counter says so."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    run = GpuRun(shape)
    run.all_stages()
    c0 = M.kernel_launch_count()
    run.all_stages()
    assert (M.kernel_launch_count() - c0 ==
            router_launches(shape, False, sms) + 3 + 2 + 1 + stats_kernels)


# ------------------------------------------------------------------ dispatch without x_perm
GATHER = [
    W.TINY_FP32,
    W.reduced(W.MIXTRAL_8X7B, 1000, 512, 768),
    W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256),
    W.reduced(W.MIXTRAL_8X22B_MIXED, 1200, 384, 640, n_decode_tokens=16),
    W.reduced(W.MIXTRAL_8X7B, 700, 256, 384, layout=W.LAYOUT_PADDED, capacity_factor=1.1),
    _edge(1, 128, 128, 8, 2),
    _edge(65, 128, 192, 1, 1),
    _edge(300, 256, 128, 200, 6, cf=1.0),
]


@pytest.mark.parametrize("shape", GATHER, ids=lambda s: s.name)
def test_gathered_ffn_equals_permuted_ffn_and_oracle(shape):
    """moe_dispatch without x_perm + moe_expert_ffn_gather gives h, y_perm and out bitwise equal
    to the permute path (the GEMM sees the same A tiles), and so matches the oracle too."""
    run = GpuRun(shape)
    st = run.all_stages()
    ref_h, ref_y, ref_out = run.b.h.clone(), run.b.y_perm.clone(), run.b.out.clone()
    b = run.b
    b.h.zero_(), b.y_perm.zero_(), b.out.zero_()
    M.moe_dispatch(run.cfg, None, b.topk_idx, b.routed_counts, b.kept_counts, b.expert_offsets,
                   b.assign_row, b.token_of_row, None, run.ws)
    M.moe_expert_ffn_gather(run.cfg, run.inp.x, b.token_of_row, b.expert_offsets, b.kept_counts,
                            run.inp.w_gate, run.inp.w_up, run.inp.w_down, b.h, b.y_perm, run.ws)
    run.combine()
    M.moe_check_device_error(run.ws)
    torch.cuda.synchronize()
    used = int(b.expert_offsets[-1])
    rows = torch.nonzero(b.token_of_row[:used] >= 0).flatten()
    assert torch.equal(b.h[rows], ref_h[rows])
    assert torch.equal(b.y_perm[rows], ref_y[rows])
    assert torch.equal(b.out, ref_out)
    r = check_routing(run)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_layer_output(run, run.b.out, r)


@pytest.mark.parametrize("shape", [W.reduced(W.MIXTRAL_8X7B, 1000, 512, 768), W.TINY_FP32],
                         ids=lambda s: s.name)
def test_layer_forward_without_x_perm(shape):
    run = GpuRun(shape)
    run.all_stages()
    i = run.inp
    layer = M.MoELayer(run.cfg, i.w_router, i.w_gate, i.w_up, i.w_down, i.logit_bias,
                       gather=True)
    assert layer.bufs.x_perm is None
    c0 = M.kernel_launch_count()
    out = layer(i.x)
    launched = M.kernel_launch_count() - c0
    M.moe_check_device_error(layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(out, run.b.out)
    assert launched == 8    # router (2), count + rank, two FFN launches, combine, stats: no permute


# ------------------------------------------------------------------ combine fused into the FFN
FUSED = GATHER + [
    W.reduced(W.DSV3_DECODE, 128, 512, 256),
    _edge(200, 64, 64, 16, 1, cf=0.05),                 # most tokens fully dropped
    _edge(500, 128, 128, 8, 2, cf=0.3),
    W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256, n_groups=8, topk_groups=4, bias_mode=1,
              drop_policy=1),
]


@pytest.mark.parametrize("shape", FUSED, ids=lambda s: s.name)
@pytest.mark.parametrize("gather", [False, True], ids=["x_perm", "gather"])
def test_fused_combine_equals_separate_combine(shape, gather):
    """moe_expert_ffn_combine writes h, y_perm and out bitwise equal to moe_expert_ffn +
    moe_combine, with the A rows from x_perm or gathered from x, fully dropped tokens
    included; a second call on the same workspace gives the same bits (counters reset)."""
    run = GpuRun(shape)
    run.all_stages()
    ref_out, ref_y = run.b.out.clone(), run.b.y_perm.clone()
    b = run.b
    for _ in range(2):
        b.out.fill_(7.0), b.y_perm.zero_()
        M.moe_expert_ffn_combine(run.cfg, run.inp.x, None if gather else b.x_perm,
                                 b.token_of_row, b.expert_offsets, b.kept_counts,
                                 run.inp.w_gate, run.inp.w_up, run.inp.w_down, b.h, b.y_perm,
                                 b.assign_row, b.topk_w, b.out, run.ws)
        M.moe_check_device_error(run.ws)
        torch.cuda.synchronize()
        assert torch.equal(b.out, ref_out)
        used = int(b.expert_offsets[-1])
        rows = torch.nonzero(b.token_of_row[:used] >= 0).flatten()
        assert torch.equal(b.y_perm[rows], ref_y[rows])
    r = check_routing(run)
    check_layer_output(run, run.b.out, r)


def test_host_pipeline_equals_layer_forward():
    """HostPipeline over five distinct pinned host batches gives, for each, the bits of
    MoELayer.forward on that batch, with copies overlapping the kernels of neighbours."""
    shape = W.reduced(W.MIXTRAL_8X7B, 600, 256, 384)
    inp = W.make_inputs(shape, device="cuda")
    cfg = M.config_from_shape(shape)
    xs = [W.make_inputs(shape.replace(seed=shape.seed + i), device="cuda", weights=False).x
          for i in range(5)]
    xs_host = [x.cpu().pin_memory() for x in xs]
    outs_host = [torch.empty((shape.T, shape.d_model), dtype=xs[0].dtype).pin_memory()
                 for _ in xs]
    pipe = M.HostPipeline(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    pipe.run(xs_host, outs_host)
    torch.cuda.current_stream().synchronize()
    for lyr in pipe.layers:
        M.moe_check_device_error(lyr.ws)
    layer = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    for x, o in zip(xs, outs_host):
        ref = layer(x).cpu()
        assert torch.equal(o, ref)


@pytest.mark.parametrize("shape", [W.reduced(W.MIXTRAL_8X7B, 600, 256, 384),
                                   W.reduced(W.DSV3_DECODE, 128, 512, 256),
                                   W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 512, 256)],
                         ids=lambda s: s.name)
def test_captured_layer_replays_bitwise(shape):
    """MoELayer.capture: a CUDA graph of the whole layer replays to the eager bits, and picks
    up new contents of the input buffer."""
    inp = W.make_inputs(shape, device="cuda")
    cfg = M.config_from_shape(shape)
    layer = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    x = inp.x.clone()
    graph = layer.capture(x)
    other = W.make_inputs(shape.replace(seed=shape.seed + 9), device="cuda", weights=False).x
    eager = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    for src in (inp.x, other, inp.x):
        x.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(layer.bufs.out, eager(src))
    M.moe_check_device_error(layer.ws)
