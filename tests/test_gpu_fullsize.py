"""The five named workloads at their full sizes, in the launch configuration the benchmark
times.  Routing, counts, permutation indices, drops and statistics are compared in full;
logits, permuted rows, FFN rows and combined tokens on samples the oracle computes one by
one (the largest, the smallest and random buckets, first and last rows included); and the
layer's output itself on sampled tokens against the oracle's per-token definition from x
(relative Frobenius error within the tolerance, max-abs error reported).  The fused
dispatch and fused combine forms of the expert FFN are checked at full size as well:
bitwise equal to the separate stages, and against the oracle from x."""
import numpy as np
import pytest
import torch

from routing_dispatch_expert_warp_b200 import workload as W

import routing_dispatch_expert_warp_b200 as M

from moe_parity import (GpuRun, check_combine, check_ffn_rows, check_layer_output,
                        check_permute, check_routing, check_stats)

pytestmark = pytest.mark.gpu

FULL = [W.TINY_FP32, W.MIXTRAL_8X7B, W.DSV3_DECODE, W.DSV3_PREFILL_ZIPF, W.MIXTRAL_8X22B_MIXED,
        W.DSV3_PREFILL_ZIPF.replace(drop_policy=2)]     # score-priority drops at full size


@pytest.mark.parametrize("shape", FULL, ids=lambda s: s.name + ("_score_drops" if s.drop_policy == 2 else ""))
def test_full_size_sampled(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.empty_cache()
    run = GpuRun(shape)
    st = run.all_stages()
    rng = np.random.default_rng(shape.seed)
    sample_rows = np.unique(np.concatenate([[0, shape.T - 1], rng.choice(shape.T, 64)]))
    r = check_routing(run, sample_rows=sample_rows)
    check_permute(run, r, sample=512)
    kept = r["kept"]
    nz = np.nonzero(kept)[0]
    experts = {int(nz[np.argmax(kept[nz])]), int(nz[np.argmin(kept[nz])])}
    experts |= set(int(e) for e in rng.choice(nz, min(2, len(nz)), replace=False))
    check_ffn_rows(run, r, experts=sorted(experts), rows_per_expert=24)
    toks = np.unique(np.concatenate([[0, shape.T - 1], rng.choice(shape.T, 256)]))
    check_combine(run, r, tokens=toks)
    check_stats(st, r)
    # the layer's output from x: every sampled token (or all of them when T is small)
    out_toks = (np.arange(shape.T) if shape.T <= 320 else
                np.unique(np.concatenate([[0, shape.T - 1],
                                          rng.choice(shape.T, 300, replace=False)])))
    assert len(out_toks) >= min(shape.T, 256)
    tag = "_score_drops" if shape.drop_policy == 2 else ""
    check_layer_output(run, run.b.out, r, tokens=out_toks, label=f"full:{shape.name}{tag}")
    if shape.capacity_factor > 0:
        assert st["max"] <= st["capacity"]
    # the public entry point (moe_layer_forward; the router weight split once at
    # construction) gives bitwise the staged calls' output
    i = run.inp
    layer = M.MoELayer(run.cfg, i.w_router, i.w_gate, i.w_up, i.w_down, i.logit_bias)
    out = layer(i.x)
    M.moe_check_device_error(layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(out, run.b.out)
    del layer, run
    torch.cuda.empty_cache()


@pytest.mark.parametrize("shape", [W.MIXTRAL_8X7B, W.DSV3_PREFILL_ZIPF], ids=lambda s: s.name)
def test_full_size_fused_dispatch_and_combine(shape):
    """The gathered-A FFN (no permuted copy) and the FFN with the combine in its down GEMM, at
    full size: bitwise the separate stages' y_perm and out, and the output within the
    tolerance of the oracle's per-token definition from x."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.empty_cache()
    run = GpuRun(shape)
    run.all_stages()
    rng = np.random.default_rng(shape.seed + 5)
    r = check_routing(run, sample_rows=np.unique(rng.choice(shape.T, 32)))
    b, i, cfg, ws = run.b, run.inp, run.cfg, run.ws
    y_ref, out_ref = b.y_perm.clone(), b.out.clone()
    b.y_perm.fill_(7.0)
    M.moe_expert_ffn_gather(cfg, i.x, b.token_of_row, b.expert_offsets, b.kept_counts, i.w_gate,
                            i.w_up, i.w_down, b.h, b.y_perm, ws)
    M.moe_check_device_error(ws)
    torch.cuda.synchronize()
    rows = int(b.kept_counts.sum())
    assert torch.equal(b.y_perm[:rows], y_ref[:rows]), "gathered-A FFN differs from the permuted one"
    out2 = torch.full_like(out_ref, 3.0)
    M.moe_expert_ffn_combine(cfg, i.x, b.x_perm, b.token_of_row, b.expert_offsets, b.kept_counts,
                             i.w_gate, i.w_up, i.w_down, b.h, b.y_perm, b.assign_row, b.topk_w,
                             out2, ws)
    M.moe_check_device_error(ws)
    torch.cuda.synchronize()
    assert torch.equal(out2, out_ref), "fused combine differs from the separate combine"
    toks = np.unique(np.concatenate([[0, shape.T - 1], rng.choice(shape.T, 256, replace=False)]))
    check_layer_output(run, out2, r, tokens=toks, label=f"full:{shape.name}_fused_ffn_combine")
    del run
    torch.cuda.empty_cache()


@pytest.mark.parametrize("shape,world", [(W.MIXTRAL_8X7B, 8), (W.DSV3_PREFILL_ZIPF, 8)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_full_size_expert_parallel_equals_single_gpu(shape, world):
    """The bench workloads' tokens split over `world` emulated EP ranks: every rank's output
    is bitwise the single-GPU layer's on its own tokens, and the EP record's totals add up."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import routing_dispatch_expert_warp_b200 as M
    from routing_dispatch_expert_warp_b200 import ep as EP
    torch.cuda.empty_cache()
    per = shape.replace(T=shape.T // world)
    inp = W.make_inputs(shape, device="cuda")
    xs = [inp.x[r * per.T:(r + 1) * per.T].contiguous() for r in range(world)]
    biases = ([inp.logit_bias[r * per.T:(r + 1) * per.T].contiguous() for r in range(world)]
              if inp.logit_bias is not None and inp.logit_bias.dim() == 2
              else [inp.logit_bias] * world)
    cfg = M.config_from_shape(per)
    emu = EP.EpEmulator(cfg, world, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, biases)
    outs = [o.clone() for o in emu.forward(xs)]
    for r in emu.ranks:
        M.moe_check_device_error(r.ws)
    st = emu.ranks[0].stats_dict()
    kept_total = sum(int(r.bufs.kept_counts.sum()) for r in emu.ranks)
    assert st["total_assignments"] == kept_total
    assert sum(st["rank_load"]) == kept_total
    del emu
    torch.cuda.empty_cache()
    layer = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, biases[0])
    for g in range(world):
        layer.logit_bias = biases[g]
        ref = layer(xs[g])
        torch.cuda.synchronize()
        assert torch.equal(outs[g], ref), f"rank {g}"
    del layer
    torch.cuda.empty_cache()
