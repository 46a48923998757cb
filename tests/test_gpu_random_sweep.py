"""A seeded random sweep of small layer configurations through every stage, against the
oracle: token counts, widths, expert counts, picks, gating, capacity (dropless, tight,
loose), layout, dtype, bias kind and the routing variants, drawn at random, so that
combinations the hand-picked cases miss are exercised too.  Each case spans several GEMM
tiles or ragged tails and is small enough for the oracle."""
import os

import numpy as np
import pytest
import torch

from routing_dispatch_expert_warp_b200 import workload as W

from moe_parity import (GpuRun, check_combine, check_ffn_rows, check_layer_output,
                        check_permute, check_routing, check_stats)

pytestmark = pytest.mark.gpu


def _draw(i: int) -> W.MoEShape:
    rng = np.random.default_rng(9000 + i)
    dtype = W.BF16 if rng.random() < 0.8 else W.F32
    E = int(rng.choice([1, 2, 5, 8, 16, 24, 32, 48, 64, 100, 128, 256]))
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.choice([1, 3, 17, 64, 129, 300, 513, 777, 1100]))
    mult = 64 if dtype == W.BF16 else 8
    d = int(rng.choice([1, 2, 3, 4, 6])) * mult
    f = int(rng.choice([1, 2, 3, 5])) * mult
    cf = float(rng.choice([0.0, 0.0, 0.3, 1.0, 1.25, 2.0]))
    layout = W.LAYOUT_PADDED if (cf > 0 and rng.random() < 0.3) else W.LAYOUT_COMPACT
    gating = W.SIGMOID if rng.random() < 0.4 else W.SOFTMAX
    bias = str(rng.choice(["none", "zipf", "chunks"])) if E > 1 else "none"
    n_groups = topk_groups = 0
    if E >= 8 and rng.random() < 0.3:
        divisors = [g for g in (2, 4, 8) if E % g == 0 and g <= E]
        if divisors:
            n_groups = int(rng.choice(divisors))
            gsize = E // n_groups
            lo = (k + gsize - 1) // gsize
            topk_groups = int(rng.integers(lo, n_groups + 1))
    bias_mode = 1 if (bias != "none" and rng.random() < 0.3) else 0
    drop_policy = 1 if (cf > 0 and rng.random() < 0.4) else 0
    if drop_policy == 0 and rng.random() < (0.4 if cf > 0 else 0.1):
        drop_policy = 2     # score priority (dropless: must equal token order)
    return W.MoEShape(f"rand{i}_T{T}_d{d}_f{f}_E{E}_k{k}_cf{cf}_{'bf16' if dtype else 'f32'}"
                      f"_d{drop_policy}",
                      T, d, f, E, k, gating, cf, dtype, bias=bias, layout=layout,
                      seed=7000 + i, n_decode_tokens=min(8, T), n_groups=n_groups,
                      topk_groups=topk_groups, bias_mode=bias_mode, drop_policy=drop_policy)


# 96 configurations by default; MOE_SWEEP_CASES=n draws n (the first 96 are always the same).
CASES = [_draw(i) for i in range(int(os.environ.get("MOE_SWEEP_CASES", "96")))]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: s.name)
def test_random_config_matches_oracle(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    run = GpuRun(shape)
    st = run.all_stages()
    r = check_routing(run)
    check_permute(run, r)
    check_ffn_rows(run, r)
    check_combine(run, r)
    check_stats(st, r)
    check_layer_output(run, run.b.out, r)


def _ep_draw(i: int):
    rng = np.random.default_rng(5000 + i)
    while True:
        shape = _draw(1000 + i + int(rng.integers(0, 10_000)))
        worlds = [g for g in (2, 3, 4, 8) if g <= shape.E]
        if worlds and shape.T >= 2:
            return shape, int(rng.choice(worlds)), int(rng.integers(0, 2**31 - 1))


EP_CASES = [_ep_draw(i) for i in range(max(16, len(CASES) // 8))]


@pytest.mark.parametrize("shape,world,pseed", EP_CASES,
                         ids=[f"{s.name}_w{w}" for s, w, _ in EP_CASES])
def test_random_expert_parallel_matches_single_gpu(shape, world, pseed):
    """Random placement (every rank owns at least one expert) and per-rank batches: each
    emulated rank's output is bitwise the single-GPU layer's on its own tokens."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import routing_dispatch_expert_warp_b200 as M
    from routing_dispatch_expert_warp_b200 import ep as EP
    g = torch.Generator().manual_seed(pseed)
    owner = torch.cat([torch.arange(world), torch.randint(0, world, (shape.E - world,),
                                                          generator=g)])
    er = owner[torch.randperm(shape.E, generator=g)].to(torch.int32)
    base = W.make_inputs(shape, device="cuda")
    xs, biases = [base.x], [base.logit_bias]
    for r in range(1, world):
        other = W.make_inputs(shape.replace(seed=shape.seed + 1000 * r), device="cuda",
                              weights=False)
        xs.append(other.x)
        biases.append(other.logit_bias if shape.bias == "chunks" else base.logit_bias)
    cfg = M.config_from_shape(shape)
    emu = EP.EpEmulator(cfg, world, base.w_router, base.w_gate, base.w_up, base.w_down, biases,
                        expert_rank=er)
    outs = [o.clone() for o in emu.forward(xs)]
    for r in emu.ranks:
        M.moe_check_device_error(r.ws)
    for rank in range(world):
        layer = M.MoELayer(cfg, base.w_router, base.w_gate, base.w_up, base.w_down,
                           biases[rank])
        ref = layer(xs[rank])
        torch.cuda.synchronize()
        assert torch.equal(outs[rank], ref), f"rank {rank}"
