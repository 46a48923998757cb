"""Microbatch ping-pong over two streams through the C ABI: every microbatch's rows are the
layer's on that microbatch alone (bitwise), which without a capacity is the whole batch's
layer; the emulated expert-parallel variant equals the single-GPU layer per rank and
microbatch; the recorded timeline is consistent and its critical path is a dependency chain."""
import pytest
import torch

import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import ep as EP
from routing_dispatch_expert_warp_b200 import microbatch as MB
from routing_dispatch_expert_warp_b200 import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


def _slice_bias(bias, start, n):
    return bias if (bias is None or bias.dim() == 1) else bias[start:start + n]


CASES = [
    (W.reduced(W.MIXTRAL_8X7B, 1000, 256, 384), 2),                   # dropless
    (W.reduced(W.MIXTRAL_8X7B, 1001, 256, 384), 3),                   # ragged split
    (W.reduced(W.MIXTRAL_8X22B_MIXED, 900, 256, 256, n_decode_tokens=8), 2),   # chunk bias, cf
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1100, 256, 128, drop_policy=2), 2),       # TC router, score drops
    (W.TINY_FP32, 4),
]


@pytest.mark.parametrize("shape,m", CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_pingpong_equals_per_microbatch_layers(shape, m):
    inp = W.make_inputs(shape, device="cuda")
    cfg = M.config_from_shape(shape)
    mb = MB.MicrobatchLayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias,
                            m=m)
    out = mb(inp.x, record=True).clone()
    for part in mb.mbs:
        M.moe_check_device_error(part["ws"])
    torch.cuda.synchronize()
    for start, n in mb.parts:
        c = M.config_from_shape(shape.replace(T=n))
        layer = M.MoELayer(c, inp.w_router, inp.w_gate, inp.w_up, inp.w_down,
                           _slice_bias(inp.logit_bias, start, n))
        ref = layer(inp.x[start:start + n])
        torch.cuda.synchronize()
        assert torch.equal(out[start:start + n], ref), (start, n)
    if shape.capacity_factor <= 0:
        whole = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
        assert torch.equal(out, whole(inp.x))
    # a second forward gives the same bits
    again = mb(inp.x)
    torch.cuda.synchronize()
    assert torch.equal(again, out)
    # the timeline of the recorded forward
    out = mb(inp.x, record=True)
    torch.cuda.synchronize()
    tl = mb.timeline()
    seg = tl["segments"]
    for (i, name), (s, e) in seg.items():
        assert 0.0 <= s <= e
    for i in range(m):
        ends = [seg[(i, n)] for n in MB.STAGES]
        assert all(a[1] <= b[0] + 1e-3 for a, b in zip(ends, ends[1:]))
    for i in range(1, m):                       # the stagger
        assert seg[(i, "route")][0] >= seg[(i - 1, "dispatch")][1] - 1e-3
    path = tl["path"]
    deps = mb.dependencies()
    assert seg[path[-1]][1] == max(e for _, e in seg.values())
    assert all(a in deps[b] for a, b in zip(path, path[1:]))
    assert tl["busy"] <= tl["wall"] + 1e-3


@pytest.mark.parametrize("shape,world,m", [
    (W.reduced(W.MIXTRAL_8X7B, 600, 256, 384), 4, 2),
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 256, 128), 8, 2),          # capacity per microbatch
    (W.reduced(W.MIXTRAL_8X22B_MIXED, 500, 256, 256, n_decode_tokens=8), 2, 3),
], ids=lambda v: getattr(v, "name", str(v)))
def test_ep_pingpong_equals_single_gpu(shape, world, m):
    base = W.make_inputs(shape, device="cuda")
    xs, biases = [base.x], [base.logit_bias]
    for r in range(1, world):
        o = W.make_inputs(shape.replace(seed=shape.seed + 1000 * r), device="cuda", weights=False)
        xs.append(o.x)
        biases.append(o.logit_bias if shape.bias == "chunks" else base.logit_bias)
    cfg = M.config_from_shape(shape)
    emu = MB.EpMicrobatchEmulator(cfg, world, base.w_router, base.w_gate, base.w_up,
                                  base.w_down, biases, m=m, ranks_per_node=2)
    outs = [o.clone() for o in emu(xs, record=True)]
    for e in emu.emus:
        for r in e.ranks:
            M.moe_check_device_error(r.ws)
    torch.cuda.synchronize()
    for g in range(world):
        for start, n in emu.parts:
            c = M.config_from_shape(shape.replace(T=n))
            layer = M.MoELayer(c, base.w_router, base.w_gate, base.w_up, base.w_down,
                               _slice_bias(biases[g], start, n))
            ref = layer(xs[g][start:start + n])
            torch.cuda.synchronize()
            assert torch.equal(outs[g][start:start + n], ref), (g, start)
    tl = emu.timeline()
    seg = tl["segments"]
    for i in range(1, m):
        assert seg[(i, "route")][0] >= seg[(i - 1, "dispatch")][1] - 1e-3
    assert tl["busy"] <= tl["wall"] + 1e-3
