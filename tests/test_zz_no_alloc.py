"""The allocation-free dispatch entry point against the workspace one.

moe_dispatch_static_scratch serves callers that cannot allocate device memory while they
dispatch (an engine whose pool owns the GPU, a plugin host that hands over only input and
output tensors): it takes no workspace and uses the library's fixed device scratch.  Its
results must equal moe_dispatch's exactly -- this is integer and copy work -- on two calls
in a row, the second with different routing so that stale scratch from the first call would
show.  Its kernel-side errors are kept in the same fixed scratch and reported, without
allocating, by moe_static_scratch_check.  This file is collected last on purpose.
"""
import pytest
import torch

import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import workload as W

pytestmark = pytest.mark.gpu

SHAPES = [
    W.reduced(W.DSV3_PREFILL_ZIPF, 1500, 256, 128),                     # capacity drops, E=256
    W.reduced(W.MIXTRAL_8X22B_MIXED, 2000, 128, 128, n_decode_tokens=8,
              layout=W.LAYOUT_PADDED),
    W.reduced(W.DSV3_PREFILL_ZIPF, 1500, 256, 128, drop_policy=1),     # k histogram planes
]


def _outputs(cfg, device):
    b = M.LayerBuffers.allocate(cfg, device)
    for t in (b.routed_counts, b.kept_counts, b.expert_offsets, b.assign_row, b.token_of_row,
              b.x_perm):
        t.fill_(0x5A if t.dtype != torch.bfloat16 else 7.0)
    return b


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_static_scratch_dispatch_matches_workspace_dispatch(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    dev = torch.device("cuda")
    cfg = M.config_from_shape(shape)
    for call in range(2):
        inp = W.make_inputs(shape.replace(seed=shape.seed + 17 * call), device=dev, weights=False)
        ws = M.alloc_workspace(cfg, dev)
        ref = _outputs(cfg, dev)
        M.moe_route(cfg, inp.x, inp.w_router, inp.logit_bias, ref.logits, ref.topk_idx,
                    ref.topk_w, ws)
        M.moe_dispatch(cfg, inp.x, ref.topk_idx, ref.routed_counts, ref.kept_counts,
                       ref.expert_offsets, ref.assign_row, ref.token_of_row, ref.x_perm, ws)
        got = _outputs(cfg, dev)
        M.moe_dispatch_static_scratch(cfg, inp.x, ref.topk_idx, got.routed_counts,
                                      got.kept_counts, got.expert_offsets, got.assign_row,
                                      got.token_of_row, got.x_perm)
        torch.cuda.synchronize()
        M.moe_check_device_error(ws)
        M.moe_static_scratch_check()      # no kernel-side error recorded
        for name in ("routed_counts", "kept_counts", "expert_offsets", "assign_row",
                     "token_of_row"):
            assert torch.equal(getattr(got, name), getattr(ref, name)), (call, name)
        used = ref.token_of_row >= 0
        assert torch.equal(got.x_perm[used], ref.x_perm[used]), call


def test_static_scratch_rejects_sizes_beyond_its_limit():
    # ceil(T/256) * E * 4 bytes must fit in 1 MiB: T = 300000 at E = 256 does not
    cfg = M.make_config(300000, 64, 64, 256, 8, gating=M.SIGMOID)
    with pytest.raises(M.MoEError) as ei:
        M.moe_dispatch_static_scratch(cfg, *([torch.empty(16, dtype=torch.uint8)] * 8), stream=0)
    assert ei.value.status == 2 and "scratch" in str(ei.value)


def test_static_scratch_reports_a_bad_expert_index():
    """A host-made expert index outside [0, E) is skipped by the kernels and recorded in the
    fixed scratch's status record; moe_static_scratch_check reports it once (and clears it),
    and it stays recorded across a later clean call until it is read."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    dev = torch.device("cuda")
    shape = SHAPES[0]
    cfg = M.config_from_shape(shape)
    inp = W.make_inputs(shape, device=dev, weights=False)
    ws = M.alloc_workspace(cfg, dev)
    b = _outputs(cfg, dev)
    M.moe_route(cfg, inp.x, inp.w_router, inp.logit_bias, b.logits, b.topk_idx, b.topk_w, ws)
    M.moe_check_device_error(ws)
    M.moe_static_scratch_check()          # start from a clean record
    good = b.topk_idx.clone()
    b.topk_idx[5, 3] = shape.E + 7
    args = (b.routed_counts, b.kept_counts, b.expert_offsets, b.assign_row, b.token_of_row,
            b.x_perm)
    M.moe_dispatch_static_scratch(cfg, inp.x, b.topk_idx, *args)
    M.moe_dispatch_static_scratch(cfg, inp.x, good, *args)    # a clean call keeps the record
    with pytest.raises(M.MoEError) as ei:
        M.moe_static_scratch_check()
    assert ei.value.status == 6 and str(5 * shape.k + 3) in str(ei.value)
    M.moe_static_scratch_check()          # cleared by the read
    M.moe_dispatch_static_scratch(cfg, inp.x, good, *args)
    M.moe_static_scratch_check()
