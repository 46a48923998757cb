"""Out-of-bounds writes, caught without a sanitizer: every output buffer and the workspace
sit inside a larger allocation whose bytes before and after them hold a guard pattern; after
every entry point of the layer runs (route, plain and scored dispatch, the three FFN forms,
combine, statistics, second-choice counters, the replica merge) the guards must be intact
and the results must still match a run on plain buffers."""
import ctypes

import pytest
import torch

import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import workload as W

pytestmark = pytest.mark.gpu

GUARD = 1024          # bytes before and after each buffer (keeps 256-byte alignment)
PATTERN = 0xA5


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


class Guarded:
    """Buffers carved out of guarded allocations; check() verifies every guard."""

    def __init__(self):
        self.blocks = []

    def empty(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = max(n, 1) * torch.tensor([], dtype=dtype).element_size()
        full = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.blocks.append((full, nbytes))
        return full[GUARD:GUARD + nbytes].view(dtype)[:n].view(shape) if n else \
            full[GUARD:GUARD + nbytes].view(dtype)[:0].view(shape)

    def check(self):
        torch.cuda.synchronize()
        for i, (full, nbytes) in enumerate(self.blocks):
            head = full[:GUARD]
            tail = full[GUARD + nbytes:]
            assert bool((head == PATTERN).all()), f"buffer {i}: write before its start"
            assert bool((tail == PATTERN).all()), f"buffer {i}: write past its end"


def _buffers(g: Guarded, cfg, gather=False):
    T, d, f, E, k = cfg.T, cfg.d_model, cfg.d_ff, cfg.E, cfg.k
    R = max(M.max_rows(cfg), 1)
    dt = torch.float32 if cfg.dtype == M.F32 else torch.bfloat16
    i32 = torch.int32
    return M.LayerBuffers(
        logits=g.empty((T, E), torch.float32), topk_idx=g.empty((T, k), i32),
        topk_w=g.empty((T, k), torch.float32), routed_counts=g.empty((E,), i32),
        kept_counts=g.empty((E,), i32), expert_offsets=g.empty((E + 1,), i32),
        assign_row=g.empty((T, k), i32), token_of_row=g.empty((R,), i32),
        x_perm=None if gather else g.empty((R, d), dt), h=g.empty((R, f), dt),
        y_perm=g.empty((R, d), dt), out=g.empty((T, d), dt),
        stats=g.empty((ctypes.sizeof(M.MoeLoadStats),), torch.uint8))


def _workspace(g: Guarded, cfg):
    ws = g.empty((M.workspace_size(cfg),), torch.uint8)
    M._abi.check(M._lib().moe_workspace_init(M._ptr(ws), ws.numel(), None))
    return ws


SHAPES = [
    W.TINY_FP32,
    W.reduced(W.MIXTRAL_8X7B, 333, 256, 384, capacity_factor=1.0),
    W.reduced(W.DSV3_PREFILL_ZIPF, 600, 256, 128, capacity_factor=0.8, drop_policy=2,
              bias_mode=1),
    W.reduced(W.MIXTRAL_8X22B_MIXED, 257, 256, 256, n_decode_tokens=8, layout=W.LAYOUT_PADDED),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name + f"_d{s.drop_policy}")
def test_no_write_outside_any_buffer(shape):
    inp = W.make_inputs(shape, device="cuda")
    cfg = M.config_from_shape(shape)
    g = Guarded()
    ws = _workspace(g, cfg)
    b = _buffers(g, cfg)
    bg = _buffers(g, cfg, gather=True)
    fused_out = g.empty(tuple(b.out.shape), b.out.dtype)
    # every stage on guarded buffers
    M.moe_route(cfg, inp.x, inp.w_router, inp.logit_bias, b.logits, b.topk_idx, b.topk_w, ws)
    M.moe_dispatch_scored(cfg, inp.x, b.topk_idx, b.logits, inp.logit_bias, b.routed_counts,
                          b.kept_counts, b.expert_offsets, b.assign_row, b.token_of_row,
                          b.x_perm, ws)
    M.moe_expert_ffn(cfg, b.x_perm, b.expert_offsets, b.kept_counts, inp.w_gate, inp.w_up,
                     inp.w_down, b.h, b.y_perm, ws)
    M.moe_combine(cfg, b.y_perm, b.assign_row, b.topk_w, b.out)
    M.moe_load_stats(cfg, b.routed_counts, b.kept_counts, b.assign_row, b.stats, host=False)
    routed, kept, differs = M.moe_pick_rank_counts(cfg, b.topk_idx, b.assign_row, ws)
    merged = g.empty((ctypes.sizeof(M.MoeLoadStats),), torch.uint8)
    M.moe_load_stats_merge(cfg, b.routed_counts, b.kept_counts, b.stats.view(1, -1), merged,
                           host=False)
    # dispatch without x_perm, gathered FFN, and the FFN with the fused combine
    M.moe_dispatch_scored(cfg, None, b.topk_idx, b.logits, inp.logit_bias, bg.routed_counts,
                          bg.kept_counts, bg.expert_offsets, bg.assign_row, bg.token_of_row,
                          None, ws)
    if cfg.dtype == M.BF16:
        M.moe_expert_ffn_gather(cfg, inp.x, bg.token_of_row, bg.expert_offsets, bg.kept_counts,
                                inp.w_gate, inp.w_up, inp.w_down, bg.h, bg.y_perm, ws)
        M.moe_expert_ffn_combine(cfg, inp.x, b.x_perm, b.token_of_row, b.expert_offsets,
                                 b.kept_counts, inp.w_gate, inp.w_up, inp.w_down, bg.h,
                                 bg.y_perm, b.assign_row, b.topk_w, fused_out, ws)
    M.moe_check_device_error(ws)
    g.check()
    # the same layer on plain buffers gives the same results
    layer = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias)
    ref = layer(inp.x)
    torch.cuda.synchronize()
    assert torch.equal(b.out, ref)
    assert torch.equal(b.assign_row, layer.bufs.assign_row)
    assert torch.equal(b.stats, layer.bufs.stats)
    if cfg.dtype == M.BF16:
        assert torch.equal(fused_out, ref)
