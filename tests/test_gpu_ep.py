"""Expert parallelism through the C ABI, with `world` ranks emulated on one GPU.

The kernels are those a multi-GPU run uses (peer tables of buffer pointers, no collective
library); only the barrier differs (stream order).  Checks: every rank's output is bitwise
the single-GPU layer's on that rank's tokens (drop before exchange, row-wise expert FFN),
the count matrix, send rows, receive layout and received rows equal the oracle's, and the
EP record equals the oracle's.
"""
import numpy as np
import pytest
import torch

from oracle import ep_oracle as EPO
import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import ep as EP
from routing_dispatch_expert_warp_b200 import workload as W

from moe_parity import router_launches

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


def _rank_inputs(shape, world):
    """Shared weights (rank 0's draw), per-rank tokens and biases."""
    base = W.make_inputs(shape, device="cuda")
    xs, biases = [base.x], [base.logit_bias]
    for r in range(1, world):
        other = W.make_inputs(shape.replace(seed=shape.seed + 1000 * r), device="cuda",
                              weights=False)
        xs.append(other.x)
        biases.append(other.logit_bias if shape.bias == "chunks" else base.logit_bias)
    return base, xs, biases


CASES = [
    # (shape, world, placement)
    (W.reduced(W.MIXTRAL_8X7B, 600, 256, 384), 2, "contiguous"),
    (W.reduced(W.MIXTRAL_8X7B, 600, 256, 384), 8, "contiguous"),           # one expert per rank
    (W.reduced(W.MIXTRAL_8X22B_MIXED, 700, 256, 256, n_decode_tokens=8), 4, "permuted"),
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 256, 128), 8, "contiguous"),     # capacity drops
    (W.reduced(W.DSV3_DECODE, 64, 256, 128), 4, "permuted"),
    (W.TINY_FP32, 2, "contiguous"),
    # routing variants: group-limited top-k, selection-only bias, pick-rank drops
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 256, 128, n_groups=8, topk_groups=4, bias_mode=1,
               drop_policy=1), 4, "permuted"),
    (W.reduced(W.MIXTRAL_8X7B, 300, 128, 128), 1, "contiguous"),
    # score-priority drops, decided on each rank before the exchange
    (W.reduced(W.DSV3_PREFILL_ZIPF, 1024, 256, 128, capacity_factor=0.8, drop_policy=2), 4,
     "permuted"),
]


@pytest.mark.parametrize("shape,world,placement", CASES,
                         ids=[f"{s.name}_w{w}_{p}" for s, w, p in CASES])
def test_ep_emulated_equals_single_gpu_per_rank(shape, world, placement):
    base, xs, biases = _rank_inputs(shape, world)
    cfg = M.config_from_shape(shape)
    er = EP.contiguous_placement(shape.E, world)
    if placement == "permuted":
        er = er[torch.randperm(shape.E, generator=torch.Generator().manual_seed(3))]
    emu = EP.EpEmulator(cfg, world, base.w_router, base.w_gate, base.w_up, base.w_down,
                        biases, expert_rank=er, ranks_per_node=2)
    outs = [o.clone() for o in emu.forward(xs)]
    for r in emu.ranks:
        M.moe_check_device_error(r.ws)
    torch.cuda.synchronize()

    er_np = er.cpu().numpy()
    kept = np.stack([r.bufs.kept_counts.cpu().numpy() for r in emu.ranks])
    lay = EPO.recv_layout(kept, er_np)
    row_bytes = shape.d_model * (2 if shape.dtype == W.BF16 else 4)
    for g, r in enumerate(emu.ranks):
        # single-GPU layer on this rank's tokens, same weights and bias
        layer = M.MoELayer(cfg, base.w_router, base.w_gate, base.w_up, base.w_down, biases[g])
        ref = layer(xs[g])
        torch.cuda.synchronize()
        assert torch.equal(outs[g], ref), f"rank {g}: EP output differs from the local layer"
        assert torch.equal(r.bufs.topk_idx, layer.bufs.topk_idx)
        # every rank holds the same full count matrix
        np.testing.assert_array_equal(r.count_mat.cpu().numpy(), kept)
        # send rows and the local bucket table
        b = r.bufs
        want = EPO.send_rows(b.assign_row.cpu().numpy(), b.topk_idx.cpu().numpy(),
                             b.expert_offsets.cpu().numpy(), lay["base"][g])
        np.testing.assert_array_equal(r.send_row.cpu().numpy(), want)
        offs = lay["offsets"][g]
        np.testing.assert_array_equal(r.recv_offsets.cpu().numpy(), offs)
        np.testing.assert_array_equal(r.recv_counts.cpu().numpy(), np.diff(offs))
        # the EP record
        st = r.stats_dict()
        ref_st = EPO.ep_stats(kept, er_np, 2, row_bytes)
        for key, val in ref_st.items():
            if isinstance(val, float):
                assert st[key] == pytest.approx(val, rel=1e-12, abs=1e-9), key
            else:
                assert st[key] == val, key
    # received rows: row send_row[t, j] of the owner holds x[t] of the source
    for s, r in enumerate(emu.ranks):
        sr = r.send_row.cpu()
        owner = er.cpu()[r.bufs.topk_idx.cpu().long()]
        for g, dst in enumerate(emu.ranks):
            sel = (sr >= 0) & (owner == g)
            t_idx = torch.nonzero(sel)[:, 0]
            rows = sr[sel].long()
            assert torch.equal(dst.recv_x[rows.cuda()], xs[s][t_idx.cuda()])


def test_ep_emulated_twice_is_deterministic():
    shape = W.reduced(W.DSV3_PREFILL_ZIPF, 512, 128, 128)
    base, xs, biases = _rank_inputs(shape, 4)
    cfg = M.config_from_shape(shape)
    emu = EP.EpEmulator(cfg, 4, base.w_router, base.w_gate, base.w_up, base.w_down, biases)
    first = [o.clone() for o in emu.forward(xs)]
    c0 = M.kernel_launch_count()
    second = emu.forward(xs)
    launched = M.kernel_launch_count() - c0
    torch.cuda.synchronize()
    for a, b in zip(first, second):
        assert torch.equal(a, b)
    # per rank: router (the W_r split + the tensor-core GEMM, with the top-k in its epilogue
    # or a kernel of its own when K is split), count + rank, put_counts, plan (2), dispatch,
    # FFN (2), combine, stats
    router = router_launches(shape, False, torch.cuda.get_device_properties(0).multi_processor_count)
    assert launched == 4 * (router + 2 + 1 + 2 + 1 + 2 + 1 + 1)


def test_ep_receive_overflow_is_reported_not_faulted():
    shape = W.reduced(W.MIXTRAL_8X7B, 200, 128, 128)
    base, xs, biases = _rank_inputs(shape, 2)
    cfg = M.config_from_shape(shape)
    emu = EP.EpEmulator(cfg, 2, base.w_router, base.w_gate, base.w_up, base.w_down, biases,
                        recv_rows=8)   # far too small: rows past it are skipped and reported
    emu.forward(xs)
    with pytest.raises(M.MoEError) as ei:
        for r in emu.ranks:
            M.moe_check_device_error(r.ws)
    assert ei.value.status == 6
