"""The job record of data-parallel replicas through the C ABI (moe_load_stats_merge):
replicas are layers run on different batches on this GPU, their counts summed and their
records stacked as the collectives would; the merged record must equal the oracle's record
of the union of their picks (integers exactly, fp64 figures to 1e-12)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    yield


@pytest.mark.parametrize("base,Ts", [
    (W.reduced(W.MIXTRAL_8X7B, 400, 256, 128), [400, 400]),                 # dropless
    (W.reduced(W.DSV3_PREFILL_ZIPF, 512, 256, 128, capacity_factor=0.9), [512, 300, 777]),
    (W.reduced(W.MIXTRAL_8X22B_MIXED, 500, 256, 128, n_decode_tokens=8), [500]),
    (W.TINY_FP32, [64, 33, 1, 64]),
], ids=lambda v: getattr(v, "name", str(v)))
def test_merged_record_equals_union_of_replicas(base, Ts):
    layers, parts = [], []
    inp0 = W.make_inputs(base, device="cuda")
    for r, T in enumerate(Ts):
        shape = base.replace(T=T, seed=base.seed + 1000 * r)
        inp = W.make_inputs(shape, device="cuda", weights=False)
        cfg = M.config_from_shape(shape)
        layer = M.MoELayer(cfg, inp0.w_router, inp0.w_gate, inp0.w_up, inp0.w_down,
                           inp.logit_bias)
        layer(inp.x)
        M.moe_check_device_error(layer.ws)
        layers.append(layer)
        C = M.capacity(cfg)
        parts.append((layer.bufs.routed_counts.cpu().numpy(), layer.bufs.kept_counts.cpu().numpy(),
                      layer.bufs.assign_row.cpu().numpy(), None if C < 0 else C))
    routed = torch.stack([l.bufs.routed_counts for l in layers]).sum(0, dtype=torch.int32)
    kept = torch.stack([l.bufs.kept_counts for l in layers]).sum(0, dtype=torch.int32)
    recs = torch.stack([l.bufs.stats for l in layers])
    out = M.stats_buffer()
    got = M.moe_load_stats_merge(layers[0].cfg, routed, kept, recs, out)
    want = O.replica_load_stats(parts)
    for key, val in want.items():
        if key in ("tokens_per_expert", "routed_per_expert"):
            continue
        if isinstance(val, float):
            assert got[key] == pytest.approx(val, rel=1e-12, abs=1e-12), key
        else:
            assert got[key] == val, key
    if len(Ts) == 1:   # one replica: its own record
        assert got == layers[0].bufs.stats_dict()


def test_merge_rejects_bad_arguments():
    cfg = M.make_config(64, 128, 256, 8, 2)
    out = M.stats_buffer()
    z = torch.zeros(8, dtype=torch.int32, device="cuda")
    recs = torch.zeros((0, out.numel()), dtype=torch.uint8, device="cuda")
    with pytest.raises(M.MoEError):
        M.moe_load_stats_merge(cfg, z, z, recs, out)
