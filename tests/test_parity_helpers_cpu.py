"""The GPU parity tests' whole-layer reference, checked on the CPU: evaluating the oracle's
per-token definition expert by expert (as the full-size checks do, to convert each expert's
weights once) gives the oracle's whole layer and its one-token-at-a-time form."""
import numpy as np

from oracle import moe_oracle as O
from routing_dispatch_expert_warp_b200 import workload as W

from moe_parity import expert_grouped_outputs


def test_expert_grouped_outputs_equal_the_oracle_layer():
    shape = W.reduced(W.DSV3_PREFILL_ZIPF, 40, 32, 24, capacity_factor=0.6)
    inp = W.make_inputs(shape)
    npx = lambda t: None if t is None else t.float().numpy()
    r = O.moe_layer(npx(inp.x), npx(inp.w_router), npx(inp.logit_bias), npx(inp.w_gate),
                    npx(inp.w_up), npx(inp.w_down), shape.k, shape.gating,
                    shape.capacity_factor)
    assert r["stats"]["dropped"] > 0 and r["stats"]["tokens_fully_dropped"] >= 0
    wts = lambda e: (npx(inp.w_gate[e]), npx(inp.w_up[e]), npx(inp.w_down[e]))
    toks = np.array([0, 3, 7, 11, 39])
    kept = r["assign_row"][toks] >= 0
    got = expert_grouped_outputs(npx(inp.x)[toks], r["idx"][toks], r["w"][toks], kept, wts)
    np.testing.assert_allclose(got, r["out"][toks], rtol=1e-12, atol=1e-12)
    per_token = O.token_outputs(toks, npx(inp.x)[toks], r["idx"][toks], r["w"][toks], kept, wts)
    np.testing.assert_allclose(got, per_token, rtol=1e-12, atol=1e-12)
