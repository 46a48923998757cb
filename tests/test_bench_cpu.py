"""The bench's measurement definitions on CPU (no GPU): the algorithmic work per step that the
roofline divides by, checked against the workload table's figures (GEMM FLOPs 6 d f per kept
row; permute and combine bytes (T + A) d s; the decode GEMM's touched weight bytes); the
binding roof chosen per workload; the recorded ncu traffic only while the GEMM's code is the
one captured; and the code hash ignoring comments."""
import pytest

import bench
from routing_dispatch_expert_warp_b200 import workload as W

PEAKS = {"bf16_tflops": 1674.7, "bf16_tflops_sustained": 1364.1, "hbm_gbs": 6538.3,
         "source": "measured"}


def test_mixtral_work_matches_the_table():
    w = bench.algorithmic_work(W.MIXTRAL_8X7B, kept_total=8192)
    assert w["gemm_flops"] == pytest.approx(2886.2e9, rel=1e-4)        # 6 d f A
    assert w["permute_bytes"] == pytest.approx(100.7e6, rel=1e-3)      # (T + A) d s + A * 4
    assert w["combine_bytes"] == pytest.approx(100.7e6, rel=1e-3)      # (A + T) d s + A * 8
    T, d, E, k = 4096, 4096, 8, 2                                      # x, W_r, logits, picks
    assert w["route_bytes"] == T * d * 2 + d * E * 4 + T * E * 4 + T * k * 8
    assert w["route_bytes"] == pytest.approx(33.7e6, rel=1e-2)


def test_work_of_a_small_layer_with_drops_by_hand():
    """Every term of the byte counts, on a layer small enough to add up by hand: T = 4
    tokens, d = 8, bf16 (s = 2), E = 4, k = 2, so A = 8 picks, of which 5 are kept."""
    shape = W.reduced(W.MIXTRAL_8X7B, 4, 8, 16).replace(E=4, k=2)
    w = bench.algorithmic_work(shape, kept_total=5)
    # x read 4*8*2 = 64, kept rows written 5*8*2 = 80, the 8 picks' rows read 8*4 = 32
    assert w["permute_bytes"] == 176
    # kept rows read 80, 8 picks' weights and rows read 8*8 = 64, out written 64
    assert w["combine_bytes"] == 208
    # x 64, W_r 8*4*4 = 128, logits 4*4*4 = 64, picks 8*8 = 64
    assert w["route_bytes"] == 320
    assert w["gemm_flops"] == 6 * 8 * 16 * 5 and w["route_flops"] == 2 * 4 * 8 * 4


def test_binding_roof_per_workload():
    # Mixtral prefill: tensor-bound; 2.244 ms for the FFN -> 1286 TFLOP/s
    r = bench.gemm_roofline(W.MIXTRAL_8X7B, 8192, 8, 2.2437, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(1286.4, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / 1674.7)
    assert r["frac_of_burst"] == r["frac"]
    assert r["frac_of_sustained"] == pytest.approx(r["achieved"] / 1364.1)
    # a power-capped timed region divides by the sustained figure, and says so
    rc = bench.gemm_roofline(W.MIXTRAL_8X7B, 8192, 8, 2.2437, PEAKS, power_capped=True)
    assert rc["peak"] == 1364.1 and rc["frac"] == pytest.approx(rc["achieved"] / 1364.1)
    assert rc["frac_of_burst"] == pytest.approx(r["frac"]) and "sustained" in rc["peak_source"]
    # DeepSeek decode: 128 tokens x 8 picks over ~252 experts -> weight streaming binds
    r = bench.gemm_roofline(W.DSV3_DECODE, 1024, 252, 3.2, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    weights = 252 * 3 * 7168 * 2048 * 2
    assert r["algorithmic_bytes_per_step"] == pytest.approx(weights + 1024 * (4 * 7168 + 4 * 2048))
    assert weights == pytest.approx(22.2e9, rel=2e-3)


def test_recorded_traffic_only_for_the_captured_code(monkeypatch):
    recs = {("some_workload", False): {"bytes": 123, "sources": bench.gemm_source_hash(),
                                       "profile": "profiles/x.md"}}
    monkeypatch.setattr(bench, "RECORDED_GEMM_TRAFFIC", recs)
    rec = bench.recorded_traffic("some_workload", False)
    assert rec is not None and rec["bytes"] == 123
    assert bench.recorded_traffic("some_workload", True) is None
    assert bench.recorded_traffic("some_other_workload", False) is None
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("some_workload", False) is None


def test_every_recorded_traffic_names_its_profile():
    import os
    for (workload, _), rec in bench.RECORDED_GEMM_TRAFFIC.items():
        assert workload in bench.W.WORKLOADS or "_with_" in workload
        assert rec["bytes"] > 0 and len(rec["sources"]) == 16
        assert os.path.exists(os.path.join(bench.ROOT, rec["profile"]))


def test_code_hash_ignores_comments():
    code = "int a;  // one\n/* two\n   three */\nint b;\n\n"
    edited = "int a;  // another comment\n/* a different\n block */\n\nint b;\n"
    assert bench._code_only(code) == bench._code_only(edited) == "int a;\nint b;"
    assert bench._code_only(code) != bench._code_only("int a;\nint c;")


def _oracle_layer(shape):
    import numpy as np
    from oracle import moe_oracle as O
    inp = W.make_inputs(shape)
    f = lambda t: None if t is None else t.float().numpy()
    return O.moe_layer(f(inp.x), f(inp.w_router), f(inp.logit_bias), f(inp.w_gate), f(inp.w_up),
                       f(inp.w_down), shape.k, shape.gating,
                       float(np.float32(shape.capacity_factor)), shape.layout), inp


def test_cpu_sample_of_all_experts_is_the_whole_layer():
    """A sample holding every kept row is the oracle's whole layer: scale 1, and the
    sample's combine gives the layer's output for every token with a kept pick."""
    import numpy as np
    shape = W.reduced(W.DSV3_PREFILL_ZIPF, 96, 64, 32)
    ref, _ = _oracle_layer(shape)
    cs = bench.CpuSample(shape, sample_rows=10 ** 9)
    assert cs.kept_sample == cs.kept_total == int(ref["kept"].sum())
    out = cs.sample_outputs(cs._route())
    np.testing.assert_allclose(out, ref["out"][cs.tokens], rtol=1e-12, atol=1e-12)
    r = cs.run()
    assert r["seconds_extrapolated"] == pytest.approx(r["seconds_measured"], rel=1e-9)
    assert r["cores"] == len(__import__("os").sched_getaffinity(0))


def test_cpu_sample_of_some_experts_is_their_share_of_the_layer():
    """A partial sample: whole experts drawn until the row budget is met, the time scale is
    kept_total / sampled rows, and the sample's combine is the layer's combine restricted to
    the sampled experts' picks."""
    import numpy as np
    from oracle import moe_oracle as O
    shape = W.reduced(W.MIXTRAL_8X22B_MIXED, 200, 64, 48)
    ref, _ = _oracle_layer(shape)
    cs = bench.CpuSample(shape, sample_rows=60)
    kept = ref["kept"]
    assert cs.kept_sample == int(kept[cs.experts].sum()) >= 60
    ar = ref["assign_row"]
    in_s = np.zeros(ar.shape, dtype=bool)
    for e in cs.experts:
        s0, n = int(ref["offsets"][e]), int(kept[e])
        in_s |= (ar >= s0) & (ar < s0 + n)
    masked = np.where(in_s, ar, -1)
    want = O.combine(ref["y_perm"], masked, ref["w"])
    toks = np.nonzero(in_s.any(axis=1))[0]
    np.testing.assert_array_equal(cs.tokens, toks)
    np.testing.assert_allclose(cs.sample_outputs(cs._route()), want[toks], rtol=1e-12, atol=1e-12)
    r = cs.run()
    scale = cs.kept_total / cs.kept_sample
    assert scale > 1 and f"scaled by {scale:.2f}" in r["sample"]


def test_route_tensor_roof_only_for_the_tensor_core_router():
    """The route stage is put against the tensor roof exactly when moe_route runs the
    tensor-core router (bf16, E > 32, d % 64 == 0), counting the two bf16 terms."""
    peaks = {"bf16_tflops": 1000.0}
    ds = W.DSV3_PREFILL_ZIPF
    work = bench.algorithmic_work(ds, 1)
    assert work["route_flops"] == 2.0 * ds.T * ds.d_model * ds.E
    r = bench.route_tensor_roof(ds, work, 0.2, peaks)
    executed = 4.0 * ds.T * ds.d_model * ds.E
    assert r["executed_TFLOP/s"] == pytest.approx(executed / 0.2e-3 / 1e12)
    assert r["frac_tensor"] == pytest.approx(r["executed_TFLOP/s"] / 1000.0)
    assert r["algorithmic_TFLOP/s"] == pytest.approx(r["executed_TFLOP/s"] / 2)
    dec = W.DSV3_DECODE                                          # 128 tokens: tensor cores too
    assert bench.route_tensor_roof(dec, bench.algorithmic_work(dec, 1), 0.2, peaks) != {}
    for shape in (W.MIXTRAL_8X7B, W.TINY_FP32):                  # E = 8, fp32
        assert bench.route_tensor_roof(shape, bench.algorithmic_work(shape, 1), 0.2, peaks) == {}
    for shape in (ds.replace(E=32),                              # E = 32: the CUDA-core router
                  ds.replace(dtype=W.F32),                       # fp32 layer
                  ds.replace(d_model=7168 + 32)):                # d not a multiple of 64
        assert not bench.tensor_core_router(shape)
        assert bench.route_tensor_roof(shape, bench.algorithmic_work(shape, 1), 0.2, peaks) == {}
    assert bench.tensor_core_router(ds.replace(E=33))
