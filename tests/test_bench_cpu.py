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


def test_binding_roof_per_workload():
    # Mixtral prefill: tensor-bound; 2.244 ms for the FFN -> 1286 TFLOP/s
    r = bench.gemm_roofline(W.MIXTRAL_8X7B, 8192, 8, 2.2437, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(1286.4, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / 1674.7)
    # DeepSeek decode: 128 tokens x 8 picks over ~252 experts -> weight streaming binds
    r = bench.gemm_roofline(W.DSV3_DECODE, 1024, 252, 3.2, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    weights = 252 * 3 * 7168 * 2048 * 2
    assert r["algorithmic_bytes_per_step"] == pytest.approx(weights + 1024 * (4 * 7168 + 4 * 2048))
    assert weights == pytest.approx(22.2e9, rel=2e-3)


def test_recorded_traffic_only_for_the_captured_code(monkeypatch):
    rec = bench.recorded_traffic("mixtral8x7b_prefill_T4096", False)
    assert rec is not None and rec["sources"] == bench.gemm_source_hash()
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("mixtral8x7b_prefill_T4096", False) is None
    assert bench.recorded_traffic("some_other_workload", False) is None


def test_code_hash_ignores_comments():
    code = "int a;  // one\n/* two\n   three */\nint b;\n\n"
    edited = "int a;  // another comment\n/* a different\n block */\n\nint b;\n"
    assert bench._code_only(code) == bench._code_only(edited) == "int a;\nint b;"
    assert bench._code_only(code) != bench._code_only("int a;\nint c;")
