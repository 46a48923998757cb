"""Host logic of the microbatch ping-pong (no GPU): the token split, the dependency graph of
the two-stream schedule, and the critical-path walk on hand-made timelines."""
import pytest

from routing_dispatch_expert_warp_b200 import microbatch as MB


def test_split_tokens():
    assert MB.split_tokens(10, 3) == [(0, 4), (4, 3), (7, 3)]
    assert MB.split_tokens(4096, 2) == [(0, 2048), (2048, 2048)]
    assert MB.split_tokens(5, 5) == [(i, 1) for i in range(5)]
    for T, m in [(1, 1), (7, 2), (1000, 7)]:
        parts = MB.split_tokens(T, m)
        assert sum(n for _, n in parts) == T
        assert all(s == sum(n for _, n in parts[:i]) for i, (s, _) in enumerate(parts))
        assert max(n for _, n in parts) - min(n for _, n in parts) <= 1
    for T, m in [(3, 0), (3, 4)]:
        with pytest.raises(ValueError):
            MB.split_tokens(T, m)


def test_pingpong_dependencies():
    d = MB.pingpong_deps(3, ["a", "b", "c"], "b")
    assert d[(0, "a")] == []
    assert d[(0, "c")] == [(0, "b")]
    assert d[(1, "a")] == [(0, "b")]                  # stagger only: the other stream
    assert d[(2, "a")] == [(1, "b"), (0, "c")]        # stagger + same stream's last stage


def _two_microbatches(gap=0.0):
    return {(0, "a"): (0.0, 1.0), (0, "b"): (1.0, 3.0), (0, "c"): (3.0, 4.0),
            (1, "a"): (3.0 + gap, 3.5 + gap), (1, "b"): (3.5 + gap, 6.0),
            (1, "c"): (6.0, 7.0)}


def test_critical_path_hand_timeline():
    deps = MB.pingpong_deps(2, ["a", "b", "c"], "b")
    cp = MB.critical_path(_two_microbatches(), deps)
    assert cp["path"] == [(0, "a"), (0, "b"), (1, "a"), (1, "b"), (1, "c")]
    assert cp["wall"] == 7.0 and cp["busy"] == 7.0 and cp["gaps"] == 0.0
    assert cp["serial"] == 8.0                        # (0, c) ran under (1, b)
    cp = MB.critical_path(_two_microbatches(gap=0.25), deps)
    assert cp["busy"] == pytest.approx(6.75) and cp["gaps"] == pytest.approx(0.25)


def test_critical_path_follows_the_later_dependency():
    deps = MB.pingpong_deps(3, ["a", "b", "c"], "b")
    iv = {(0, "a"): (0, 1), (0, "b"): (1, 2), (0, "c"): (2, 9),      # a long back stage
          (1, "a"): (2, 3), (1, "b"): (3, 4), (1, "c"): (4, 5),
          (2, "a"): (9, 10), (2, "b"): (10, 11), (2, "c"): (11, 12)}
    cp = MB.critical_path(iv, deps)
    # microbatch 2 shares a stream with microbatch 0 and waited for its long last stage
    assert cp["path"] == [(0, "a"), (0, "b"), (0, "c"), (2, "a"), (2, "b"), (2, "c")]
    assert cp["wall"] == 12 and cp["gaps"] == 0
    assert MB.critical_path({}, {})["path"] == []


def test_stage_record_sums_stages_into_the_record_fields():
    iv = {(0, "route"): (0.0, 0.1), (0, "dispatch"): (0.1, 0.3), (0, "expert_ffn"): (0.3, 2.3),
          (0, "combine"): (2.3, 2.4), (0, "stats"): (2.4, 2.45),
          (1, "route"): (0.3, 0.35), (1, "dispatch"): (0.35, 0.5), (1, "expert_ffn"): (2.3, 4.0),
          (1, "combine"): (4.0, 4.1), (1, "stats"): (4.1, 4.2)}
    deps = MB.pingpong_deps(2, MB.STAGES, "dispatch")
    rec = MB.stage_record({"segments": iv, **MB.critical_path(iv, deps)})
    assert rec["router_ms"] == pytest.approx(0.15)
    assert rec["dispatch_ms"] == pytest.approx(0.35)
    assert rec["expert_compute_ms"] == pytest.approx(3.7)
    assert rec["combine_ms"] == pytest.approx(0.2) and rec["stats_ms"] == pytest.approx(0.15)
    assert rec["pack_ms"] == 0.0 and rec["wall_ms"] == pytest.approx(4.2)
    # expert parallel steps: the count exchange and the plan are the pack
    ep = {(0, "route"): (0, 1), (0, "rank"): (1, 2), (0, "put_counts"): (2, 3),
          (0, "plan"): (3, 5), (0, "dispatch"): (5, 6), (0, "expert_ffn"): (6, 9),
          (0, "combine"): (9, 10), (0, "stats"): (10, 11)}
    steps = ["route", "rank", "put_counts", "plan", "dispatch", "expert_ffn", "combine", "stats"]
    rec = MB.stage_record({"segments": ep, **MB.critical_path(ep, MB.pingpong_deps(1, steps,
                                                                                 "dispatch"))})
    assert rec["pack_ms"] == 4 and rec["dispatch_ms"] == 1 and rec["wall_ms"] == 11
