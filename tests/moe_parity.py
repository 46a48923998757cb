"""Shared machinery of the GPU parity tests: run the layer through the C ABI stage by stage
and compare every stage with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import moe_oracle as O
import routing_dispatch_expert_warp_b200 as M
from routing_dispatch_expert_warp_b200 import workload as W

# Tolerances.  Routing, counts, permutation and drops: bit-exact.  Gate weights: 1e-6
# absolute against fp64 from the same fp32 logits.  Outputs: relative Frobenius error
# 1e-5 (fp32 layers) and 2e-2 (bf16 layers).  Logits: fp32 accumulation over d terms.
TOL_OUT = {W.F32: 1e-5, W.BF16: 2e-2}
TOL_W = 1e-6
TOL_LOGIT = 1e-5          # fp32 FMA router
TOL_LOGIT_SPLIT = 1e-4    # tensor-core router with W_r split into two bf16 terms


def router_on_tensor_cores(shape) -> bool:
    """The library's documented rule (include/moe.h, moe_route)."""
    return shape.dtype == W.BF16 and shape.E > 32 and shape.d_model % 64 == 0


def router_tc_splits(shape, sms: int) -> int:
    """Pieces the tensor-core router cuts each 128-token tile's K steps into (1: none): with
    fewer tiles than half the SMs, sms // tiles pieces, at most K steps / 4 and 16, each an
    even number of 64-wide K steps."""
    tiles = (shape.T + 127) // 128
    kb = 2 * shape.d_model // 64
    if 2 * tiles >= sms:
        return 1
    ks = min(sms // tiles, kb // 4, 16)
    if ks < 2:
        return 1
    per = -(-kb // ks)
    per += per & 1
    return -(-kb // per)


def router_launches(shape, presplit: bool, sms: int) -> int:
    """Kernels one moe_route (or moe_route_ex with a split weight) launches."""
    if router_on_tensor_cores(shape):
        topk = shape.n_groups > 1 or router_tc_splits(shape, sms) > 1
        return (0 if presplit else 1) + 1 + (1 if topk else 0)
    return 2   # lane-ordered W_r + fused small-E router, or the fp32 GEMM + top-k


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def i64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.int64).numpy()


def cf32(shape) -> float:
    """The capacity factor as the library sees it (an fp32 field)."""
    return float(np.float32(shape.capacity_factor))


class GpuRun:
    """Inputs on the GPU and every stage's outputs, produced through the C ABI."""

    def __init__(self, shape: W.MoEShape, inputs: W.MoEInputs | None = None):
        self.shape = shape
        self.inp = inputs if inputs is not None else W.make_inputs(shape, device="cuda")
        self.cfg = M.config_from_shape(shape)
        self.ws = M.alloc_workspace(self.cfg)
        self.b = M.LayerBuffers.allocate(self.cfg)

    def route(self):
        i, b = self.inp, self.b
        M.moe_route(self.cfg, i.x, i.w_router, i.logit_bias, b.logits, b.topk_idx, b.topk_w,
                    self.ws)

    def dispatch(self):
        b = self.b
        if self.shape.drop_policy == O.DROP_SCORE:   # the drop decision reads the scores
            M.moe_dispatch_scored(self.cfg, self.inp.x, b.topk_idx, b.logits,
                                  self.inp.logit_bias, b.routed_counts, b.kept_counts,
                                  b.expert_offsets, b.assign_row, b.token_of_row, b.x_perm,
                                  self.ws)
        else:
            M.moe_dispatch(self.cfg, self.inp.x, b.topk_idx, b.routed_counts, b.kept_counts,
                           b.expert_offsets, b.assign_row, b.token_of_row, b.x_perm, self.ws)

    def ffn(self):
        i, b = self.inp, self.b
        M.moe_expert_ffn(self.cfg, b.x_perm, b.expert_offsets, b.kept_counts, i.w_gate, i.w_up,
                         i.w_down, b.h, b.y_perm, self.ws)

    def combine(self):
        b = self.b
        M.moe_combine(self.cfg, b.y_perm, b.assign_row, b.topk_w, b.out)

    def stats(self) -> dict:
        b = self.b
        return M.moe_load_stats(self.cfg, b.routed_counts, b.kept_counts, b.assign_row, b.stats)

    def all_stages(self) -> dict:
        self.route()
        self.dispatch()
        self.ffn()
        self.combine()
        st = self.stats()
        M.moe_check_device_error(self.ws)
        torch.cuda.synchronize()
        return st

    def layer_forward(self):
        i = self.inp
        layer = M.MoELayer(self.cfg, i.w_router, i.w_gate, i.w_up, i.w_down, i.logit_bias)
        out = layer(i.x)
        M.moe_check_device_error(layer.ws)
        torch.cuda.synchronize()
        return layer, out


def check_routing(run: GpuRun, sample_rows=None) -> dict:
    """Logits against fp64, then picks / weights / dispatch bit-exact from the GPU's fp32
    logits.  Returns the oracle's routing (from the GPU logits)."""
    s, b, i = run.shape, run.b, run.inp
    z32 = b.logits.cpu().numpy()
    rows = np.arange(s.T) if sample_rows is None else np.asarray(sample_rows)
    bias = None
    trows = torch.from_numpy(rows).to(i.x.device)
    sel_only = s.bias_mode == O.BIAS_SELECTION_ONLY
    if i.logit_bias is not None and not sel_only:
        bias = f64(i.logit_bias) if i.logit_bias.dim() == 1 else f64(i.logit_bias[trows])
    z64 = O.router_logits(f64(i.x[trows]), f64(i.w_router), bias)
    err = np.abs(z32[rows].astype(np.float64) - z64) / (1.0 + np.abs(z64))
    tol = TOL_LOGIT_SPLIT if router_on_tensor_cores(s) else TOL_LOGIT
    assert err.max() <= tol, f"logits max scaled error {err.max():.3g} (tol {tol})"
    sel_bias = None
    if sel_only and i.logit_bias is not None:
        sel_bias = i.logit_bias.detach().cpu().numpy().astype(np.float32)
    r = O.route(z32, s.k, s.gating, cf32(s), s.layout, s.n_groups, s.topk_groups, sel_bias,
                s.bias_mode, s.drop_policy)
    np.testing.assert_array_equal(i64(b.topk_idx), r["idx"])
    w_err = np.abs(f64(b.topk_w) - r["w"]).max()
    assert w_err <= TOL_W, f"gate weights max abs error {w_err:.3g}"
    np.testing.assert_array_equal(i64(b.routed_counts), r["routed"])
    np.testing.assert_array_equal(i64(b.kept_counts), r["kept"])
    np.testing.assert_array_equal(i64(b.expert_offsets), r["offsets"])
    np.testing.assert_array_equal(i64(b.assign_row), r["assign_row"])
    R = r["rows"]
    np.testing.assert_array_equal(i64(b.token_of_row)[:R], r["token_of_row"])
    assert (i64(b.token_of_row)[R:] == -1).all()
    r["z32"] = z32
    return r


def check_permute(run: GpuRun, r: dict, sample=None):
    b, i = run.b, run.inp
    used = np.nonzero(r["token_of_row"] >= 0)[0]
    if sample is not None and len(used) > sample:
        rng = np.random.default_rng(0)
        used = np.unique(np.concatenate([used[:8], used[-8:], rng.choice(used, sample)]))
    got = b.x_perm[torch.from_numpy(used).to(b.x_perm.device)].cpu()
    want = i.x[torch.from_numpy(r["token_of_row"][used]).to(i.x.device)].cpu()
    assert torch.equal(got, want), "x_perm rows differ from x[token_of_row]"


def check_ffn_rows(run: GpuRun, r: dict, experts=None, rows_per_expert=None) -> float:
    """y_perm (and h) of bucket rows against the fp64 SwiGLU of the GPU's x_perm rows."""
    s, b, i = run.shape, run.b, run.inp
    tol = TOL_OUT[s.dtype]
    experts = range(s.E) if experts is None else experts
    worst = 0.0
    for e in experts:
        n = int(r["kept"][e])
        if n == 0:
            continue
        start = int(r["offsets"][e])
        rows = np.arange(start, start + n)
        if rows_per_expert is not None and n > rows_per_expert:
            rng = np.random.default_rng(e)
            pick = rng.choice(n, rows_per_expert - 2, replace=False)
            rows = np.unique(np.concatenate([[start, start + n - 1], start + pick]))
        ridx = torch.from_numpy(rows).to(b.x_perm.device)
        xr = f64(b.x_perm[ridx])
        h, y = O.swiglu_expert(xr, f64(i.w_gate[e]), f64(i.w_up[e]), f64(i.w_down[e]))
        eh = rel_fro(f64(b.h[ridx]), h)
        ey = rel_fro(f64(b.y_perm[ridx]), y)
        assert eh <= tol, f"expert {e}: h rel error {eh:.3g}"
        assert ey <= tol, f"expert {e}: y rel error {ey:.3g}"
        worst = max(worst, ey)
    return worst


def check_combine(run: GpuRun, r: dict, tokens=None) -> float:
    """out against the fp64 gate-weighted sum of the GPU's y_perm rows."""
    s, b = run.shape, run.b
    toks = np.arange(s.T) if tokens is None else np.asarray(tokens)
    ar = r["assign_row"][toks]
    used = np.unique(ar[ar >= 0])
    # only the rows the sampled tokens use, renumbered 0..len(used)-1
    y = np.zeros((max(len(used), 1), s.d_model))
    if len(used):
        y[: len(used)] = f64(b.y_perm[torch.from_numpy(used).to(b.y_perm.device)])
    local = np.where(ar >= 0, np.searchsorted(used, np.maximum(ar, 0)), -1)
    want = O.combine(y, local, f64(b.topk_w)[toks])
    got = f64(b.out[torch.from_numpy(toks).to(b.out.device)])
    e = rel_fro(got, want)
    # the combine itself only rounds the fp32 sum to the output type
    assert e <= (1e-6 if s.dtype == W.F32 else 8e-3), f"combine rel error {e:.3g}"
    return e


def check_stats(st: dict, r: dict):
    want = O.load_stats(r["routed"], r["kept"], r["assign_row"], r["C"])
    for key in ("E", "k", "active_tokens", "capacity", "routed_total", "kept_total", "dropped",
                "tokens_with_drop", "tokens_fully_dropped", "dropped_by_rank"):
        assert st[key] == want[key], (key, st[key], want[key])
    for key in ("p50", "p95", "p99", "max", "mean", "max_to_mean", "routed_max",
                "routed_max_to_mean", "top5pct_share"):
        assert math.isclose(st[key], want[key], rel_tol=1e-12, abs_tol=1e-12), \
            (key, st[key], want[key])
    # invariants the pages fix
    assert st["kept_total"] == st["active_tokens"] * st["k"] - st["dropped"]
    if st["capacity"] >= 0:
        assert st["max"] <= st["capacity"]


# Worst errors of the whole-layer checks, printed at the end of the session (conftest).
LAYER_REPORT = []


def expert_grouped_outputs(xs, idx, w, kept, expert_weights) -> np.ndarray:
    """out[i] = sum over kept picks j of w[i, j] * FFN_{idx[i, j]}(xs[i]): the oracle's
    per-token definition (token_outputs), evaluated expert by expert -- each expert's fp64
    weights are made once and applied to every sampled token that kept a pick of it -- and
    summed in pick order by the oracle's combine.  At full size the per-token form would
    convert an expert's weights once per pick."""
    n, k = idx.shape
    d = xs.shape[1]
    y = np.zeros((n, k, d), dtype=np.float64)
    for e in np.unique(idx[kept]):
        ti, tj = np.nonzero(kept & (idx == e))
        _, ye = O.swiglu_expert(xs[ti], *expert_weights(int(e)))
        y[ti, tj] = ye
    local = np.where(kept, np.arange(n * k).reshape(n, k), -1)
    return O.combine(y.reshape(n * k, d), local, w)


def check_layer_output(run: GpuRun, out: torch.Tensor, r: dict, tokens=None,
                       label: str | None = None) -> dict:
    """Whole-layer output against the oracle's per-token definition (fp64 FFN of x, gate-
    weighted sum of the kept picks): relative Frobenius error within the tolerance, the
    max-abs error reported beside it."""
    s, i = run.shape, run.inp
    toks = np.arange(s.T) if tokens is None else np.asarray(tokens)
    tt = torch.from_numpy(toks).to(i.x.device)

    def weights_of(e):   # fp64 on the GPU, then one copy (the 22 GB layers have no room twice)
        return tuple(t[e].to(torch.float64).cpu().numpy() for t in (i.w_gate, i.w_up, i.w_down))

    want = expert_grouped_outputs(f64(i.x[tt]), r["idx"][toks], r["w"][toks],
                                  r["assign_row"][toks] >= 0, weights_of)
    got = f64(out[torch.from_numpy(toks).to(out.device)])
    e = rel_fro(got, want)
    m = float(np.abs(got - want).max()) if len(toks) else 0.0
    rec = {"case": label or s.name, "tokens": int(len(toks)), "rel_fro": e, "max_abs": m,
           "max_abs_ref": float(np.abs(want).max()) if len(toks) else 0.0,
           "tol": TOL_OUT[s.dtype]}
    LAYER_REPORT.append(rec)
    assert e <= TOL_OUT[s.dtype], f"layer output rel error {e:.3g} (max abs {m:.3g})"
    return rec
