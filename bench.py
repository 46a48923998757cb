"""Benchmark of one MoE layer forward on B200: tokens/s of the whole layer, with the grouped
GEMM's tensor throughput and the permute/combine bandwidth beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = the whole hot path on one batch: route -> dispatch (count, scan, rank, permute)
-> expert SwiGLU grouped GEMM (gate/up, down) -> combine -> load statistics, each stage one
C-ABI call on the same stream with CUDA events between them.  Inputs are resident in HBM;
L2 is flushed (a 256 MB write) between timed steps, outside the timed events.  With N > 1
(torchrun, one process per GPU) every GPU runs its own replica of the layer on its own batch
-- the path has no exchange at EP=1 -- and the slowest rank's time is taken.

--impl reference times the CPU oracle (fp64 numpy) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import routing_dispatch_expert_warp_b200 as M  # noqa: E402
from routing_dispatch_expert_warp_b200 import workload as W  # noqa: E402

DEFAULT = W.DSV3_PREFILL_ZIPF
METRIC = "MoE-layer tokens/s on 1 B200; grouped-GEMM % BF16 peak; permute/combine % HBM BW"
L2_FLUSH_BYTES = 256 << 20

# DRAM traffic of the grouped GEMM (gate/up + down launch, bytes per layer step) from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), keyed by workload and dispatch
# mode, with the hash of the GEMM's source code (comments stripped) at capture time: a
# changed kernel reports null.
GEMM_SOURCES = ("routing_dispatch_expert_warp_b200/csrc/moe_ffn_tc.cu",
                "routing_dispatch_expert_warp_b200/csrc/moe_device.cuh",
                "routing_dispatch_expert_warp_b200/csrc/moe_internal.h")
RECORDED_GEMM_TRAFFIC = {
    ("mixtral8x7b_prefill_T4096", False): {
        "bytes": 3668137216, "sources": "9f1036f2df2eb2be",
        "profile": "profiles/grouped_gemm_tc_mixtral8x7b_T4096_traffic.md"},
    ("dsv3_prefill_zipf_T16384", False): {
        "bytes": 27606953472, "sources": "9f1036f2df2eb2be",
        "profile": "profiles/grouped_gemm_tc_dsv3_prefill_T16384_traffic.md"},
}


def _code_only(text: str) -> str:
    """C/C++ source without its comments and blank lines (a comment edit keeps the hash)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def gemm_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), rel)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, gather: bool):
    rec = RECORDED_GEMM_TRAFFIC.get((workload, gather))
    if rec is None or rec["sources"] != gemm_source_hash():
        return None
    return rec


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


# NVML clock-event reason bits (public NVML API constants) that the record names.
CLOCK_REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                 "hw_thermal_slowdown": 0x40}


class ClockSampler:
    """SM clock and clock-event reasons during the timed region, read (never set) through
    NVML every `interval` seconds on a host thread; mark_start() / mark_end() bracket the
    timed region, and the record is the median SM clock and the union of the reasons over
    the samples inside it (all samples if none fell inside).  Without NVML it polls
    nvidia-smi every 100 ms instead."""

    def __init__(self, index: int, interval: float = 0.005, nvml=None):
        import threading
        self.samples, self.t0, self.t1 = [], None, None
        self.proc, self.thread, self.source = None, None, None
        try:
            if nvml is None:
                import pynvml as nvml
            nvml.nvmlInit()
            self.nvml, self.handle = nvml, self._handle(nvml, index)
            self.source = "nvml"
        except Exception:
            self.nvml = None
            self._start_smi(index)
            return
        self._stop = threading.Event()
        self.interval = interval
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    @staticmethod
    def _handle(nvml, index: int):
        try:  # the CUDA device's own PCI address: CUDA and NVML may number GPUs differently
            p = torch.cuda.get_device_properties(index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nvml.nvmlDeviceGetHandleByIndex(index)

    def _run(self) -> None:
        n = self.nvml
        get_reasons = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(n, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(),
                                     float(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)),
                                     float(n.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                       n.NVML_CLOCK_SM)),
                                     int(get_reasons(self.handle))))
            except Exception:
                pass
            self._stop.wait(self.interval)

    def _start_smi(self, index: int) -> None:
        # BENCH_CLOCKS_DIR keeps the raw samples somewhere chosen; default: a temp dir
        out_dir = os.environ.get("BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"moe_bench_clocks_gpu{index}.csv")
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi"
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_start(self) -> None:
        self.t0 = time.perf_counter()

    def mark_end(self) -> None:
        self.t1 = time.perf_counter()

    def stop(self) -> dict | None:
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            return self.summary()
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            bits = sum(CLOCK_REASONS[n] for n, v in zip(names, parts[5:9]) if v.lower() == "active")
            self.samples.append((None, sm, mx, bits))
        return self.summary()

    def summary(self) -> dict | None:
        if not self.samples:
            return None
        inside = [x for x in self.samples if x[0] is not None and self.t0 is not None and
                  self.t1 is not None and self.t0 <= x[0] <= self.t1]
        use = inside or self.samples
        reasons = sorted(n for n, bit in CLOCK_REASONS.items() if any(x[3] & bit for x in use))
        return {"sm_mhz": statistics.median(x[1] for x in use),
                "sm_max_mhz": max(x[2] for x in use), "reasons": reasons,
                "samples": len(use), "source": self.source,
                "window": "timed region" if inside else "whole sampling period"}


def tensor_core_router(shape) -> bool:
    """The layer shapes whose router runs on the tensor cores (moe_route's rule)."""
    return shape.dtype == W.BF16 and shape.E > 32 and shape.d_model % 64 == 0


def route_tensor_roof(shape, work: dict, route_ms: float, peaks: dict) -> dict:
    """For the tensor-core router, the route stage against the tensor roof: it executes the
    contraction twice (x against the bf16 hi and lo terms of W_r), 4 T d E FLOP for the
    2 T d E of the definition."""
    if not tensor_core_router(shape) or route_ms <= 0:
        return {}
    executed = 2.0 * work["route_flops"]
    tf = executed / (route_ms * 1e-3) / 1e12
    return {"bound": "tensor (two bf16 terms of W_r)",
            "executed_TFLOP/s": tf, "frac_tensor": tf / peaks["bf16_tflops"],
            "algorithmic_TFLOP/s": work["route_flops"] / (route_ms * 1e-3) / 1e12}


def algorithmic_work(shape, kept_total: int) -> dict:
    T, d, f, E, k, s = (shape.T, shape.d_model, shape.d_ff, shape.E, shape.k,
                        2 if shape.dtype == W.BF16 else 4)
    A = T * k
    return {
        "gemm_flops": 6.0 * d * f * kept_total,
        "route_bytes": T * d * s + d * E * 4 + T * E * 4 + T * k * 8,
        "route_flops": 2.0 * T * d * E,
        "permute_bytes": T * d * s + kept_total * d * s + A * 4,
        "combine_bytes": kept_total * d * s + A * 8 + T * d * s,
    }


def gemm_roofline(shape, kept_total: int, touched: int, ffn_ms: float, peaks: dict,
                  power_capped: bool = False) -> dict:
    """The grouped GEMM (both launches) against the roof that binds it.  FLOPs: 6 d f per kept
    row.  Bytes: the weights of every expert that got rows (3 d f each), plus the kept rows of
    x_perm read, h written and read back, y_perm written.  The binding roof is the one whose
    time at the measured peak is longer (tensor for prefill, HBM for decode).  The tensor peak
    is the bf16 burst figure, or the sustained one when the clock record of the timed region
    shows the power cap (the GEMM then runs inside a long stretch of work at the capped clock,
    the regime the sustained figure was measured in); both fractions are reported."""
    d, f = shape.d_model, shape.d_ff
    s = 2 if shape.dtype == W.BF16 else 4
    flops = 6.0 * d * f * kept_total
    nbytes = touched * 3.0 * d * f * s + kept_total * (2.0 * d * s + 2.0 * f * s)
    sec = ffn_ms * 1e-3
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    base = {"kernel": "grouped_gemm_tc_kernel (expert FFN: gate/up + down launches)",
            "algorithmic_flops_per_step": flops, "algorithmic_bytes_per_step": nbytes,
            "experts_touched": touched}
    if t_hbm > t_tensor:
        achieved = nbytes / sec / 1e9
        base.update(bound="hbm", achieved=achieved, peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=achieved / peaks["hbm_gbs"], peak_source=f"{peaks['source']} HBM copy")
        return base
    achieved = flops / sec / 1e12
    sustained = peaks.get("bf16_tflops_sustained")
    use_sustained = power_capped and bool(sustained)
    peak = sustained if use_sustained else peaks["bf16_tflops"]
    base.update(bound="tensor", achieved=achieved, peak=peak, unit="TFLOP/s",
                frac=achieved / peak,
                peak_source=(f"{peaks['source']} bf16 sustained (sw_power_cap in the timed "
                             f"region's clock record)" if use_sustained else
                             f"{peaks['source']} bf16 burst"),
                frac_of_burst=achieved / peaks["bf16_tflops"],
                frac_of_sustained=(achieved / sustained if sustained else None))
    return base


def rank_shape(shape, rank: int):
    """Replicas draw different token batches (and weights) per rank: seed + 1000 * rank."""
    return shape.replace(seed=shape.seed + 1000 * rank) if rank else shape


def max_over_ranks(values, dist, device) -> list:
    """Element-wise max of per-rank timings (the slowest rank sets the job's time)."""
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


DROP_POLICIES = {"token": 0, "pick_rank": 1, "score": 2}


def workload_shape(args) -> "W.MoEShape":
    """The workload the command line names, with its overrides applied."""
    shape = W.WORKLOADS[args.config] if args.config else DEFAULT
    if args.tokens:
        shape = shape.replace(name=f"{shape.name}_with_T{args.tokens}", T=args.tokens)
    if args.d_ff:
        shape = shape.replace(name=f"{shape.name}_with_f{args.d_ff}", d_ff=args.d_ff)
    if args.experts:
        shape = shape.replace(name=f"{shape.name}_with_E{args.experts}", E=args.experts)
    if args.drop_policy != "token":
        shape = shape.replace(name=f"{shape.name}_drops_by_{args.drop_policy}",
                              drop_policy=DROP_POLICIES[args.drop_policy])
    return shape


def run_gpu(args) -> None:
    shape = workload_shape(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    # every rank holds a full replica; ranks draw different token batches
    mem_points = {}

    def mem_point(name):  # allocator state at the points the memory record asks for
        mem_points[name] = {"allocated_bytes": int(torch.cuda.memory_allocated(dev)),
                            "reserved_bytes": int(torch.cuda.memory_reserved(dev)),
                            "peak_allocated_bytes": int(torch.cuda.max_memory_allocated(dev))}

    inp = W.make_inputs(rank_shape(shape, rank), device=dev)
    mem_point("inputs_and_weights")
    cfg = M.config_from_shape(shape)
    ws = M.alloc_workspace(cfg, dev)
    b = M.LayerBuffers.allocate(cfg, dev, gather=args.gather)
    mem_point("layer_buffers_and_workspace")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the router weight is the layer's: its split (tensor-core router) is made once, as
    # MoELayer does, not in every step
    w_split = M.router_split(cfg, inp.w_router)

    def step(ev):
        ev[0].record(stream)
        M.moe_route_ex(cfg, inp.x, inp.w_router, w_split, inp.logit_bias, b.logits, b.topk_idx,
                       b.topk_w, ws)
        ev[1].record(stream)
        M.moe_dispatch_scored(cfg, inp.x, b.topk_idx, b.logits, inp.logit_bias, b.routed_counts,
                              b.kept_counts, b.expert_offsets, b.assign_row, b.token_of_row,
                              b.x_perm, ws)
        ev[2].record(stream)
        if args.fused_combine:
            M.moe_expert_ffn_combine(cfg, inp.x, b.x_perm, b.token_of_row, b.expert_offsets,
                                     b.kept_counts, inp.w_gate, inp.w_up, inp.w_down, b.h,
                                     b.y_perm, b.assign_row, b.topk_w, b.out, ws)
        elif args.gather:
            M.moe_expert_ffn_gather(cfg, inp.x, b.token_of_row, b.expert_offsets, b.kept_counts,
                                    inp.w_gate, inp.w_up, inp.w_down, b.h, b.y_perm, ws)
        else:
            M.moe_expert_ffn(cfg, b.x_perm, b.expert_offsets, b.kept_counts, inp.w_gate,
                             inp.w_up, inp.w_down, b.h, b.y_perm, ws)
        ev[3].record(stream)
        if not args.fused_combine:
            M.moe_combine(cfg, b.y_perm, b.assign_row, b.topk_w, b.out)
        ev[4].record(stream)
        M.moe_load_stats(cfg, b.routed_counts, b.kept_counts, b.assign_row, b.stats, host=False)
        ev[5].record(stream)

    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(args.warmup):
        flush.zero_()
        step(mk())
    M.moe_check_device_error(ws)
    mem_point("after_warmup")

    evs = [mk() for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    launches0 = M.kernel_launch_count()
    clocks.mark_start()
    for i in range(args.steps):
        flush.zero_()
        step(evs[i])
    timed_launches = M.kernel_launch_count() - launches0
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    clk = clocks.stop()
    M.moe_check_device_error(ws)

    names = ["route", "dispatch", "expert_ffn", "combine", "stats"]
    per_stage = {n: [] for n in names}
    step_ms = []
    for ev in evs:
        for j, n in enumerate(names):
            per_stage[n].append(ev[j].elapsed_time(ev[j + 1]))
        step_ms.append(ev[0].elapsed_time(ev[5]))
    total_ms = max_over_ranks([sum(step_ms)], dist, dev)[0]
    ms_per_step = total_ms / args.steps
    tensors_bytes = lambda ts: int(sum(t.numel() * t.element_size() for t in ts if t is not None))
    memory = {"weights_bytes": tensors_bytes([inp.w_router, inp.w_gate, inp.w_up, inp.w_down]),
              "layer_buffers_bytes": tensors_bytes(vars(b).values()),
              "workspace_bytes": int(ws.numel()),
              "peak_allocated_bytes": int(torch.cuda.max_memory_allocated(dev)),
              "peak_reserved_bytes": int(torch.cuda.max_memory_reserved(dev)),
              "note": "torch allocator peaks at the end of the timed region: inputs, weights, "
                      "layer buffers, workspace and the L2-flush buffer"}
    mem_point("after_timed_region")
    memory["points"] = mem_points
    stats = b.stats_dict()
    job_stats = None
    if dist:  # the job's record of the layer over the replicas (every rank takes part)
        from routing_dispatch_expert_warp_b200 import replicas as RP
        try:
            job_stats = RP.job_load_stats(cfg, b)
        except Exception as exc:  # the timing stands without the record
            job_stats = {"error": f"{type(exc).__name__}: {exc}"}
    kept_total = stats["kept_total"]
    work = algorithmic_work(shape, kept_total)
    peaks = measured_peaks()
    ffn_ms = sum(per_stage["expert_ffn"]) / args.steps
    touched = int((b.kept_counts > 0).sum())
    roof = gemm_roofline(shape, kept_total, touched, ffn_ms, peaks,
                         power_capped="sw_power_cap" in clk.get("reasons", []))
    if args.fused_combine:
        roof["kernel"] += ", the combine fused into the down launch (its time included)"
    gbs = lambda byts, n: byts / (sum(per_stage[n]) / args.steps * 1e-3) / 1e9

    # end to end through the public API: pinned host x -> device, layer, device -> host out
    layer = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias,
                       device=dev, gather=args.gather)
    x_host = inp.x.cpu().pin_memory()
    out_host = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()
    x_dev = torch.empty_like(inp.x)
    for _ in range(max(1, args.warmup)):
        x_dev.copy_(x_host, non_blocking=True)
        out_host.copy_(layer(x_dev), non_blocking=True)
    torch.cuda.synchronize(dev)
    e2e_ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        out_host.copy_(layer(x_dev), non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    e2e_total = max_over_ranks([sum(e2e_ms)], dist, dev)[0]
    M.moe_check_device_error(layer.ws)

    # the whole layer replayed as one CUDA graph (no launch gaps between the kernels)
    glayer = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias,
                        device=dev, gather=args.gather)
    gx = inp.x.clone()
    graph = glayer.capture(gx)
    for _ in range(args.warmup):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize(dev)
    g_ms = []
    for _ in range(args.steps):
        flush.zero_()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        graph.replay()
        g1.record(stream)
        g1.synchronize()
        g_ms.append(g0.elapsed_time(g1))
    graph_total = max_over_ranks([sum(g_ms)], dist, dev)[0]
    M.moe_check_device_error(glayer.ws)
    del graph, glayer, gx

    # the same through HostPipeline: batch i's upload and batch i-1's download overlap the
    # layer's kernels (two copy streams, two sets of device buffers); every step still copies
    # its input in and its output out, all inside one timed region
    pipe = M.HostPipeline(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias,
                          device=dev, depth=2)
    outs_pinned = [torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory() for _ in range(2)]
    xs_host = [x_host] * args.steps
    outs_host = [outs_pinned[i % 2] for i in range(args.steps)]
    pipe.run(xs_host[:args.warmup], outs_host[:args.warmup], stream)
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    pipe.run(xs_host, outs_host, stream)
    p1.record(stream)
    p1.synchronize()
    pipe_total = max_over_ranks([p0.elapsed_time(p1)], dist, dev)[0]
    for lyr in pipe.layers:
        M.moe_check_device_error(lyr.ws)

    if rank == 0:
        cpu = cpu_baseline(shape, args.cpu_sample_rows) if (world == 1 and not args.no_cpu) else None
        line = {
            "metric": METRIC,
            "value": shape.T * world / (ms_per_step * 1e-3),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if shape.dtype == W.BF16 else "f32",
            "data": "synthetic (seeded; x~N(0,1), weights~N(0,1/fan_in))",
            "config": {"workload": shape.name, "T": shape.T, "d_model": shape.d_model,
                       "d_ff": shape.d_ff, "E": shape.E, "k": shape.k,
                       "gating": "softmax" if shape.gating == W.SOFTMAX else "sigmoid",
                       "capacity_factor": shape.capacity_factor,
                       "drop_order": args.drop_policy,
                       "l2": "flushed between timed steps (256 MB write)",
                       "dispatch": ("no x_perm: gate/up GEMM gathers rows of x" if args.gather
                                    else "permuted copy x_perm"),
                       "combine": ("fused into the down GEMM epilogue" if args.fused_combine
                                   else "separate kernel"),
                       "ffn_kernel": {"token_n": "weight rows as M, tokens as N (tails to 16)",
                                      "token_major": "single CTAs, 128-token x 256-column tiles",
                                      "pairs": "CTA pairs, 256 x 256 tiles"}[args.ffn_kernel],
                       "parallelism": f"replicas x{world} (EP=1, no exchange)"},
            "roofline": dict(
                roof,
                traffic=(recorded_traffic(shape.name, args.gather) or {}).get("bytes"),
                traffic_source=(recorded_traffic(shape.name, args.gather) or {}).get("profile")),
            "stages_ms": {n: sum(v) / args.steps for n, v in per_stage.items()},
            "stage_bandwidth": {
                "route": dict(
                    {"GB/s": gbs(work["route_bytes"], "route"),
                     "frac_hbm": gbs(work["route_bytes"], "route") / peaks["hbm_gbs"]},
                    **route_tensor_roof(shape, work, sum(per_stage["route"]) / args.steps,
                                        peaks)),
                "dispatch": ({"us": sum(per_stage["dispatch"]) / args.steps * 1e3,
                              "note": "bookkeeping only (no copy)"} if args.gather else
                             {"GB/s": gbs(work["permute_bytes"], "dispatch"),
                              "frac_hbm": gbs(work["permute_bytes"], "dispatch") / peaks["hbm_gbs"]}),
                "combine": ({"note": "fused into the down GEMM (expert_ffn stage)"}
                            if args.fused_combine else
                            {"GB/s": gbs(work["combine_bytes"], "combine"),
                             "frac_hbm": gbs(work["combine_bytes"], "combine") / peaks["hbm_gbs"]}),
                "hbm_peak_gbs": peaks["hbm_gbs"],
            },
            "load_stats": {k2: stats[k2] for k2 in ("kept_total", "dropped", "p50", "p95", "max",
                                                    "max_to_mean")},
            "load_stats_job": (job_stats if (job_stats is None or "error" in job_stats) else
                               {k2: job_stats[k2] for k2 in ("active_tokens", "kept_total",
                                                             "dropped", "p50", "p95", "max",
                                                             "max_to_mean", "top5pct_share")}),
            "e2e": {"value": shape.T * world / (pipe_total / args.steps * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": inp.x.numel() * inp.x.element_size(),
                    "d2h_bytes_per_step": b.out.numel() * b.out.element_size(),
                    "api": "HostPipeline.run -> moe_layer_forward per batch, pinned host "
                           "buffers, copies overlapped with the previous/next batch's kernels",
                    "l2": "not flushed: the per-step working set (expert weights) exceeds L2",
                    "unpipelined": {"value": shape.T * world / (e2e_total / args.steps * 1e-3),
                                    "api": "MoELayer.forward with its copies in series, "
                                           "L2 flushed between steps"}},
            "graph": {"ms_per_step": graph_total / args.steps,
                      "tokens_per_s": shape.T * world / (graph_total / args.steps * 1e-3),
                      "api": "MoELayer.capture -> CUDA graph replay of moe_layer_forward",
                      "l2": "flushed between replays"},
            "gpu_launches": timed_launches,
            "memory": memory,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_ep_emulated(args) -> None:
    """The expert-parallel layer with args.ep_emulate ranks emulated on this one GPU: the
    workload's T tokens split evenly over the ranks (capacity per source rank), experts in
    contiguous blocks, every step of the EP schedule timed with CUDA events.  A measurement
    of the EP kernels' cost next to the single-GPU layer on the same tokens; the NVLink
    transfers of a real multi-GPU run are local copies here."""
    from routing_dispatch_expert_warp_b200 import ep as EP
    G = args.ep_emulate
    base = W.WORKLOADS[args.config] if args.config else DEFAULT
    if base.T % G or base.E % G:
        raise SystemExit("T and E must be multiples of the emulated rank count")
    shape = base.replace(name=f"{base.name}_ep{G}_emulated", T=base.T // G)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_inputs(base, device=dev)
    xs = [inp.x[r * shape.T:(r + 1) * shape.T].contiguous() for r in range(G)]
    if inp.logit_bias is not None and inp.logit_bias.dim() == 2:
        biases = [inp.logit_bias[r * shape.T:(r + 1) * shape.T].contiguous() for r in range(G)]
    else:
        biases = [inp.logit_bias] * G
    cfg = M.config_from_shape(shape)
    emu = EP.EpEmulator(cfg, G, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, biases,
                        device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = [s for s in EP.SCHEDULE if s != "barrier"] + ["end"]

    def run(evs):
        emu.forward(xs, on_step=lambda n: evs[n].record(stream))

    mk = lambda: {n: torch.cuda.Event(enable_timing=True) for n in names}
    for _ in range(args.warmup):
        flush.zero_()
        run(mk())
    for r in emu.ranks:
        M.moe_check_device_error(r.ws)
    evs = [mk() for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(0)
    time.sleep(0.3)
    clocks.mark_start()
    for i in range(args.steps):
        flush.zero_()
        run(evs[i])
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    time.sleep(0.2)
    clk = clocks.stop()
    for r in emu.ranks:
        M.moe_check_device_error(r.ws)
    per = {n: sum(e[n].elapsed_time(e[names[i + 1]]) for e in evs) / args.steps
           for i, n in enumerate(names[:-1])}
    ms = sum(e[names[0]].elapsed_time(e["end"]) for e in evs) / args.steps
    st = emu.ranks[0].stats_dict()
    row_bytes = base.d_model * (2 if base.dtype == W.BF16 else 4)
    moved = st["total_assignments"] * row_bytes          # rows written by dispatch
    x_bytes = base.T * row_bytes
    line = {
        "metric": f"MoE-layer tokens/s, expert parallel over {G} ranks emulated on 1 B200",
        "value": base.T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": "bf16" if base.dtype == W.BF16 else "f32", "data": "synthetic",
        "config": {"workload": base.name, "ranks": G, "tokens_per_rank": shape.T,
                   "placement": "contiguous", "l2": "flushed between timed steps (256 MB write)"},
        "steps_ms": per,
        "dispatch_GBps": (x_bytes + moved) / (per["dispatch"] * 1e-3) / 1e9,
        "combine_GBps": (moved + x_bytes) / (per["combine"] * 1e-3) / 1e9,
        "ep_stats": {k: st[k] for k in ("local_fraction", "remote_bytes", "pair_bytes_p50",
                                         "pair_bytes_p99", "rank_load_max_to_mean",
                                         "cross_node_fraction")},
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def ep_rank_inputs(shape, rank: int, world: int, device) -> dict:
    """This rank's part of the expert-parallel layer (weak scaling: every rank brings its own
    batch of T tokens, as the replicas do): its batch x (seed + 1000 rank); the layer's router
    weight and per-expert logit bias, the same on every rank; a per-token bias, drawn with
    the batch; and the weights of the experts it owns -- contiguous blocks of E / world --
    each from that expert's own seeded stream, so they equal the single-GPU layer's."""
    if shape.E % world:
        raise SystemExit(f"E={shape.E} is not a multiple of the {world} ranks")
    base = W.make_inputs(shape, device=device, weights=False)
    batch = W.make_inputs(rank_shape(shape, rank), device=device, weights=False) if rank else base
    per_token = batch.logit_bias is not None and batch.logit_bias.dim() == 2
    n_local = shape.E // world
    experts = list(range(rank * n_local, (rank + 1) * n_local))
    d, f, dt = shape.d_model, shape.d_ff, shape.torch_dtype
    wg = torch.empty((n_local, f, d), dtype=dt, device=device)
    wu = torch.empty((n_local, f, d), dtype=dt, device=device)
    wd = torch.empty((n_local, d, f), dtype=dt, device=device)
    for i, e in enumerate(experts):
        wg[i], wu[i], wd[i] = W.expert_weights(shape, e, device)
    return {"x": batch.x, "w_router": base.w_router,
            "logit_bias": batch.logit_bias if per_token else base.logit_bias,
            "w_gate": wg, "w_up": wu, "w_down": wd, "experts": experts}


def run_ep_group(args) -> None:
    """The expert-parallel layer over the job's GPUs, one process per GPU (torchrun; a single
    process without it): rank r owns experts [r E/N, (r+1) E/N) and its own batch of T tokens;
    dispatch and combine move rows over peer memory (CUDA IPC mappings, plain 16-byte loads
    and stores) and the steps are separated by one-element NCCL all-reduces on the stream.
    Every step of the EP schedule is timed with CUDA events; the job's time is the slowest
    rank's."""
    import datetime
    import torch.distributed as dist
    from routing_dispatch_expert_warp_b200 import ep as EP
    if "WORLD_SIZE" not in os.environ:   # one process: a one-rank group on this host
        import socket
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0",
                          WORLD_SIZE="1", LOCAL_RANK="0")
    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    shape = workload_shape(args)
    inp = ep_rank_inputs(shape, rank, world, dev)
    cfg = M.config_from_shape(shape)
    grp = EP.EpGroup(cfg, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"],
                     EP.contiguous_placement(shape.E, world, dev), inp["logit_bias"],
                     ranks_per_node=world, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = [s_ for s_ in EP.SCHEDULE if s_ != "barrier"] + ["end"]
    mk = lambda: {n: torch.cuda.Event(enable_timing=True) for n in names}
    for _ in range(args.warmup):
        flush.zero_()
        grp.forward(inp["x"])
    M.moe_check_device_error(grp.me.ws)
    evs = [mk() for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    clocks.mark_start()
    for i in range(args.steps):
        flush.zero_()
        grp.forward(inp["x"], on_step=lambda n, e=evs[i]: e[n].record(stream))
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    dist.barrier()
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    clk = clocks.stop()
    M.moe_check_device_error(grp.me.ws)
    per = {n: sum(e[n].elapsed_time(e[names[i + 1]]) for e in evs) / args.steps
           for i, n in enumerate(names[:-1])}
    mine = [sum(e[names[0]].elapsed_time(e["end"]) for e in evs) / args.steps]
    mine += [per[n] for n in names[:-1]]
    slowest = max_over_ranks(mine, dist, dev)
    ms = slowest[0]
    st = grp.me.stats_dict()
    if rank == 0:
        line = {
            "metric": f"MoE-layer tokens/s, expert parallel over {world} GPU(s)",
            "value": world * shape.T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak",
            "dtype": "bf16" if shape.dtype == W.BF16 else "f32",
            "data": "synthetic (seeded; every rank its own batch of T tokens)",
            "config": {"workload": shape.name, "T_per_rank": shape.T, "E": shape.E,
                       "experts_per_rank": shape.E // world, "placement": "contiguous",
                       "parallelism": f"EP{world}: dispatch/combine over peer memory (CUDA "
                                      "IPC), NCCL all-reduce barriers",
                       "l2": "flushed between timed steps (256 MB write)"},
            "steps_ms_max_over_ranks": dict(zip(names[:-1], slowest[1:])),
            "ep_stats": {k: st[k] for k in ("local_fraction", "remote_bytes", "pair_bytes_p50",
                                             "pair_bytes_p99", "rank_load",
                                             "rank_load_max_to_mean", "cross_node_fraction")},
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    dist.barrier()
    grp.close()
    dist.destroy_process_group()


def run_microbatch(args) -> None:
    """The layer cut into args.microbatches microbatches that ping-pong over two streams
    (with --ep-emulate G: the expert-parallel layer over G ranks emulated on this GPU, each
    rank's tokens cut the same way), timed with CUDA events against the same layer on one
    stream in the same process, plus the segments and critical path of one recorded step.
    A separate measurement, not the headline line."""
    from routing_dispatch_expert_warp_b200 import ep as EP
    from routing_dispatch_expert_warp_b200 import microbatch as MB
    m, G = args.microbatches, args.ep_emulate
    base = W.WORKLOADS[args.config] if args.config else DEFAULT
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_inputs(base, device=dev)
    if G:
        if base.T % G or base.E % G:
            raise SystemExit("T and E must be multiples of the emulated rank count")
        shape = base.replace(T=base.T // G)
        xs = [inp.x[r * shape.T:(r + 1) * shape.T].contiguous() for r in range(G)]
        if inp.logit_bias is not None and inp.logit_bias.dim() == 2:
            biases = [inp.logit_bias[r * shape.T:(r + 1) * shape.T].contiguous()
                      for r in range(G)]
        else:
            biases = [inp.logit_bias] * G
        cfg = M.config_from_shape(shape)
        pp = MB.EpMicrobatchEmulator(cfg, G, inp.w_router, inp.w_gate, inp.w_up, inp.w_down,
                                     biases, m=m, device=dev)
        one = EP.EpEmulator(cfg, G, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, biases,
                            device=dev, local_weights=[(r.w_gate, r.w_up, r.w_down)
                                                       for r in pp.emus[0].ranks])
        run_pp = lambda rec=False: pp(xs, record=rec)
        run_one = lambda: one.forward(xs)
        errs = [r.ws for e in pp.emus + [one] for r in e.ranks]
    else:
        cfg = M.config_from_shape(base)
        pp = MB.MicrobatchLayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down,
                                inp.logit_bias, m=m, device=dev)
        one = M.MoELayer(cfg, inp.w_router, inp.w_gate, inp.w_up, inp.w_down, inp.logit_bias,
                         device=dev)
        run_pp = lambda rec=False: pp(inp.x, record=rec)
        run_one = lambda: one(inp.x)
        errs = [p_["ws"] for p_ in pp.mbs] + [one.ws]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        evs = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in evs) / args.steps

    for _ in range(args.warmup):
        flush.zero_()
        run_pp()
        flush.zero_()
        run_one()
    torch.cuda.synchronize(dev)
    for ws in errs:
        M.moe_check_device_error(ws)
    clocks = ClockSampler(0)
    time.sleep(0.3)
    clocks.mark_start()
    ms_pp = timed(run_pp)
    ms_one = timed(run_one)
    clocks.mark_end()
    time.sleep(0.2)
    clk = clocks.stop()
    flush.zero_()
    run_pp(True)
    torch.cuda.synchronize(dev)
    for ws in errs:
        M.moe_check_device_error(ws)
    tl = pp.timeline()
    seg = tl["segments"]
    name = lambda n: f"mb{n[0]}:{n[1]}"
    line = {
        "metric": (f"MoE-layer tokens/s, {m} microbatches ping-ponging on two streams"
                   + (f", expert parallel over {G} ranks emulated on 1 B200" if G else "")),
        "value": base.T / (ms_pp * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_pp,
        "higher_is_better": True, "dtype": "bf16" if base.dtype == W.BF16 else "f32",
        "data": "synthetic",
        "config": {"workload": base.name, "microbatches": m, "ranks": G or 1,
                   "tokens_per_microbatch": [n for _, n in pp.parts],
                   "l2": "flushed between timed steps (256 MB write)"},
        "single_stream_ms_per_step": ms_one,
        "speedup_vs_single_stream": ms_one / ms_pp,
        "timeline": {
            "segments_ms": {name(n): [round(s_, 4), round(e_, 4)] for n, (s_, e_) in seg.items()},
            "critical_path": [name(n) for n in tl["path"]],
            "wall_ms": tl["wall"], "serial_ms": tl["serial"],
            "path_busy_ms": tl["busy"], "path_gaps_ms": tl["gaps"],
            "off_path_ms": tl["serial"] - tl["busy"],
            "stage_record": MB.stage_record(tl),
            "note": "one recorded step (events around every stage); off_path_ms is stage "
                    "time that ran beside the critical path"},
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def run_dense_calibration(args) -> None:
    """The expert FFN's GEMMs on one dense expert (E = 1: every token's row in one bucket)
    through the library's kernels and through cuBLAS (torch.mm) on the same shapes: x [T, d]
    against W_g, W_u [f, d] and h [T, f] against W_d [d, f], bf16 in, fp32 accumulate.  A
    calibration of the grouped GEMM against the vendor library, not the layer's timing."""
    T, d, f = (int(v) for v in args.dense_calibration.split(","))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    x = torch.randn(T, d, device=dev, generator=g).to(torch.bfloat16)
    wg = (torch.randn(1, f, d, device=dev, generator=g) * d ** -0.5).to(torch.bfloat16)
    wu = (torch.randn(1, f, d, device=dev, generator=g) * d ** -0.5).to(torch.bfloat16)
    wd = (torch.randn(1, d, f, device=dev, generator=g) * f ** -0.5).to(torch.bfloat16)
    h = torch.empty(T, f, device=dev, dtype=torch.bfloat16)
    y = torch.empty(T, d, device=dev, dtype=torch.bfloat16)
    flops = 6.0 * T * d * f

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) / args.steps

    def cublas():
        torch.mm(x, wg[0].t())
        torch.mm(x, wu[0].t())
        torch.mm(h, wd[0].t())

    res = {"cublas_3mm": timed(cublas)}
    cfg = M.make_config(T, d, f, 1, 1, dtype=M.BF16)
    ws = M.alloc_workspace(cfg, dev)
    offs = torch.tensor([0, T], dtype=torch.int32, device=dev)
    kept = torch.tensor([T], dtype=torch.int32, device=dev)
    for kind in ("token_major", "pairs", "token_n"):
        M.set_ffn_kernel(kind)
        res[kind] = timed(lambda: M.moe_expert_ffn(cfg, x, offs, kept, wg, wu, wd, h, y, ws))
        M.moe_check_device_error(ws)
    M.set_ffn_kernel("token_major")
    line = {"metric": "dense expert FFN GEMMs, TFLOP/s (calibration)", "T": T, "d_model": d,
            "d_ff": f, "steps": args.steps, "warmup": args.warmup,
            "ms": res, "tflops": {k: flops / v / 1e9 for k, v in res.items()}}
    print(json.dumps(line), flush=True)


def _cpu_cores() -> dict:
    """Host cores this process may run on (its affinity mask) and the threads numpy's BLAS
    pool uses, which is what the oracle's matrix products run on."""
    cores = len(os.sched_getaffinity(0))
    blas = None
    try:
        from threadpoolctl import threadpool_info
        blas = max((int(i.get("num_threads", 1)) for i in threadpool_info()), default=None)
    except Exception:
        pass
    return {"cores": cores, "blas_threads": blas}


class CpuSample:
    """The oracle as it stands, timed on the host cores on a bounded, seeded sample of the
    workload, and extrapolated to the whole layer.

    Routing (fp64 logits, fp32 top-k, capacity, slots) and the load statistics run on all T
    tokens: capacity needs them all.  The expert FFN, with the permute of its rows and its
    share of the combine, runs on a seeded sample of whole experts (every kept row of each),
    drawn until the sample holds `sample_rows` kept rows; its time is scaled by kept_total /
    kept rows in the sample.  Whole experts keep the oracle's per-row cost (each expert's
    weights are converted to fp64 once, then used for all its rows) as it is at full size,
    so the estimate does not change with the sample size.  Inputs are the workload's own
    (generated on the GPU when there is one, as the GPU path's are) copied to the host."""

    def __init__(self, shape, sample_rows: int):
        import numpy as np
        from oracle import moe_oracle as O
        self.O, self.np = O, np
        self.shape, self.sample_rows = shape, sample_rows
        src = "cuda" if torch.cuda.is_available() else "cpu"
        inp = W.make_inputs(shape, device=src, weights=False)
        host = lambda t: None if t is None else t.detach().float().cpu().numpy()
        self.x, self.w_router, self.bias = host(inp.x), host(inp.w_router), host(inp.logit_bias)
        del inp
        self.x64 = self.x.astype(np.float64)
        r = self._route()
        kept = r["kept"]
        nz = np.nonzero(kept)[0]
        order = np.random.default_rng(shape.seed).permutation(nz)
        chosen, rows = [], 0
        for e in order:
            chosen.append(int(e))
            rows += int(kept[e])
            if rows >= sample_rows:
                break
        self.experts = sorted(chosen)
        self.kept_sample, self.kept_total = rows, int(kept.sum())
        self.weights = {}
        for e in self.experts:
            wg, wu, wd = W.expert_weights(shape, e, device=src)
            self.weights[e] = (host(wg), host(wu), host(wd))
        # the sample's part of the combine: the tokens with a kept pick in the sample, their
        # other picks masked, rows renumbered into the sample's stacked FFN output
        ar = r["assign_row"]
        local = np.full(ar.shape, -1, dtype=np.int64)
        base = 0
        for e in self.experts:
            s0, n = int(r["offsets"][e]), int(kept[e])
            m = (ar >= s0) & (ar < s0 + n)
            local[m] = ar[m] - s0 + base
            base += n
        self.tokens = np.nonzero((local >= 0).any(axis=1))[0]
        self.local = local[self.tokens]

    def _route(self):
        O, s = self.O, self.shape
        sel_only = s.bias_mode == O.BIAS_SELECTION_ONLY
        z64 = O.router_logits(self.x, self.w_router, None if sel_only else self.bias)
        z32 = O.logits_to_fp32(z64)
        return O.route(z32, s.k, s.gating, float(self.np.float32(s.capacity_factor)), s.layout,
                       s.n_groups, s.topk_groups, self.bias if sel_only else None, s.bias_mode,
                       s.drop_policy)

    def sample_outputs(self, r):
        """The sample's FFN and combine: for the tokens with a kept pick among the sampled
        experts, the gate-weighted sum of those picks' expert outputs (other picks left out)."""
        O, np = self.O, self.np
        ys = []
        for e in self.experts:
            s0, n = int(r["offsets"][e]), int(r["kept"][e])
            x_rows = O.permute(self.x64, r["token_of_row"][s0:s0 + n])
            _, y = O.swiglu_expert(x_rows, *self.weights[e])
            ys.append(y)
        return O.combine(np.concatenate(ys), self.local, r["w"][self.tokens])

    def run(self) -> dict:
        O = self.O
        t0 = time.perf_counter()
        r = self._route()
        t1 = time.perf_counter()
        self.sample_outputs(r)
        t2 = time.perf_counter()
        O.load_stats(r["routed"], r["kept"], r["assign_row"], r["C"])
        t3 = time.perf_counter()
        scale = self.kept_total / max(self.kept_sample, 1)
        est = (t1 - t0) + (t2 - t1) * scale + (t3 - t2)
        cores = _cpu_cores()
        return {"value": self.shape.T / est, "unit": "tokens/s", "cores": cores["cores"],
                "blas_threads": cores["blas_threads"], "kind": "oracle",
                "seconds_measured": t3 - t0, "seconds_extrapolated": est,
                "sample": (f"{self.shape.name}: oracle routing and load statistics on all "
                           f"{self.shape.T} tokens; permute + expert FFN + combine on "
                           f"{len(self.experts)} seeded experts holding {self.kept_sample} of "
                           f"{self.kept_total} kept rows, time scaled by {scale:.2f} "
                           f"(extrapolated); fp64 numpy")}


def cpu_baseline(shape, sample_rows: int, repeats: int = 3) -> dict:
    """One untimed run, then the median of `repeats` timed runs."""
    cs = CpuSample(shape, sample_rows)
    cs.run()
    vals = [cs.run() for _ in range(repeats)]
    out = dict(vals[0])
    out["value"] = statistics.median(v["value"] for v in vals)
    return out


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape = workload_shape(args)
    sample = CpuSample(shape, args.cpu_sample_rows)
    for _ in range(args.warmup):
        sample.run()
    vals = [sample.run() for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": shape.T / v * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": shape.name, "T": shape.T, "d_model": shape.d_model,
                   "d_ff": shape.d_ff, "E": shape.E, "k": shape.k,
                   "gating": "softmax" if shape.gating == W.SOFTMAX else "sigmoid",
                   "capacity_factor": shape.capacity_factor, "drop_order": args.drop_policy},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[0]["cores"],
                         "blas_threads": vals[0]["blas_threads"], "kind": "oracle",
                         "sample": vals[0]["sample"]},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=None, choices=sorted(W.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T of the workload (small profiling cases)")
    ap.add_argument("--d-ff", type=int, default=0,
                    help="override d_ff of the workload (small profiling cases of the router "
                         "and dispatch kernels)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E of the workload (small profiling cases with the full "
                         "per-expert GEMM shapes)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-sample-rows", type=int, default=2048,
                    help="kept rows of the seeded expert sample the CPU oracle's FFN runs on "
                         "(both the cpu_baseline leg and --impl reference)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--ep-emulate", type=int, default=0,
                    help="time the expert-parallel layer with this many ranks emulated on one "
                         "GPU (a separate measurement, not the headline line)")
    ap.add_argument("--dense-calibration", default="",
                    help="T,d,f: time the FFN's three GEMMs on one dense expert through each "
                         "FFN kernel and through cuBLAS (a calibration, not the headline line)")
    ap.add_argument("--ep", action="store_true",
                    help="time the expert-parallel layer across the job's GPUs (one process per "
                         "GPU under torchrun): experts split in contiguous blocks, every rank "
                         "its own batch (a separate measurement, not the headline line)")
    ap.add_argument("--fused-combine", action="store_true",
                    help="time the expert FFN with the combine fused into its down GEMM")
    ap.add_argument("--gather", action="store_true",
                    help="dispatch without the permuted copy: the gate/up GEMM gathers rows of x")
    ap.add_argument("--microbatches", type=int, default=1,
                    help="time the layer as this many microbatches ping-ponging over two "
                         "streams against the one-stream layer (a separate measurement)")
    ap.add_argument("--ffn-kernel", default="token_major",
                    choices=["token_major", "token_n", "pairs"],
                    help="the plain expert FFN kernel: 128-token x 256-column tiles, weight rows "
                         "as the MMA's M and tokens as its N (tails rounded to 16 tokens), or "
                         "256 x 256 tiles on CTA pairs")
    ap.add_argument("--drop-policy", default="token", choices=sorted(DROP_POLICIES),
                    help="which picks an overflowing expert keeps: token order, pick rank "
                         "first, or highest selection score")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)   # at least three untimed warm-up steps
    if args.impl != "reference":
        M.set_ffn_kernel(args.ffn_kernel)
    if args.impl == "reference":
        run_reference(args)
    elif args.microbatches > 1:
        run_microbatch(args)
    elif args.dense_calibration:
        run_dense_calibration(args)
    elif args.ep:
        run_ep_group(args)
    elif args.ep_emulate:
        run_ep_emulated(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
