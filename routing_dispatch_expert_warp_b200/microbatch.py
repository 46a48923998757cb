"""Microbatch ping-pong on two streams, and the critical path of the layer.

"MegaScale-Infer: expert parallelism", slide 8: microbatches take turns through the stages, so
that no stage waits idle for the next one.  "MoE expert parallelism needs measurements before
launch", "Synchronise the measurement correctly": a profile has to give every segment's
duration and the critical path of the layer.

The layer's tokens are cut into m microbatches of consecutive tokens.  Microbatch i runs all
stages of the layer on stream i % 2, with its own buffers and workspace.  It starts once
microbatch i-1 has entered its expert FFN.  So the front of one microbatch runs under the
other's tensor-core FFN: route and dispatch on one GPU, and under expert parallelism also the
count exchange and the dispatch into the owners' buffers.  The back (combine, statistics) runs
under the next microbatch's FFN in the same way.

Each microbatch's result is the layer run on that microbatch alone.  Where there is a capacity,
each microbatch applies it to its own T, just as each source rank does under expert
parallelism.  With no capacity, the outputs equal the whole batch's layer bit for bit, because
the FFN is row-wise and the combine sums each token's rows in pick order.

The host only enqueues work and records events: it never waits on the GPU inside forward().
"""
from __future__ import annotations

import copy
from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import (LayerBuffers, alloc_workspace, moe_combine, moe_dispatch_scored, moe_expert_ffn,
               moe_load_stats, moe_route, F32)

STAGES = ("route", "dispatch", "expert_ffn", "combine", "stats")


def split_tokens(T: int, m: int) -> List[Tuple[int, int]]:
    """(first token, token count) of each of m microbatches of consecutive tokens; the first
    T % m microbatches hold one token more than the others."""
    if not 1 <= m <= T:
        raise ValueError("need 1 <= m <= T microbatches")
    base, extra = divmod(T, m)
    out, start = [], 0
    for i in range(m):
        n = base + (1 if i < extra else 0)
        out.append((start, n))
        start += n
    return out


def pingpong_deps(m: int, stages: Sequence[str], stagger_after: str) -> Dict[tuple, List[tuple]]:
    """What each (microbatch, stage) segment of the ping-pong waits for: its microbatch's
    previous stage; for a first stage, the previous microbatch's `stagger_after` stage (the
    stagger) and the last stage of the microbatch before that, which ran on the same stream."""
    deps: Dict[tuple, List[tuple]] = {}
    for i in range(m):
        for k, name in enumerate(stages):
            d = []
            if k > 0:
                d.append((i, stages[k - 1]))
            else:
                if i >= 1:
                    d.append((i - 1, stagger_after))
                if i >= 2:
                    d.append((i - 2, stages[-1]))
            deps[(i, name)] = d
    return deps


def critical_path(intervals: Dict[tuple, Tuple[float, float]],
                  deps: Dict[tuple, Sequence[tuple]]) -> dict:
    """The chain of segments that sets the end time.

    intervals: segment -> (start, end) on one clock.  deps: segment -> the segments that must
    finish before it may start (the previous stage of its microbatch, the stagger, the previous
    work on its stream).  From the segment that ends last, walk back each time to the
    dependency that ended last: that one held the segment back.  Returns the chain in time
    order, the wall time (last end - first start), the sum of all segment durations (the time
    one stream would need with no overlap), the chain's busy time and its gaps (time on the
    path where the chain's next segment had not started yet: launch gaps and waits)."""
    if not intervals:
        return {"path": [], "wall": 0.0, "serial": 0.0, "busy": 0.0, "gaps": 0.0}
    first = min(s for s, _ in intervals.values())
    last = max(intervals, key=lambda n: (intervals[n][1], str(n)))
    path = [last]
    while True:
        ds = [d for d in deps.get(path[-1], ()) if d in intervals]
        if not ds:
            break
        path.append(max(ds, key=lambda n: (intervals[n][1], str(n))))
    path.reverse()
    busy = sum(intervals[n][1] - intervals[n][0] for n in path)
    wall = intervals[last][1] - first
    return {"path": path, "wall": wall,
            "serial": sum(e - s for s, e in intervals.values()),
            "busy": busy, "gaps": wall - busy}


# The per-stage record of "MoE expert parallelism needs measurements before launch",
# "Profile all-to-all separately from compute": router, pack, dispatch, expert compute,
# combine and unpack times.  Stage names of this library -> the record's fields.  With the
# experts local, pack and dispatch are one stage (bookkeeping + permute), and so are combine
# and unpack; under expert parallelism the count exchange and the plan are the pack.
RECORD_FIELDS = {"route": "router_ms", "rank": "pack_ms", "put_counts": "pack_ms",
                 "plan": "pack_ms", "dispatch": "dispatch_ms", "expert_ffn": "expert_compute_ms",
                 "combine": "combine_ms", "stats": "stats_ms"}


def stage_record(timeline: dict) -> dict:
    """The per-stage record of one recorded forward: each field is the summed duration of
    its stages over the microbatches (ms), plus the wall time and the critical path's
    busy time and gaps."""
    rec = {f: 0.0 for f in dict.fromkeys(RECORD_FIELDS.values())}
    for (_, name), (s, e) in timeline["segments"].items():
        rec[RECORD_FIELDS[name]] += e - s
    rec.update(wall_ms=timeline["wall"], critical_path_busy_ms=timeline["busy"],
               critical_path_gaps_ms=timeline["gaps"])
    return rec


class MicrobatchLayer:
    """One MoE layer on one GPU, run as m microbatches ping-ponging over two streams.

    forward(x) enqueues everything and returns the [T, d_model] output (each microbatch
    writes its own rows).  With record=True it also records an event around every stage;
    timeline() then gives each segment's interval and the critical path."""

    def __init__(self, cfg, w_router, w_gate, w_up, w_down, logit_bias=None, m: int = 2,
                 device="cuda"):
        self.device = torch.device(device)
        self.cfg = cfg
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.parts = split_tokens(cfg.T, m)
        dt = torch.float32 if cfg.dtype == F32 else torch.bfloat16
        self.out = torch.empty((cfg.T, cfg.d_model), dtype=dt, device=self.device)
        self.mbs = []
        for start, n in self.parts:
            c = copy.copy(cfg)
            c.T = n
            bufs = LayerBuffers.allocate(c, self.device)
            bufs.out = self.out[start:start + n]     # rows of the shared output, no copy
            bias = logit_bias
            if logit_bias is not None and logit_bias.dim() == 2:
                bias = logit_bias[start:start + n]
            self.mbs.append({"cfg": c, "ws": alloc_workspace(c, self.device), "bufs": bufs,
                             "bias": bias, "start": start, "T": n})
        self.streams = [torch.cuda.Stream(self.device), torch.cuda.Stream(self.device)]
        self._events: Optional[dict] = None

    def _stage(self, i: int, name: str, x: torch.Tensor, st) -> None:
        mb = self.mbs[i]
        c, b, ws = mb["cfg"], mb["bufs"], mb["ws"]
        if name == "route":
            moe_route(c, x, self.w_router, mb["bias"], b.logits, b.topk_idx, b.topk_w, ws, st)
        elif name == "dispatch":
            moe_dispatch_scored(c, x, b.topk_idx, b.logits, mb["bias"], b.routed_counts,
                                b.kept_counts, b.expert_offsets, b.assign_row, b.token_of_row,
                                b.x_perm, ws, st)
        elif name == "expert_ffn":
            moe_expert_ffn(c, b.x_perm, b.expert_offsets, b.kept_counts, self.w_gate, self.w_up,
                           self.w_down, b.h, b.y_perm, ws, st)
        elif name == "combine":
            moe_combine(c, b.y_perm, b.assign_row, b.topk_w, b.out, st)
        elif name == "stats":
            moe_load_stats(c, b.routed_counts, b.kept_counts, b.assign_row, b.stats, host=False,
                           stream=st)

    def forward(self, x: torch.Tensor, stream=None, record: bool = False) -> torch.Tensor:
        comp = stream or torch.cuda.current_stream(self.device)
        ev = (lambda: torch.cuda.Event(enable_timing=True)) if record else torch.cuda.Event
        begin = ev()
        begin.record(comp)
        for s in self.streams:
            s.wait_event(begin)
        marks: Dict[tuple, torch.cuda.Event] = {}
        entered_ffn: List[torch.cuda.Event] = []
        for i, mb in enumerate(self.mbs):
            st = self.streams[i % 2]
            if i > 0:
                st.wait_event(entered_ffn[i - 1])
            xi = x[mb["start"]:mb["start"] + mb["T"]]
            for name in STAGES:
                if name == "expert_ffn":
                    e = ev()
                    e.record(st)
                    entered_ffn.append(e)
                if record:
                    marks[(i, name, "start")] = e = ev()
                    e.record(st)
                self._stage(i, name, xi, st)
                if record:
                    marks[(i, name, "end")] = e = ev()
                    e.record(st)
        for s in self.streams:
            done = torch.cuda.Event()
            done.record(s)
            comp.wait_event(done)
        self._events = {"begin": begin, "marks": marks} if record else None
        return self.out

    __call__ = forward

    def dependencies(self) -> Dict[tuple, List[tuple]]:
        return pingpong_deps(len(self.mbs), STAGES, "dispatch")

    def timeline(self) -> dict:
        """After a recorded forward has finished (synchronise first): every segment's
        (start, end) in ms from the forward's first event, and critical_path() over them."""
        if self._events is None:
            raise RuntimeError("call forward(x, record=True) and synchronise first")
        b, marks = self._events["begin"], self._events["marks"]
        iv = {}
        for i in range(len(self.mbs)):
            for name in STAGES:
                iv[(i, name)] = (b.elapsed_time(marks[(i, name, "start")]),
                                 b.elapsed_time(marks[(i, name, "end")]))
        cp = critical_path(iv, self.dependencies())
        return {"segments": iv, **cp}

    def stats_dicts(self) -> List[dict]:
        return [mb["bufs"].stats_dict() for mb in self.mbs]


class EpMicrobatchEmulator:
    """The expert-parallel layer with `world` ranks emulated on one GPU (ep.EpEmulator), each
    rank's tokens cut into m microbatches that ping-pong over two streams: while microbatch
    i-1 runs its experts, microbatch i routes, exchanges counts and dispatches its rows into
    the owners' buffers; microbatch i-1 combines from the owners' buffers while microbatch i
    computes.  One EpEmulator per microbatch (own buffers and receive areas); the ranks' local
    expert weights are sliced once and shared.  forward(xs) returns each rank's [T, d_model]
    output."""

    def __init__(self, cfg, world: int, w_router, w_gate, w_up, w_down,
                 logit_biases: Optional[Sequence] = None, m: int = 2, expert_rank=None,
                 ranks_per_node: int = 1, device="cuda"):
        from .ep import EpEmulator, SCHEDULE
        self.device = torch.device(device)
        self.steps = [s for s in SCHEDULE if s != "barrier"]
        self.parts = split_tokens(cfg.T, m)
        dt = torch.float32 if cfg.dtype == F32 else torch.bfloat16
        self.outs = [torch.empty((cfg.T, cfg.d_model), dtype=dt, device=self.device)
                     for _ in range(world)]
        self.emus = []
        shared = None
        for start, n in self.parts:
            c = copy.copy(cfg)
            c.T = n
            biases = None
            if logit_biases is not None:
                biases = [b if (b is None or b.dim() == 1) else b[start:start + n]
                          for b in logit_biases]
            emu = EpEmulator(c, world, w_router, w_gate, w_up, w_down, biases, expert_rank,
                             ranks_per_node, None, device, local_weights=shared)
            shared = [(r.w_gate, r.w_up, r.w_down) for r in emu.ranks]
            for g, r in enumerate(emu.ranks):
                r.bufs.out = self.outs[g][start:start + n]
            self.emus.append(emu)
        self.streams = [torch.cuda.Stream(self.device), torch.cuda.Stream(self.device)]
        self._events: Optional[dict] = None

    def forward(self, xs: Sequence[torch.Tensor], stream=None,
                record: bool = False) -> List[torch.Tensor]:
        comp = stream or torch.cuda.current_stream(self.device)
        ev = (lambda: torch.cuda.Event(enable_timing=True)) if record else torch.cuda.Event
        begin = ev()
        begin.record(comp)
        for s in self.streams:
            s.wait_event(begin)
        marks: Dict[tuple, torch.cuda.Event] = {}
        entered_ffn: List[torch.cuda.Event] = []
        for i, ((start, n), emu) in enumerate(zip(self.parts, self.emus)):
            st = self.streams[i % 2]
            if i > 0:
                st.wait_event(entered_ffn[i - 1])

            def on_step(name, i=i, st=st):
                if name == "expert_ffn":
                    e = ev()
                    e.record(st)
                    entered_ffn.append(e)
                if record:
                    e = ev()
                    e.record(st)
                    marks[(i, name)] = e

            emu.forward([x[start:start + n] for x in xs], st, on_step)
        for s in self.streams:
            done = torch.cuda.Event()
            done.record(s)
            comp.wait_event(done)
        self._events = {"begin": begin, "marks": marks} if record else None
        return self.outs

    __call__ = forward

    def dependencies(self) -> Dict[tuple, List[tuple]]:
        return pingpong_deps(len(self.emus), self.steps, "dispatch")

    def timeline(self) -> dict:
        """As MicrobatchLayer.timeline(): a step's segment runs from its mark to the next."""
        if self._events is None:
            raise RuntimeError("call forward(xs, record=True) and synchronise first")
        b, marks = self._events["begin"], self._events["marks"]
        names = self.steps + ["end"]
        iv = {}
        for i in range(len(self.emus)):
            for k, name in enumerate(self.steps):
                iv[(i, name)] = (b.elapsed_time(marks[(i, name)]),
                                 b.elapsed_time(marks[(i, names[k + 1])]))
        return {"segments": iv, **critical_path(iv, self.dependencies())}
