"""B200-native MoE layer forward (route -> dispatch -> SwiGLU grouped GEMM -> combine ->
load statistics) behind the C-ABI library libmoe.so.

This package is the thin Python binding: it turns torch tensors into pointers and sizes
and calls the entry points of include/moe.h under the same names.  Every step of the layer
runs in the library's CUDA kernels; PyTorch only provides device memory and streams.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _abi
from ._abi import MoEError, MoeConfig, MoeLayerBuffers, MoeLayerInputs, MoeLoadStats, check

SOFTMAX, SIGMOID = 0, 1
COMPACT, PADDED = 0, 1
F32, BF16 = 0, 1
BIAS_SCORE_AND_WEIGHT, BIAS_SELECTION_ONLY = 0, 1
DROP_TOKEN_ORDER, DROP_PICK_RANK, DROP_SCORE = 0, 1, 2

__all__ = ["MoEError", "make_config", "workspace_size", "capacity", "max_rows",
           "alloc_workspace", "moe_route", "moe_route_ex", "router_split_size", "router_split",
           "moe_dispatch", "moe_dispatch_scored",
           "moe_dispatch_static_scratch", "moe_static_scratch_check", "moe_pick_rank_counts",
           "moe_expert_ffn", "moe_expert_ffn_gather", "moe_expert_ffn_combine", "moe_combine",
           "moe_load_stats", "moe_load_stats_merge", "moe_layer_forward",
           "moe_check_device_error",
           "moe_selftest_bounded_wait", "set_wait_limit_ns", "set_ffn_kernel", "kernel_launch_count",
           "LayerBuffers", "MoELayer", "HostPipeline"]


def _lib():
    return _abi.lib()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_config(T: int, d_model: int, d_ff: int, E: int, k: int, gating: int = SOFTMAX,
                capacity_factor: float = 0.0, layout: int = COMPACT, dtype: int = BF16,
                n_groups: int = 0, topk_groups: int = 0, bias_mode: int = BIAS_SCORE_AND_WEIGHT,
                drop_policy: int = DROP_TOKEN_ORDER) -> MoeConfig:
    return MoeConfig(T=T, d_model=d_model, d_ff=d_ff, E=E, k=k, gating=gating, layout=layout,
                     dtype=dtype, capacity_factor=capacity_factor, n_groups=n_groups,
                     topk_groups=topk_groups, bias_mode=bias_mode, drop_policy=drop_policy)


def config_from_shape(shape) -> MoeConfig:
    """moe_config_t for a workload.MoEShape."""
    return make_config(shape.T, shape.d_model, shape.d_ff, shape.E, shape.k, shape.gating,
                       shape.capacity_factor, shape.layout, shape.dtype, shape.n_groups,
                       shape.topk_groups, shape.bias_mode, shape.drop_policy)


def workspace_size(cfg: MoeConfig) -> int:
    n = ctypes.c_size_t(0)
    check(_lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def capacity(cfg: MoeConfig) -> int:
    return _lib().moe_capacity(ctypes.byref(cfg))


def max_rows(cfg: MoeConfig) -> int:
    r = _lib().moe_max_rows(ctypes.byref(cfg))
    if r < 0:
        raise MoEError(1, _lib().moe_last_error().decode())
    return r


def alloc_workspace(cfg: MoeConfig, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(workspace_size(cfg), dtype=torch.uint8, device=device)
    check(_lib().moe_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))
    return ws


def set_wait_limit_ns(ns: int) -> None:
    _lib().moe_set_wait_limit_ns(ns)


FFN_TOKEN_MAJOR, FFN_CTA_PAIRS, FFN_TOKEN_N = 0, 1, 2
FFN_KERNELS = {"token_n": FFN_TOKEN_N, "token_major": FFN_TOKEN_MAJOR, "pairs": FFN_CTA_PAIRS}


def set_ffn_kernel(kind) -> None:
    """Which kernel runs the plain expert FFN, process-wide: FFN_TOKEN_MAJOR (the default),
    FFN_TOKEN_N or FFN_CTA_PAIRS, or their names in FFN_KERNELS."""
    check(_lib().moe_set_ffn_kernel(FFN_KERNELS.get(kind, kind)))


# ------------------------------------------------------------------ stages
def moe_route(cfg, x, w_router, logit_bias, logits, topk_idx, topk_w, ws, stream=None):
    stride = 0 if (logit_bias is None or logit_bias.dim() == 1) else logit_bias.shape[1]
    check(_lib().moe_route(ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(logit_bias), stride,
                           _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel(),
                           _stream(stream)))


def moe_route_ex(cfg, x, w_router, w_router_split, logit_bias, logits, topk_idx, topk_w, ws,
                 stream=None):
    """moe_route reading a split router weight made by router_split (or None: moe_route)."""
    stride = 0 if (logit_bias is None or logit_bias.dim() == 1) else logit_bias.shape[1]
    check(_lib().moe_route_ex(ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(w_router_split),
                              _ptr(logit_bias), stride, _ptr(logits), _ptr(topk_idx),
                              _ptr(topk_w), _ptr(ws), ws.numel(), _stream(stream)))


def router_split_size(cfg) -> int:
    """Bytes of the split router weight for cfg (0: the layer never uses the tensor-core
    router)."""
    n = ctypes.c_size_t(0)
    check(_lib().moe_router_split_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def router_split(cfg, w_router, stream=None) -> Optional[torch.Tensor]:
    """The split router weight of w_router (a uint8 device tensor), or None when the layer
    never uses the tensor-core router.  It stays valid while w_router is unchanged."""
    n = router_split_size(cfg)
    if n == 0:
        return None
    out = torch.empty(n, dtype=torch.uint8, device=w_router.device)
    check(_lib().moe_router_split(ctypes.byref(cfg), _ptr(w_router), _ptr(out), n,
                                  _stream(stream)))
    return out


def moe_dispatch(cfg, x, topk_idx, routed_counts, kept_counts, expert_offsets, assign_row,
                 token_of_row, x_perm, ws, stream=None):
    check(_lib().moe_dispatch(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(routed_counts),
                              _ptr(kept_counts), _ptr(expert_offsets), _ptr(assign_row),
                              _ptr(token_of_row), _ptr(x_perm), _ptr(ws), ws.numel(),
                              _stream(stream)))


def moe_dispatch_scored(cfg, x, topk_idx, logits, logit_bias, routed_counts, kept_counts,
                        expert_offsets, assign_row, token_of_row, x_perm, ws, stream=None):
    """moe_dispatch with the selection scores (needed for DROP_SCORE): logits [T, E] fp32
    as moe_route wrote them, logit_bias None, [E] or [T, >=E] fp32 as given to moe_route."""
    stride = 0 if (logit_bias is None or logit_bias.dim() == 1) else logit_bias.shape[1]
    check(_lib().moe_dispatch_scored(
        ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(logits), _ptr(logit_bias), stride,
        _ptr(routed_counts), _ptr(kept_counts), _ptr(expert_offsets), _ptr(assign_row),
        _ptr(token_of_row), _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)))


def moe_pick_rank_counts(cfg, topk_idx, assign_row, ws, group_of_expert=None, stream=None):
    """Second-choice counters: returns (routed [k, E], kept [k, E], differs [k]) int32 device
    tensors, enqueued on the stream (see include/moe.h)."""
    dev = topk_idx.device
    routed = torch.empty((cfg.k, cfg.E), dtype=torch.int32, device=dev)
    kept = torch.empty((cfg.k, cfg.E), dtype=torch.int32, device=dev)
    differs = torch.empty(cfg.k, dtype=torch.int32, device=dev)
    check(_lib().moe_pick_rank_counts(
        ctypes.byref(cfg), _ptr(topk_idx), _ptr(assign_row), _ptr(group_of_expert),
        _ptr(routed), _ptr(kept), _ptr(differs), _ptr(ws), ws.numel(), _stream(stream)))
    return routed, kept, differs


def moe_dispatch_static_scratch(cfg, x, topk_idx, routed_counts, kept_counts, expert_offsets,
                                assign_row, token_of_row, x_perm, stream=None):
    """moe_dispatch for callers that cannot allocate device memory: no workspace argument;
    the library's fixed device scratch is used instead (see include/moe.h for the limit and
    for why concurrent calls must be ordered)."""
    check(_lib().moe_dispatch_static_scratch(
        ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(routed_counts), _ptr(kept_counts),
        _ptr(expert_offsets), _ptr(assign_row), _ptr(token_of_row), _ptr(x_perm),
        _stream(stream)))


def moe_expert_ffn(cfg, x_perm, expert_offsets, kept_counts, w_gate, w_up, w_down, h, y_perm,
                   ws, stream=None):
    check(_lib().moe_expert_ffn(ctypes.byref(cfg), _ptr(x_perm), _ptr(expert_offsets),
                                _ptr(kept_counts), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                _ptr(h), _ptr(y_perm), _ptr(ws), ws.numel(), _stream(stream)))


def moe_expert_ffn_gather(cfg, x, token_of_row, expert_offsets, kept_counts, w_gate, w_up,
                          w_down, h, y_perm, ws, stream=None):
    """moe_expert_ffn reading bucket row r as x[token_of_row[r]] (no permuted copy of x)."""
    check(_lib().moe_expert_ffn_gather(ctypes.byref(cfg), _ptr(x), _ptr(token_of_row),
                                       _ptr(expert_offsets), _ptr(kept_counts), _ptr(w_gate),
                                       _ptr(w_up), _ptr(w_down), _ptr(h), _ptr(y_perm),
                                       _ptr(ws), ws.numel(), _stream(stream)))


def moe_expert_ffn_combine(cfg, x, x_perm, token_of_row, expert_offsets, kept_counts, w_gate,
                           w_up, w_down, h, y_perm, assign_row, topk_w, out, ws, stream=None):
    """Expert FFN with the combine fused into the down GEMM (x_perm None: gather rows of x)."""
    check(_lib().moe_expert_ffn_combine(ctypes.byref(cfg), _ptr(x), _ptr(x_perm),
                                        _ptr(token_of_row), _ptr(expert_offsets),
                                        _ptr(kept_counts), _ptr(w_gate), _ptr(w_up),
                                        _ptr(w_down), _ptr(h), _ptr(y_perm), _ptr(assign_row),
                                        _ptr(topk_w), _ptr(out), _ptr(ws), ws.numel(),
                                        _stream(stream)))


def moe_combine(cfg, y_perm, assign_row, topk_w, out, stream=None):
    check(_lib().moe_combine(ctypes.byref(cfg), _ptr(y_perm), _ptr(assign_row), _ptr(topk_w),
                             _ptr(out), _stream(stream)))


def stats_buffer(device="cuda") -> torch.Tensor:
    return torch.zeros(ctypes.sizeof(MoeLoadStats), dtype=torch.uint8, device=device)


def moe_load_stats(cfg, routed_counts, kept_counts, assign_row, dev_out, host: bool = True,
                   stream=None) -> Optional[dict]:
    hs = MoeLoadStats()
    check(_lib().moe_load_stats(ctypes.byref(cfg), _ptr(routed_counts), _ptr(kept_counts),
                                _ptr(assign_row), _ptr(dev_out),
                                ctypes.byref(hs) if host else None, _stream(stream)))
    return hs.as_dict() if host else None


def moe_load_stats_merge(cfg, routed_sum, kept_sum, parts, dev_out, host: bool = True,
                         stream=None) -> Optional[dict]:
    """The job record of data-parallel replicas: routed_sum / kept_sum [E] int32 (summed over
    the replicas), parts [n, sizeof(moe_load_stats_t)] uint8 (their records)."""
    hs = MoeLoadStats()
    check(_lib().moe_load_stats_merge(ctypes.byref(cfg), _ptr(routed_sum), _ptr(kept_sum),
                                      _ptr(parts), int(parts.shape[0]), _ptr(dev_out),
                                      ctypes.byref(hs) if host else None, _stream(stream)))
    return hs.as_dict() if host else None


def moe_layer_forward(cfg, inputs: MoeLayerInputs, bufs: MoeLayerBuffers, ws, stream=None):
    check(_lib().moe_layer_forward(ctypes.byref(cfg), ctypes.byref(inputs), ctypes.byref(bufs),
                                   _ptr(ws), ws.numel(), _stream(stream)))


def moe_static_scratch_check(stream=None):
    """Report (MoEError) and clear the kernel-side errors recorded by
    moe_dispatch_static_scratch since the last check; allocates nothing."""
    check(_lib().moe_static_scratch_check(_stream(stream)))


def moe_check_device_error(ws, stream=None):
    check(_lib().moe_check_device_error(_ptr(ws), ws.numel(), _stream(stream)))


def moe_selftest_bounded_wait(ws, stream=None):
    check(_lib().moe_selftest_bounded_wait(_ptr(ws), ws.numel(), _stream(stream)))


def kernel_launch_count() -> int:
    """Kernels the library has launched in this process so far (all devices and streams)."""
    return int(_lib().moe_kernel_launch_count())


# ------------------------------------------------------------------ whole layer
@dataclass
class LayerBuffers:
    """Every output and intermediate of one layer forward, allocated with torch."""
    logits: torch.Tensor
    topk_idx: torch.Tensor
    topk_w: torch.Tensor
    routed_counts: torch.Tensor
    kept_counts: torch.Tensor
    expert_offsets: torch.Tensor
    assign_row: torch.Tensor
    token_of_row: torch.Tensor
    x_perm: Optional[torch.Tensor]   # None: the gate/up GEMM gathers rows of x
    h: torch.Tensor
    y_perm: torch.Tensor
    out: torch.Tensor
    stats: torch.Tensor

    @staticmethod
    def allocate(cfg: MoeConfig, device="cuda", gather: bool = False) -> "LayerBuffers":
        T, d, f, E, k = cfg.T, cfg.d_model, cfg.d_ff, cfg.E, cfg.k
        R = max_rows(cfg)
        dt = torch.float32 if cfg.dtype == F32 else torch.bfloat16
        i32 = dict(dtype=torch.int32, device=device)
        return LayerBuffers(
            logits=torch.empty((T, E), dtype=torch.float32, device=device),
            topk_idx=torch.empty((T, k), **i32), topk_w=torch.empty((T, k), dtype=torch.float32,
                                                                    device=device),
            routed_counts=torch.empty(E, **i32), kept_counts=torch.empty(E, **i32),
            expert_offsets=torch.empty(E + 1, **i32), assign_row=torch.empty((T, k), **i32),
            token_of_row=torch.empty(max(R, 1), **i32),
            x_perm=None if gather else torch.empty((max(R, 1), d), dtype=dt, device=device),
            h=torch.empty((max(R, 1), f), dtype=dt, device=device),
            y_perm=torch.empty((max(R, 1), d), dtype=dt, device=device),
            out=torch.empty((T, d), dtype=dt, device=device),
            stats=stats_buffer(device))

    def as_struct(self, with_stats: bool = True) -> MoeLayerBuffers:
        return MoeLayerBuffers(
            logits=_ptr(self.logits), topk_idx=_ptr(self.topk_idx), topk_w=_ptr(self.topk_w),
            routed_counts=_ptr(self.routed_counts), kept_counts=_ptr(self.kept_counts),
            expert_offsets=_ptr(self.expert_offsets), assign_row=_ptr(self.assign_row),
            token_of_row=_ptr(self.token_of_row), x_perm=_ptr(self.x_perm), h=_ptr(self.h),
            y_perm=_ptr(self.y_perm), out=_ptr(self.out),
            stats=_ptr(self.stats) if with_stats else None)

    def stats_dict(self) -> dict:
        raw = bytes(self.stats.cpu().numpy().tobytes())
        return MoeLoadStats.from_buffer_copy(raw).as_dict()


class MoELayer:
    """One MoE layer with resident weights: the public entry point for a forward pass.

    forward(x) enqueues the whole layer (moe_layer_forward) on the current stream and
    returns the output tensor (a view of the layer's own buffer, overwritten by the next
    call).  gather=True drops the permuted copy of x: dispatch only ranks the assignments
    and the gate/up GEMM gathers its rows from x (same results and less memory, but slower
    than the permuted copy on B200).

    The split router weight of the tensor-core router is made once here (router_split);
    call resplit_router() after changing w_router in place."""

    def __init__(self, cfg: MoeConfig, w_router, w_gate, w_up, w_down, logit_bias=None,
                 device="cuda", gather: bool = False):
        self.cfg = cfg
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.logit_bias = logit_bias
        self.ws = alloc_workspace(cfg, device)
        self.bufs = LayerBuffers.allocate(cfg, device, gather=gather)
        self._structs = self.bufs.as_struct(True)
        self.resplit_router()

    def resplit_router(self, stream=None) -> None:
        self.w_router_split = router_split(self.cfg, self.w_router, stream)

    def inputs(self, x) -> MoeLayerInputs:
        b = self.logit_bias
        return MoeLayerInputs(
            x=_ptr(x), w_router=_ptr(self.w_router), logit_bias=_ptr(b),
            bias_row_stride=0 if (b is None or b.dim() == 1) else b.shape[1],
            w_gate=_ptr(self.w_gate), w_up=_ptr(self.w_up), w_down=_ptr(self.w_down),
            w_router_split=_ptr(self.w_router_split))

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        moe_layer_forward(self.cfg, self.inputs(x), self._structs, self.ws, stream)
        return self.bufs.out

    __call__ = forward

    def pick_rank_counts(self, group_of_expert=None, stream=None):
        """The second-choice counters of the last forward: (routed [k, E], kept [k, E],
        differs [k]) int32 device tensors; group_of_expert: None or an [E] int32 map."""
        return moe_pick_rank_counts(self.cfg, self.bufs.topk_idx, self.bufs.assign_row,
                                    self.ws, group_of_expert, stream)

    def capture(self, x: torch.Tensor) -> "torch.cuda.CUDAGraph":
        """Record one forward on the fixed input buffer x into a CUDA graph: replay() then
        runs the whole layer (every kernel, no host work) on whatever x holds, into
        self.bufs.out.  The layer enqueues no host synchronisation and allocates nothing, so
        it captures as is; one eager forward first sets up the per-device state."""
        self.forward(x)
        torch.cuda.synchronize(x.device)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(x.device)
        side.wait_stream(torch.cuda.current_stream(x.device))
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                self.forward(x, side)
        torch.cuda.current_stream(x.device).wait_stream(side)
        return graph


class HostPipeline:
    """Runs one MoE layer over a sequence of token batches held in pinned host memory,
    overlapping every batch's host-to-device copy and the previous result's device-to-host
    copy with the layer's kernels: two copy streams (in and out) around the compute stream,
    and `depth` sets of device buffers used in turn.  The results are those of
    MoELayer.forward on each batch."""

    def __init__(self, cfg: MoeConfig, w_router, w_gate, w_up, w_down, logit_bias=None,
                 device="cuda", depth: int = 2):
        if depth < 2:
            raise ValueError("depth must be >= 2 to overlap copies with compute")
        self.device = torch.device(device)
        self.layers = [MoELayer(cfg, w_router, w_gate, w_up, w_down, logit_bias, device)
                       for _ in range(depth)]
        dt = torch.float32 if cfg.dtype == F32 else torch.bfloat16
        self.x_dev = [torch.empty((cfg.T, cfg.d_model), dtype=dt, device=self.device)
                      for _ in range(depth)]
        self.s_in = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)

    def run(self, xs_host, outs_host, stream=None) -> None:
        """Enqueue every batch: xs_host[i] -> layer -> outs_host[i] (pinned host tensors of
        shape [T, d_model]).  Returns once everything is enqueued; synchronise on `stream`
        (default: the current stream) to wait for the last result."""
        comp = stream or torch.cuda.current_stream(self.device)
        depth = len(self.layers)
        n = len(xs_host)
        copied, computed, fetched = [], [], []
        start = torch.cuda.Event()
        start.record(comp)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        for i in range(n):
            slot = i % depth
            with torch.cuda.stream(self.s_in):
                if i >= depth:  # the slot's input buffer is free once its last layer ran
                    self.s_in.wait_event(computed[i - depth])
                self.x_dev[slot].copy_(xs_host[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_in)
                copied.append(ev)
            comp.wait_event(copied[i])
            if i >= depth:      # the slot's output buffer is free once it was fetched
                comp.wait_event(fetched[i - depth])
            self.layers[slot].forward(self.x_dev[slot], comp)
            ev = torch.cuda.Event()
            ev.record(comp)
            computed.append(ev)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(computed[i])
                outs_host[i].copy_(self.layers[slot].bufs.out, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_out)
                fetched.append(ev)
        if n:
            comp.wait_event(fetched[-1])

