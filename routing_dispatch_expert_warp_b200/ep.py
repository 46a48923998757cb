"""Expert parallelism across ranks: buffers, peer-pointer tables and the step order.

"Expert Parallelism for MoE Serving" (aiunderstanding.org), "Deep dive" / "Technical
insight": each rank owns a subset of the experts; every MoE layer sends each token's row to
its experts' owners (dispatch) and brings the results back (combine).  "MoE expert
parallelism needs measurements before launch" (airouter.kz): tokens past the capacity are
dropped before the exchange; "Expert and GPU can be balanced differently": the rank / node /
pair-traffic record (moe_ep_stats).

Everything that touches data runs in the library's kernels (moe_ep_* in include/moe.h);
this module only allocates, builds the device tables of peer pointers and orders the steps.
Two drivers share one per-rank state (EpRank):
  * EpEmulator -- `world` ranks on one GPU and one stream; the peer tables point at the
    ranks' own buffers and stream order is the barrier;
  * EpGroup    -- one process per GPU; peers' buffers are mapped through CUDA IPC and the
    barrier is a one-element all-reduce on the current stream (stream-ordered, so no host
    synchronisation).
"""
from __future__ import annotations

import ctypes
from typing import Callable, Dict, List, Optional, Sequence

import torch

from . import _abi
from ._abi import MoeEpConfig, MoeEpStats, check
from . import (LayerBuffers, alloc_workspace, moe_dispatch_scored, moe_route, F32)

# The per-layer step order (see include/moe.h, "expert parallelism"): a "barrier" entry
# means every rank's previous steps must be complete before any rank's next one.
SCHEDULE = ("route", "rank", "put_counts", "barrier", "plan", "dispatch", "barrier",
            "expert_ffn", "barrier", "combine", "stats", "barrier")


def _lib():
    return _abi.lib()


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def contiguous_placement(E: int, world: int, device="cuda") -> torch.Tensor:
    """expert_rank[e] = e // (E / world) as a device int32 tensor."""
    if world < 1 or E % world:
        raise ValueError("E must be a multiple of world")
    return (torch.arange(E, dtype=torch.int32) // (E // world)).to(device)


def local_experts(expert_rank: torch.Tensor, rank: int) -> torch.Tensor:
    """The experts `rank` owns, ascending: local expert i is global expert [i]."""
    return torch.nonzero(expert_rank.cpu() == rank).flatten()


def common_recv_rows(cfg, expert_rank: torch.Tensor, world: int) -> int:
    """Receive-buffer rows every rank allocates: the library's bound for the rank that owns
    the most experts.  The kernels check a destination row against the sender's recv_rows,
    so the value must be the same on every rank."""
    owners = expert_rank.cpu().to(torch.int64)
    most = int(torch.bincount(owners, minlength=world).max())
    probe = MoeEpConfig(world=world, rank=0, ranks_per_node=1, n_local=most, expert_rank=None,
                        recv_rows=0)
    rows = int(_lib().moe_ep_recv_rows_bound(ctypes.byref(cfg), ctypes.byref(probe)))
    if rows < 0:
        check(1)
    return rows


class EpRank:
    """One rank's state for the EP layer: its config, workspace, routing buffers, count
    matrix, receive / hidden / result buffers and its local experts' weights."""

    def __init__(self, cfg, world: int, rank: int, expert_rank: torch.Tensor, w_router,
                 w_gate_local, w_up_local, w_down_local, logit_bias=None,
                 ranks_per_node: int = 1, recv_rows: Optional[int] = None, device="cuda"):
        self.cfg = cfg
        self.world, self.rank = world, rank
        self.expert_rank = expert_rank.to(device=device, dtype=torch.int32).contiguous()
        n_local = int(local_experts(self.expert_rank, rank).numel())
        if n_local != w_gate_local.shape[0]:
            raise ValueError("local weights do not match the placement")
        self.ep = MoeEpConfig(world=world, rank=rank, ranks_per_node=ranks_per_node,
                              n_local=n_local, expert_rank=_p(self.expert_rank), recv_rows=0)
        if recv_rows is None:
            recv_rows = common_recv_rows(cfg, self.expert_rank, world)
        self.ep.recv_rows = recv_rows
        self.w_router, self.logit_bias = w_router, logit_bias
        self.w_gate, self.w_up, self.w_down = w_gate_local, w_up_local, w_down_local
        T, d, f, E, k = cfg.T, cfg.d_model, cfg.d_ff, cfg.E, cfg.k
        dt = torch.float32 if cfg.dtype == F32 else torch.bfloat16
        i32 = dict(dtype=torch.int32, device=device)
        self.ws = alloc_workspace(cfg, device)
        self.bufs = LayerBuffers.allocate(cfg, device, gather=True)   # no x_perm
        self.count_mat = torch.zeros((world, E), **i32)
        R = max(recv_rows, 1)
        self.recv_x = torch.empty((R, d), dtype=dt, device=device)
        self.h = torch.empty((R, f), dtype=dt, device=device)
        self.y_recv = torch.empty((R, d), dtype=dt, device=device)
        self.send_row = torch.empty((T, k), **i32)
        self.recv_offsets = torch.empty(n_local + 1, **i32)
        self.recv_counts = torch.empty(n_local, **i32)
        self.stats_buf = torch.zeros(ctypes.sizeof(MoeEpStats), dtype=torch.uint8,
                                     device=device)

    @property
    def out(self) -> torch.Tensor:
        return self.bufs.out

    # ---- one library call per step
    def route(self, x, stream=None):
        b = self.bufs
        moe_route(self.cfg, x, self.w_router, self.logit_bias, b.logits, b.topk_idx, b.topk_w,
                  self.ws, stream)

    def rank_assignments(self, stream=None):
        b = self.bufs
        moe_dispatch_scored(self.cfg, None, b.topk_idx, b.logits, self.logit_bias,
                            b.routed_counts, b.kept_counts, b.expert_offsets, b.assign_row,
                            b.token_of_row, None, self.ws, stream)

    def put_counts(self, mats_table: torch.Tensor, stream=None):
        check(_lib().moe_ep_put_counts(ctypes.byref(self.cfg), ctypes.byref(self.ep),
                                       _p(self.bufs.kept_counts), _p(mats_table),
                                       _stream(stream)))

    def plan(self, stream=None):
        b = self.bufs
        check(_lib().moe_ep_plan(ctypes.byref(self.cfg), ctypes.byref(self.ep),
                                 _p(self.count_mat), _p(b.topk_idx), _p(b.assign_row),
                                 _p(b.expert_offsets), _p(self.send_row),
                                 _p(self.recv_offsets), _p(self.recv_counts), _p(self.ws),
                                 self.ws.numel(), _stream(stream)))

    def dispatch(self, x, recv_table: torch.Tensor, stream=None):
        check(_lib().moe_ep_dispatch(ctypes.byref(self.cfg), ctypes.byref(self.ep), _p(x),
                                     _p(self.bufs.topk_idx), _p(self.send_row),
                                     _p(recv_table), _p(self.ws), self.ws.numel(),
                                     _stream(stream)))

    def expert_ffn(self, stream=None):
        check(_lib().moe_ep_expert_ffn(ctypes.byref(self.cfg), ctypes.byref(self.ep),
                                       _p(self.recv_x), _p(self.recv_offsets),
                                       _p(self.recv_counts), _p(self.w_gate), _p(self.w_up),
                                       _p(self.w_down), _p(self.h), _p(self.y_recv),
                                       _p(self.ws), self.ws.numel(), _stream(stream)))

    def combine(self, y_table: torch.Tensor, stream=None):
        b = self.bufs
        check(_lib().moe_ep_combine(ctypes.byref(self.cfg), ctypes.byref(self.ep), _p(y_table),
                                    _p(b.topk_idx), _p(self.send_row), _p(b.topk_w), _p(b.out),
                                    _p(self.ws), self.ws.numel(), _stream(stream)))

    def stats(self, host: bool = False, stream=None) -> Optional[dict]:
        hs = MoeEpStats()
        check(_lib().moe_ep_stats(ctypes.byref(self.cfg), ctypes.byref(self.ep),
                                  _p(self.count_mat), _p(self.stats_buf),
                                  ctypes.byref(hs) if host else None, _stream(stream)))
        return hs.as_dict() if host else None

    def stats_dict(self) -> dict:
        raw = bytes(self.stats_buf.cpu().numpy().tobytes())
        return MoeEpStats.from_buffer_copy(raw).as_dict()


def _table(ptrs: Sequence[int], device) -> torch.Tensor:
    return torch.tensor(list(ptrs), dtype=torch.int64, device=device)


def run_schedule(ranks: Sequence[EpRank], xs: Sequence[torch.Tensor], tables: dict,
                 barrier: Callable[[], None], stream=None,
                 on_step: Optional[Callable[[str], None]] = None) -> None:
    """The steps of SCHEDULE for the ranks held by this process (all ranks when emulated on
    one GPU, one rank per process otherwise).  on_step(name) is called before each step (and
    with "end" after the last), e.g. to record timing events."""
    for step in SCHEDULE:
        if step == "barrier":
            barrier()
            continue
        if on_step is not None:
            on_step(step)
        for r, x in zip(ranks, xs):
            if step == "route":
                r.route(x, stream)
            elif step == "rank":
                r.rank_assignments(stream)
            elif step == "put_counts":
                r.put_counts(tables["mats"], stream)
            elif step == "plan":
                r.plan(stream)
            elif step == "dispatch":
                r.dispatch(x, tables["recv"], stream)
            elif step == "expert_ffn":
                r.expert_ffn(stream)
            elif step == "combine":
                r.combine(tables["ybuf"], stream)
            elif step == "stats":
                r.stats(False, stream)
    if on_step is not None:
        on_step("end")


class EpEmulator:
    """`world` EP ranks sharing one GPU (and one stream).  Each rank has its own tokens,
    buffers and local weights; the peer tables point at the ranks' own buffers, so the
    kernels are exactly those a multi-GPU run uses, and stream order is the barrier."""

    def __init__(self, cfg, world: int, w_router, w_gate, w_up, w_down,
                 logit_biases: Optional[Sequence] = None, expert_rank=None,
                 ranks_per_node: int = 1, recv_rows: Optional[int] = None, device="cuda",
                 local_weights: Optional[Sequence] = None):
        """local_weights: None, or per rank the (w_gate, w_up, w_down) of its local experts,
        already sliced (another emulator's, to share them) -- then w_gate/w_up/w_down are
        not read."""
        E = cfg.E
        self.world = world
        self.expert_rank = (contiguous_placement(E, world, device) if expert_rank is None
                            else expert_rank.to(device=device, dtype=torch.int32))
        self.ranks: List[EpRank] = []
        for r in range(world):
            if local_weights is not None:
                wg, wu, wd = local_weights[r]
            else:
                mine = local_experts(self.expert_rank, r).to(w_gate.device)
                wg, wu, wd = (w_gate[mine].contiguous(), w_up[mine].contiguous(),
                              w_down[mine].contiguous())
            bias = None if logit_biases is None else logit_biases[r]
            self.ranks.append(EpRank(cfg, world, r, self.expert_rank, w_router, wg, wu, wd,
                                     bias, ranks_per_node, recv_rows, device))
        self.tables = {
            "mats": _table([r.count_mat.data_ptr() for r in self.ranks], device),
            "recv": _table([r.recv_x.data_ptr() for r in self.ranks], device),
            "ybuf": _table([r.y_recv.data_ptr() for r in self.ranks], device),
        }

    def forward(self, xs: Sequence[torch.Tensor], stream=None,
                on_step: Optional[Callable[[str], None]] = None) -> List[torch.Tensor]:
        run_schedule(self.ranks, xs, self.tables, lambda: None, stream, on_step)
        return [r.out for r in self.ranks]


# ------------------------------------------------------------------ one process per GPU
class CudaIpcTransport:
    """Peer mappings through CUDA IPC (moe_ipc_*) and a stream-ordered barrier."""

    def export(self, ptr: int):
        h = ctypes.create_string_buffer(64)
        off = ctypes.c_int64(0)
        check(_lib().moe_ipc_handle(ptr, h, ctypes.byref(off)))
        return bytes(h.raw), int(off.value)

    def open(self, handle: bytes) -> int:
        out = ctypes.c_void_p(0)
        check(_lib().moe_ipc_open(handle, ctypes.byref(out)))
        return int(out.value)

    def close(self, base: int) -> None:
        check(_lib().moe_ipc_close(base))

    def barrier(self, group, device) -> None:
        import torch.distributed as dist
        flag = torch.ones(1, dtype=torch.int32, device=device)
        dist.all_reduce(flag, group=group)   # an NCCL kernel on the current stream


def exchange_peer_pointers(local: Dict[str, int], transport, group=None) -> dict:
    """Every rank exports its buffers, gathers everyone's exports and maps the peers'.
    Returns {name: [pointer usable here for rank g's buffer, g = 0..world-1]} and the list
    of mapped bases to close."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    me = dist.get_rank(group)
    mine = {name: transport.export(ptr) for name, ptr in local.items()}
    everyone: list = [None] * world
    dist.all_gather_object(everyone, mine, group=group)
    tables: Dict[str, List[int]] = {name: [] for name in local}
    opened = []
    mapped: Dict[bytes, int] = {}
    for g in range(world):
        for name in local:
            if g == me:
                tables[name].append(local[name])
                continue
            handle, off = everyone[g][name]
            if handle not in mapped:          # buffers of one allocation share a mapping
                mapped[handle] = transport.open(handle)
                opened.append(mapped[handle])
            tables[name].append(mapped[handle] + off)
    return {"tables": tables, "opened": opened}


class EpGroup:
    """This process's rank of a multi-GPU EP layer (one process per GPU, torch.distributed
    initialised, NCCL for the barrier)."""

    def __init__(self, cfg, w_router, w_gate_local, w_up_local, w_down_local, expert_rank,
                 logit_bias=None, ranks_per_node: int = 1, recv_rows: Optional[int] = None,
                 group=None, transport=None, device=None):
        import torch.distributed as dist
        self.group = group
        world, rank = dist.get_world_size(group), dist.get_rank(group)
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.transport = transport or CudaIpcTransport()
        self.me = EpRank(cfg, world, rank, expert_rank, w_router, w_gate_local, w_up_local,
                         w_down_local, logit_bias, ranks_per_node, recv_rows, self.device)
        torch.cuda.synchronize(self.device)   # buffers exist before peers map them
        sizes: list = [None] * world
        dist.all_gather_object(sizes, int(self.me.ep.recv_rows), group=group)
        if len(set(sizes)) != 1:   # rows are checked against the sender's value: one size
            raise ValueError(f"recv_rows differs across ranks: {sizes}")
        ex = exchange_peer_pointers({"mats": self.me.count_mat.data_ptr(),
                                     "recv": self.me.recv_x.data_ptr(),
                                     "ybuf": self.me.y_recv.data_ptr()},
                                    self.transport, group)
        self._opened = ex["opened"]
        self.tables = {name: _table(ptrs, self.device) for name, ptrs in ex["tables"].items()}

    def forward(self, x: torch.Tensor, stream=None,
                on_step: Optional[Callable[[str], None]] = None) -> torch.Tensor:
        run_schedule([self.me], [x], self.tables,
                     lambda: self.transport.barrier(self.group, self.device), stream, on_step)
        return self.me.out

    def close(self) -> None:
        torch.cuda.synchronize(self.device)
        for base in self._opened:
            self.transport.close(base)
        self._opened = []
