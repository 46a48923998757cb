"""Host logic of multi-process expert parallelism on CPU gloo ranks (no GPU, no kernels):
the exchange of buffer exports into per-rank peer tables, and the step order with its
barriers -- every rank's steps before a barrier finish before any rank's step after it."""
import os
import socket
import time

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from routing_dispatch_expert_warp_b200 import ep as EP


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class FakeTransport:
    """Exports name a (rank, buffer) pair and a 64-byte offset; opening a peer's export maps
    it at a base address derived from the peer's rank and the buffer."""

    NAMES = ("mats", "recv", "ybuf")

    def __init__(self, rank):
        self.rank = rank
        self.opened, self.closed = [], []

    def export(self, ptr):
        return f"{self.rank}:{ptr}".encode(), 64

    def open(self, handle):
        rank, ptr = handle.decode().split(":")
        base = 10_000_000 * (int(rank) + 1) + int(ptr) * 1000
        self.opened.append(base)
        return base

    def close(self, base):
        self.closed.append(base)


class FakeRank:
    """Duck-typed EpRank: records each step with a wall-clock stamp."""

    def __init__(self, rank, log):
        self.rank, self.log = rank, log

    def _rec(self, step):
        time.sleep(0.02 * (1 + self.rank))     # ranks drift apart between barriers
        self.log.append((step, time.time()))

    def route(self, x, stream=None): self._rec("route")
    def rank_assignments(self, stream=None): self._rec("rank")
    def put_counts(self, t, stream=None): self._rec("put_counts")
    def plan(self, stream=None): self._rec("plan")
    def dispatch(self, x, t, stream=None): self._rec("dispatch")
    def expert_ffn(self, stream=None): self._rec("expert_ffn")
    def combine(self, t, stream=None): self._rec("combine")
    def stats(self, host=False, stream=None): self._rec("stats")


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tr = FakeTransport(rank)
        local = {name: 100 * rank + i for i, name in enumerate(FakeTransport.NAMES)}
        ex = EP.exchange_peer_pointers(local, tr)
        log = []
        EP.run_schedule([FakeRank(rank, log)], [None], {"mats": None, "recv": None, "ybuf": None},
                        lambda: dist.barrier())
        q.put((rank, ex["tables"], ex["opened"], log))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_peer_tables_and_barrier_order(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=120) for _ in procs], key=lambda o: o[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    names = FakeTransport.NAMES
    for me, tables, opened, _ in out:
        for i, name in enumerate(names):
            want = []
            for g in range(world):
                ptr = 100 * g + i
                want.append(ptr if g == me else 10_000_000 * (g + 1) + ptr * 1000 + 64)
            assert tables[name] == want, (me, name)
        assert len(opened) == (world - 1) * len(names)    # one mapping per peer buffer

    # phases between barriers: every rank's phase-i steps end before any phase-(i+1) step
    phases, cur = [], []
    for step in EP.SCHEDULE:
        if step == "barrier":
            phases.append(cur)
            cur = []
        else:
            cur.append(step)
    assert cur == []
    assert phases == [["route", "rank", "put_counts"], ["plan", "dispatch"], ["expert_ffn"],
                      ["combine", "stats"]]
    stamps = {}
    for rank, _, _, log in out:
        assert [s for s, _ in log] == [s for ph in phases for s in ph]
        for s, t in log:
            stamps.setdefault(s, []).append(t)
    for a, b in zip(phases, phases[1:]):
        last_a = max(t for s in a for t in stamps[s])
        first_b = min(t for s in b for t in stamps[s])
        assert last_a <= first_b, (a, b)


def _inputs_worker(rank, world, port, q):
    import torch
    import bench
    from routing_dispatch_expert_warp_b200 import workload as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = {}
        for name, shape in (("zipf", W.reduced(W.DSV3_PREFILL_ZIPF, 48, 64, 32, E=16)),
                            ("chunks", W.reduced(W.MIXTRAL_8X22B_MIXED, 300, 64, 32,
                                                 n_decode_tokens=4))):
            inp = bench.ep_rank_inputs(shape, rank, world, "cpu")
            same = all(torch.equal(inp[k][i], w)
                       for i, e in enumerate(inp["experts"])
                       for k, w in zip(("w_gate", "w_up", "w_down"), W.expert_weights(shape, e)))
            out[name] = (inp["experts"], float(inp["x"].float().sum()),
                         inp["w_router"].clone(), inp["logit_bias"].clone(), same)
        dist.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_bench_ep_rank_inputs_on_two_gloo_ranks():
    """bench.py --ep's per-rank inputs: the experts split in disjoint contiguous blocks that
    cover all E, each rank's local weights those of the single-GPU layer, one router weight
    and one per-expert bias for the layer, and each rank its own batch (and the per-token
    bias drawn with it)."""
    import torch
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_inputs_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for name, E in (("zipf", 16), ("chunks", 8)):
        a, b = out[0][name], out[1][name]
        assert a[0] == list(range(E // 2)) and b[0] == list(range(E // 2, E))
        assert a[1] != b[1]                                   # distinct batches
        assert torch.equal(a[2], b[2])                        # one router weight
        assert a[4] and b[4]                                  # the single-GPU layer's weights
        if name == "zipf":
            assert torch.equal(a[3], b[3]) and a[3].dim() == 1   # one per-expert bias
        else:
            assert a[3].dim() == 2 and not torch.equal(a[3], b[3])  # per-token, per batch
