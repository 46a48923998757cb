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
