"""Collective plumbing of the replicas' job record on two and three CPU gloo ranks (no GPU):
the counts are summed over the ranks and every rank's record is gathered in rank order."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from routing_dispatch_expert_warp_b200 import replicas as R


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        routed = torch.arange(6, dtype=torch.int32) * (rank + 1)
        kept = torch.full((6,), rank, dtype=torch.int32)
        record = torch.full((16,), 10 + rank, dtype=torch.uint8)
        r, k, recs = R.gather_counts(routed, kept, record)
        q.put((rank, r.tolist(), k.tolist(), recs.tolist(), routed.tolist(), kept.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_counts_summed_and_records_gathered(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=120) for _ in procs])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tri = sum(range(1, world + 1))
    for rank, r, k, recs, own_r, own_k in out:
        assert r == [i * tri for i in range(6)]
        assert k == [sum(range(world))] * 6
        assert recs == [[10 + g] * 16 for g in range(world)]
        assert own_r == [i * (rank + 1) for i in range(6)] and own_k == [rank] * 6
