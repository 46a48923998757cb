"""The N > 1 path of bench.py on CPU: two gloo ranks, no GPU.  Each GPU runs an independent
replica of the layer (no exchange at EP=1); ranks draw different batches and the job's time is
the slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from routing_dispatch_expert_warp_b200 import workload as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 3.0 - rank]
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        shape = bench.rank_shape(W.TINY_FP32, rank)
        x = W.make_inputs(shape, weights=False).x
        dist.barrier()
        q.put((rank, got, shape.seed, float(x.sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert out[0][1] == out[1][1] == [11.0, 3.0]      # element-wise max over ranks
    assert out[0][2] != out[1][2]                     # different seeds per rank
    assert out[0][3] != out[1][3]                     # hence different token batches


def test_single_process_passthrough():
    assert bench.max_over_ranks([1.5, 2.5], None, torch.device("cpu")) == [1.5, 2.5]
    assert bench.rank_shape(W.TINY_FP32, 0) is W.TINY_FP32
