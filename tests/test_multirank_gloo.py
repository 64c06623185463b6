"""The multi-rank host logic of bench.py (one process per GPU, weak scaling,
no collective in the data path) on two CPU processes with the gloo backend:
per-rank timings reduce to the slowest rank, the job throughput counts every
rank's tokens against that time, and every rank draws a different input."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from linear_attention_video_block_b200.synth import Layout, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports times (r + 1, 10 - r, 3): the job takes the slowest rank's
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 3.0], world)
        lay = Layout(B=1, F=3, N=4, T=2, c=2, H=1, d=16)
        inp = make_inputs(lay, "f32", bench.rank_seed(7, rank))
        # every rank's own input, gathered to compare
        qs = [torch.empty_like(inp["q"]) for _ in range(world)]
        dist.all_gather(qs, inp["q"])
        distinct = not torch.equal(qs[0], qs[1])
        q.put((rank, got, distinct))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_independent_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    for rank, got, distinct in res:
        assert got == [2.0, 10.0, 3.0]
        assert distinct


def test_single_rank_is_identity_and_throughput():
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    # 4 ranks x 145152 tokens in 200 ms
    assert bench.job_throughput(145152, 4, 200.0) == pytest.approx(4 * 145152 / 0.2)
    assert bench.rank_seed(3, 0) != bench.rank_seed(3, 1)
