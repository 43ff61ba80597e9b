"""The bench's multi-rank host logic on CPU: two gloo ranks.

Each rank runs its own sequences (different seeded inputs per rank), the
job's time is the slowest rank's (a MAX all-reduce), and the job's throughput
counts the rounds of every rank within that time.  No GPU, no NCCL.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_draft_tree_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 7.5][rank]
        job_ms = bench.max_over_ranks(local_ms, world, "cpu")
        w = synth.WORKLOADS["tiny"]
        x, seed = bench.make_inputs(w, rank, 0)
        digest = float(np.asarray(x["draft"], dtype=np.float64).sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (seed, digest))
        out.put((rank, job_ms, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, job_ms, gathered in res:
        assert job_ms == 7.5  # the slowest rank's time, on every rank
        (s0, d0), (s1, d1) = gathered
        assert s0 != s1 and d0 != d1  # each rank drafts its own sequences


def test_job_throughput_counts_every_rank():
    # 2 ranks x batch 4 x 10 rounds in 5 ms = 16000 rounds/s
    assert bench.job_throughput(2, 4, 10, 5.0) == pytest.approx(16000.0)
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
