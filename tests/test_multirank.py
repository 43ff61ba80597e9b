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


def test_bench_spawns_its_own_ranks():
    """`bench.py --gpus 2` started without a launcher runs itself again as two
    torchrun ranks; here the ranks only exercise the host logic on gloo (no
    GPU): the job time is the slower rank's and rank 0 prints one line."""
    import json
    import subprocess
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--selftest-ranks", "--steps", "10"], env=env, capture_output=True,
                         text=True, timeout=240)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["job_ms"] == 3.0  # ranks took 2 ms and 3 ms
    assert line["value"] == pytest.approx(2 * 10 / 3e-3)


def test_relaunch_command():
    cmd = bench.relaunch_command(["--gpus", "8", "--steps", "5"], 8, 29555)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "8"
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "8", "--steps", "5"]
