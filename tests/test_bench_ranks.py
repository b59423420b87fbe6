"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): every rank
meets at the barriers, takes the max of the ranks' times, and the job value
counts every rank's tokens.  No GPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_env()
        assert (w, r) == (world, rank)
        bench.sync_ranks(torch, dist, world)
        local_ms = [3.0, 5.0][rank]                # rank 1 is the slow one
        t = bench.max_over_ranks(local_ms, torch, dist, world, torch.device("cpu"))
        e = bench.max_over_ranks(10.0 + rank, torch, dist, world, torch.device("cpu"))
        bench.sync_ranks(torch, dist, world)
        out[rank] = (t, e)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (5.0, 11.0)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, torch, None, 1, torch.device("cpu")) == 7.5


def test_job_value_counts_every_rank():
    # B=4, T=4096 per rank; 2 ranks in 0.5 ms -> 2 * 16384 tokens / 0.5 ms
    assert bench.job_tokens_per_s(4, 4096, 2, 0.5) == pytest.approx(2 * 4 * 4096 / 0.5e-3)
    assert bench.job_tokens_per_s(4, 4096, 1, 0.5) == pytest.approx(4 * 4096 / 0.5e-3)
