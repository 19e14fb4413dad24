"""Host logic of the multi-rank bench path, on CPU with world size 2 over
gloo: every rank reduces its times to the slowest rank's, the whole-job
rate counts every rank's units over that time, and the reference arm runs
on rank 0 only."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r timed (r + 1) * 10 ms in total and r + 0.5 ms per GEMM
        got = bench.max_over_ranks([(rank + 1) * 10.0, rank + 0.5], dist, "cpu")
        rate = bench.replica_throughput(world, 100.0, 5, got[0])
        q.put((rank, got, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, got, rate in out:
        assert got == [20.0, 1.5]                      # the slower rank's numbers, on every rank
        assert rate == world * 100.0 * 5 / 0.020       # both ranks' units over the max time


def test_single_rank_is_identity_and_env_parsing(monkeypatch):
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.env_rank() == (1, 1, 2)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""
