"""The multi-rank host logic of bench.py on CPU: two gloo ranks (replicas with no
data-path collective) agree on the slowest rank's time, the job throughput counts
every rank's requests, and the reference arm runs on rank 0 only."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, ms_by_rank, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slow = bench.max_over_ranks(ms_by_rank[rank], world, "cpu")
        dist.barrier()
        out[rank] = slow
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    ms_by_rank = [300.5, 312.25]
    mp.start_processes(_rank, args=(2, _free_port(), ms_by_rank, out), nprocs=2, join=True,
                       start_method="spawn")
    assert dict(out) == {0: 312.25, 1: 312.25}


def test_job_throughput_counts_every_rank():
    one = bench.job_throughput(256, 1, 3.0)
    assert abs(one - 256 / 3e-3) < 1e-6
    assert abs(bench.job_throughput(256, 4, 3.0) - 4 * one) < 1e-6
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5


def test_reference_arm_is_rank_zero_only(capsys, monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "1",
                                     "--warmup", "3", "--gpus", "2"])
    bench.main()  # rank 1 does no work and prints nothing
    assert capsys.readouterr().out == ""
