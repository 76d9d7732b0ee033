"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank reports its own timings; the line must carry the slowest rank's time
and the work of both ranks (weak scaling), as under torchrun with NCCL."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 is slower in total and in the GEMM, rank 0 in the activation kernel
        mine = [1.0 + rank, 0.3 - 0.1 * rank, 0.5 + 0.2 * rank]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        assert out[rank] == pytest.approx([2.0, 0.3, 0.7])
    # 2 ranks x 10 steps x 1e12 FLOP each over the slowest rank's 2 s
    assert bench.job_throughput(2, 1e12, 10, 2.0) == pytest.approx(10.0)
    assert bench.job_throughput(1, 1e12, 10, 2.0) == pytest.approx(5.0)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([3.0, 1.5], 1, torch.device("cpu")) == [3.0, 1.5]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun only rank 0 times the oracle; the other ranks exit at once."""
    import argparse
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(config="c2_qkv", layer=None, M=None, cpu_rows=64, steps=1, warmup=3)
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""
