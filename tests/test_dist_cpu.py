"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): each rank owns its own batch,
the timing reduction is a max over ranks, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    bench.barrier(world)
    m = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    out[rank] = m
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of a multi-threaded process
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == 15.0 and out[1] == 15.0


def test_reference_arm_non_zero_rank_exits_quietly(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = bench.main.__wrapped__ if hasattr(bench.main, "__wrapped__") else None
    assert bench.bench_reference(type("A", (), dict(steps=1, warmup=3, gpus=2))()) == 0
    assert capsys.readouterr().out == ""
