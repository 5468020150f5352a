"""The multi-process plumbing of bench.py on CPU: two gloo ranks. On GPUs every rank runs
an independent problem (replicas, weak scaling); the only cross-rank step is the maximum
of the timings, and the reference arm runs on rank 0 alone."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([float(rank), 10.0 - rank, 3.5])
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0] == results[1] == [1.0, 10.0, 3.5]


def test_max_over_ranks_single_process():
    import bench
    assert bench.max_over_ranks([2.0, 5.0]) == [2.0, 5.0]


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload=bench.HEADLINE.name, steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
