"""Replica scaling (the path has no exchange step): the job figure is the slowest rank's time and
the sum of every rank's bytes. Checked with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = bench.aggregate_ranks(torch, dist, "cpu", ms=1.0 + rank, decode_ms=0.5 * (rank + 1),
                                    e2e_ms=3.0 - rank, step_bytes=100.0 * (rank + 1), errors=float(rank == 1) * 4)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_sum_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    for r in (0, 1):
        assert res[r] == {"ms": 2.0, "decode_ms": 1.0, "e2e_ms": 3.0, "step_bytes": 300.0, "errors": 4.0}


def test_single_process_is_identity():
    v = dict(ms=1.5, decode_ms=1.0, e2e_ms=2.0, step_bytes=7.0, errors=0.0)
    assert bench.aggregate_ranks(torch, None, "cpu", **v) == v
