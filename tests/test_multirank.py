"""The multi-GPU bench path's host logic with two gloo ranks on the CPU: each
rank gets its own problem of the same shape, and the reported time is the max
over ranks; the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wp, wd = bench.rank_workloads("full", rank)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        ref = bench.run_reference(None, rank, world) if rank != 0 else "rank0"
        out.put((rank, wp.seed, wd.seed, wp.n_q, wd.batch, t, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, sp0, sd0, n0, b0, t0, ref0), (r1, sp1, sd1, n1, b1, t1, ref1) = res
    assert (n0, b0) == (n1, b1) == (131072, 64)       # same shapes on every rank
    assert sp0 != sp1 and sd0 != sd1                  # independent problems
    assert t0 == t1 == 15.0                           # max over ranks on every rank
    assert ref1 is None                               # the reference arm is rank 0's alone
