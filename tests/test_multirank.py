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


def _bench_env():
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["PYTHONPATH"] = bench.ROOT
    return env


def test_bench_gpus_flag_launches_that_many_ranks():
    # `bench.py --gpus 2` run directly relaunches itself under torchrun with
    # two processes; the reference arm (CPU only) prints from rank 0 and
    # reports the world size it ran with.
    import json
    import subprocess
    import sys
    cmd = [sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
           "--case", "tiny", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=_bench_env())
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1          # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_bench_gpus_flag_must_match_world_size():
    import subprocess
    import sys
    env = _bench_env()
    env.update(WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    cmd = [sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
           "--case", "tiny", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
    c = bench.relaunch_command(["--gpus", "4"], 4, 29500)
    assert c[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"] and "--nproc-per-node" in c
    assert c[c.index("--nproc-per-node") + 1] == "4" and c[c.index("--master-addr") + 1] == "127.0.0.1"
