"""The benchmark's multi-rank host logic on CPU: two ranks on the gloo backend
(127.0.0.1), spawned processes, no GPU.  Every rank must see the slowest rank's
time, and the job's throughput must count every rank's replica (weak scaling);
the reference arm runs on rank 0 only."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        total_ms = 100.0 + 20.0 * rank          # rank 1 is the slow one
        out.put((rank, bench.replica_throughput(1000, total_ms, 10, world)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_count_every_replica():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    world, port = 2, free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        ms, value = res[r]
        assert ms == pytest.approx(12.0)                # max(100, 120) ms over 10 steps
        assert value == pytest.approx(2 * 1000 / 12e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload, warmup, steps, gpus, ref_seconds = "causal_fp32_small", 3, 1, 2, 0.1

    assert bench.run_reference(Args, 2, 1) == 0       # rank 1: no work, no line
    assert capsys.readouterr().out == ""
