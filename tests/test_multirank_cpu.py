"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).  The path runs as
independent replicas (one per GPU, no data-path collective), so what ranks share is
the timing: the job's time is its slowest rank's, the throughput adds the replicas,
and only rank 0 runs and reports the reference arm."""
from __future__ import annotations

import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out) -> None:
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu", world)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_job_time_is_the_slowest_rank():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_time_is_its_own():
    assert bench.max_over_ranks(12.5, "cpu", 1) == 12.5


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_throughput_adds_the_replicas(world):
    # 4 sequences per rank per step, 128 steps, 1.75 s for the slowest rank
    assert bench.job_tokens_per_s(4, 128, world, 1750.0) == pytest.approx(world * 4 * 128 / 1.75)


def test_reference_arm_runs_on_rank_0_only(capsys):
    bench.run_reference(None, None, 1)   # any other rank returns without work or output
    assert capsys.readouterr().out == ""
