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


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with
    the benchmark's metric, a positive throughput, and its own cpu_baseline and e2e."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_l1_b1_h8x2_d64_n2048", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_l1_b1_h8x2_d64_n2048"
