"""The multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path runs as independent replicas (one per GPU, no exchange); the only
cross-rank steps are the barrier and the max over ranks of the measured time,
from which the whole-job throughput is computed.  Those helpers are exercised
here with a real two-process group, without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r measured 10 * (r + 1) ms: every rank must see the slowest one
        slowest = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        dist.barrier()
        # the same call twice in a row keeps every rank in step
        again = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
        results[rank] = (slowest, again)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert dict(results) == {0: (20.0, 2.0), 1: (20.0, 2.0)}


def test_job_throughput_counts_every_replica():
    import bench

    # 2 replicas, 1e9 bytes each, slowest rank 1000 ms -> 2e9 bytes/s
    assert bench.job_throughput(1e9, 2, 1000.0) == pytest.approx(2e9)
    assert bench.job_throughput(3.0, 1, 1.5) == pytest.approx(2000.0)


def test_single_rank_max_is_identity():
    import bench

    assert bench.max_over_ranks(12.5, 1, None) == 12.5


def test_reference_arm_on_other_ranks_does_no_work(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class Args:
        steps, warmup, ref_budget = 1, 0, 0.2

    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` (the CPU oracle arm) on one rank: one JSON line with the
    contract's keys, the same metric and unit as the GPU arm."""
    import json
    import subprocess

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--ref-budget", "0.2"], capture_output=True, text=True, timeout=300,
                         env={k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    import bench

    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    for key in ("value", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
