"""The N > 1 path of bench.py without a GPU: replicas on `gloo` ranks (world size 2)
agree on the slowest rank's time, the whole-job throughput counts every replica's tokens,
and the reference arm does its work on rank 0 only."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")   # rank 1 is the slow one
        tput = bench.replica_throughput(4096, world, ms)
        q.put((rank, ms, tput))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[1] for g in got] == [15.0, 15.0]
    # 2 replicas x 4096 tokens per 15 ms step
    assert all(abs(g[2] - 2 * 4096 / 0.015) < 1e-6 for g in got)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.replica_throughput(128, 1, 2.0) == 64000.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class Args:
        workload = "tiny"
        steps = 2
        warmup = 3
    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_on_one_rank_prints_one_line(monkeypatch, capsys):
    if torch.cuda.is_available():
        pytest.skip("CPU-only check")
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class Args:
        workload = "tiny"
        steps = 2
        warmup = 3
    bench.run_reference(Args())
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    import json
    line = json.loads(out[0])
    assert line["impl"] == "reference" and line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
