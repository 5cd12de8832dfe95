"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

Every rank runs an independent replica of the decode batch (no data-path
collective); the only cross-rank steps are the barriers around the timed region
and the reduction of the result: the slowest rank's time and the sum of the
units all ranks processed.
"""
import multiprocessing as mp
import os
import socket

import pytest

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    assert bench.dist_env() == (world, rank, rank)
    bench.init_dist("gloo", world)
    bench.barrier(world)
    ms, units = bench.aggregate(10.0 + 5 * rank, 100.0 * (rank + 1), world)
    bench.barrier(world)
    q.put((rank, ms, units))
    dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 15.0, 300.0), (1, 15.0, 300.0)]


def test_single_rank_aggregate_is_identity():
    import bench
    assert bench.aggregate(3.5, 7.0, 1) == (3.5, 7.0)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", "2"]))
    assert capsys.readouterr().out == ""


def test_reference_arm_line(monkeypatch, capsys):
    # the oracle timed on a small sample of the tiny workload: the line's contract
    import json

    import bench
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    bench.run_reference(bench.parse_args(["--impl", "reference", "--workload", "tiny",
                                          "--steps", "2", "--warmup", "3"]))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["higher_is_better"] is True and line["metric"] == bench.METRIC
