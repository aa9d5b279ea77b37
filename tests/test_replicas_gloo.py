"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

The path runs as independent replicas (one round per GPU, no exchange), so
the only cross-rank steps are the barriers and the max-over-ranks timing; the
reference arm runs on rank 0 alone.
"""
import argparse
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, w)  # rank 1 is the slow one
        dist.barrier()
        out.put((rank, slowest, bench.whole_job_rate(50, w, slowest)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(out.get(timeout=10) for _ in range(world))
    for rank, slowest, rate in got:
        assert slowest == 15.0
        assert rate == pytest.approx(50 * 2 / 0.015)


def test_single_rank_is_its_own_maximum():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.whole_job_rate(10, 1, 5.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(workload="tiny", warmup=0, steps=1, gpus=2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = argparse.Namespace(workload="tiny", warmup=0, steps=10, gpus=1)
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "rounds/s" and line["value"] > 0
    assert line["metric"] == "draft+schedule+verify rounds/sec" and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "rounds/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
