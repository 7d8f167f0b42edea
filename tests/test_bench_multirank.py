"""The bench's multi-rank host logic on CPU: two gloo ranks (one process per rank,
as torchrun starts them) reduce their local timings and byte counts exactly as
one GPU per rank would over NCCL; the reference arm does its work on rank 0
only."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: 10 (r + 1) ms of device time over (r + 1) GB
        value, ms = bench.aggregate(float(rank + 1) * 1e9, 10.0 * (rank + 1), world)
        mx = bench.reduce_max(float(rank), world)
        sm = bench.reduce_sum(float(rank + 1), world)
        out[rank] = (value, ms, mx, sm)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    # total 3 GB over the slowest rank's 20 ms = 150 GB/s, the same on every rank
    for r in range(world):
        value, ms, mx, sm = res[r]
        assert ms == pytest.approx(20.0)
        assert value == pytest.approx(3e9 / 20e-3 / 1e9)
        assert mx == 1.0 and sm == 3.0


def test_single_rank_aggregate_is_local():
    sys.path.insert(0, ROOT)
    import bench
    value, ms = bench.aggregate(2e9, 4.0, 1)
    assert ms == 4.0 and value == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    import argparse
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, impl="reference", splits=0,
                              no_cpu_baseline=True, no_quantize=True, workload="gqa32k")
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_oracle_samples_of_the_bench_legs_run_on_the_host():
    """The CPU oracle timings beside the multi-token and key-moments legs draw their
    inputs on the host and run the oracle only."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.WORKLOADS["gqa32k"].scaled(seed=0)
    sec, comp, thr = bench.oracle_prefill_sample(w, n=4, context=512, reps=1)
    assert sec > 0 and comp == 512 - w.W and thr >= 1
    sec, nb, thr = bench.oracle_moments_sample(synth.WORKLOADS["aqjl"], tokens=64, reps=1)
    assert sec > 0 and nb == 8 * 64 * 128 * 2 and thr >= 1
