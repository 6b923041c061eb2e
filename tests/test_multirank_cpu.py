"""The multi-rank host logic of bench.py with 2 gloo ranks on CPU.

Each rank runs its own copy of the workload (batches and heads are
independent, so there is no exchange on the data path); the job time is the
slowest rank's, and the reference arm runs on rank 0 only.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 3.0 * rank          # rank 1 is the slower one
        ms_max = bench.max_over_ranks(ms)
        value = bench.weak_scaled_value(4096, 100, world, ms_max)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(rank))
        q.put((rank, ms_max, value, seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, value, seeds in results:
        assert ms_max == 13.0                       # max over ranks
        assert value == pytest.approx(2 * 4096 * 100 / 0.013)
        assert len(set(seeds)) == world             # each replica draws its own batch


def test_single_process_is_identity():
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.weak_scaled_value(10, 2, 1, 1000.0) == pytest.approx(20.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    args = argparse.Namespace(steps=1, warmup=1)
    w = bench.wl.WORKLOADS["sana0.6b_512px"]
    bench.main_reference(args, w, rank=1, world=2)
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("op", ["layer", "qkv"])
def test_reference_arm_prints_one_contract_line(capsys, op):
    import argparse
    import json
    args = argparse.Namespace(steps=1, warmup=3, op=op, ref_budget=2.0)
    w = bench.wl.WORKLOADS["sana0.6b_512px"]
    bench.main_reference(args, w, rank=0, world=1)
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["metric"] == bench.METRICS[op]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
