"""The N > 1 host logic of bench.py on CPU: two gloo ranks, each timing its
own replica, agree on the max-over-ranks time and on the job throughput."""

from __future__ import annotations

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" 100 + 25 r ms for 10 steps of 1e12 FLOP each
        ms = bench.max_over_ranks(100.0 + 25.0 * rank, world)
        value = bench.aggregate_throughput(world, 10, 1e12, ms)
        results[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(results)
    assert res[0] == res[1]
    ms, value = res[0]
    assert ms == 125.0
    # 2 replicas x 10 steps x 1e12 FLOP in 0.125 s
    assert value == pytest.approx(2 * 10 * 1e12 / 0.125 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(42.0, 1) == 42.0
    assert bench.aggregate_throughput(1, 4, 2e12, 1000.0) == pytest.approx(8.0)


def test_reference_arm_prints_on_rank0_only(capsys, monkeypatch):
    import argparse
    from ring_attention_ordered_b200.inputs import WORKLOADS
    args = argparse.Namespace(steps=1, warmup=0)
    assert bench.run_reference(args, WORKLOADS["l512_d64_noncausal"], 2, 1) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank0(capsys):
    import argparse
    import json
    from ring_attention_ordered_b200.inputs import WORKLOADS
    args = argparse.Namespace(steps=1, warmup=0, ref_budget=0.05)
    assert bench.run_reference(args, WORKLOADS["l512_d64_noncausal"], 1, 0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
