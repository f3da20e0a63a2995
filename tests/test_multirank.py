"""The N > 1 path of bench.py on CPU: two gloo ranks (no GPU).

Every (sequence, head) pair is independent, so N GPUs run N replicas on
independent batches (weak scaling) with no collective on the data path; the
only exchange is the timing: a barrier on both sides of the timed steps and
the maximum of the per-rank times.  These tests run that host logic with the
gloo backend in two processes on 127.0.0.1.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench.rank_helpers(world)
        barrier()
        # per-rank step times differ; the job is as slow as its slowest rank
        local_ms = 100.0 + 25.0 * rank
        worst = max_over_ranks(local_ms)
        value = bench.job_throughput(world, 1000, 4, worst)
        # replicas draw independent batches (seed = rank)
        from kda_inputs import make_prefill
        inp = make_prefill("tiny_f32", device="cpu", seed=rank)
        mine = torch.tensor([float(inp.q.double().sum()), float(inp.v.double().sum())], dtype=torch.float64)
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, mine)
        barrier()
        out[rank] = (worst, value, [g.tolist() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        worst, value, gathered = out[r]
        assert worst == 125.0                                  # max over ranks, seen by every rank
        assert value == pytest.approx(world * 1000 * 4 / 0.125)  # whole-job units per second
        assert gathered[0] != gathered[1]                     # independent replica inputs
    assert out[0][2] == out[1][2]


def test_single_rank_helpers_are_no_ops():
    barrier, max_over_ranks = bench.rank_helpers(1)
    barrier()
    assert max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 10, 2, 1000.0) == pytest.approx(20.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup = 2, 3
    assert bench.run_reference(Args(), world=2, rank=1) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_its_json_line(capsys):
    """bench.py --impl reference on rank 0: one JSON line with the keys the
    contract reads (the fp64 oracle timed on the host cores, a bounded sample)."""
    import json

    class Args:
        steps, warmup, gpus = 1, 0, 1
    bench.run_reference(Args(), world=1, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("packed varlen prefill: 64 sequences")
