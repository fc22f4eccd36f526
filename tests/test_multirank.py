"""The multi-GPU path of bench.py on CPU ranks (gloo, world size 2).

There is no data-path collective: the replicas make independent chunks (own
seeds). The only cross-rank step is the timing reduction, which takes the
slowest rank's time and counts the chunks of all ranks. It runs here on gloo
with rank-dependent times. The reference arm does its work on rank 0 only.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        out[rank] = (ms, bench.job_ms_per_chunk(ms / 4, world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timing_takes_the_slowest_rank_and_counts_all_chunks():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        ms, value = out[r]
        assert ms == 15.0                  # max over ranks, on every rank
        assert value == 15.0 / 4 / world   # 4 steps, 2 chunks per step for the job


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.job_ms_per_chunk(3.0, 1) == 3.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class A:
        config, seed, warmup, steps, gpus = 2, 0, 0, 1, 2
    assert bench.run_reference(A(), rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


def test_step_percentiles():
    q = bench.step_percentiles([4.0, 4.1, 3.9, 4.05, 5.0])
    assert q == {"median": 4.05, "p10": 3.94, "p90": 4.64}
