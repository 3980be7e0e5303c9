"""Host logic of the multi-rank bench on CPU: world size 2 over gloo.

The bench runs one process per GPU, each a replica of the whole linear
sweep on its own micro-batch (no data-path collective).  What crosses ranks
is the timing: every rank's device time is reduced with MAX and the
whole-job throughput counts all ranks' work over that slowest time.  These
tests run that code on gloo ranks; no GPU is involved.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, results):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], "cpu", world)
        flop_step = 69.269232549888e12
        value = bench.job_tflops(world, flop_step, 30, ms)
        # a second collective in the same order on every rank (the e2e leg)
        ms2 = bench.max_over_ranks(times[rank] / 2, "cpu", world)
        results[rank] = (ms, value, ms2)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo_world2():
    world = 2
    times = [2000.0, 2100.0]          # rank 1 is the slower replica
    with mp.get_context("spawn").Manager() as mgr:   # no fork of a process that may hold CUDA
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), times, results), nprocs=world, join=True)
        got = dict(results)
    assert set(got) == {0, 1}
    for rank in range(world):
        ms, value, ms2 = got[rank]
        assert ms == 2100.0                     # every rank sees the slowest time
        assert ms2 == 1050.0
        # all ranks' work over the slowest rank's time
        assert value == pytest.approx(2 * 69.269232549888e12 * 30 / 2.1 / 1e12, rel=1e-12)


def test_single_rank_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(12.5, "cpu", 1) == 12.5
    assert bench.job_tflops(1, 1e12, 10, 1000.0) == pytest.approx(10.0)


def test_job_throughput_is_weak_scaling_sum():
    # the same per-rank step time at N ranks gives N times the throughput
    one = bench.job_tflops(1, 5e12, 7, 350.0)
    for n in (2, 4, 8):
        assert bench.job_tflops(n, 5e12, 7, 350.0) == pytest.approx(n * one)


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def _exchange_main(rank, world, port, results):
    import torch

    import blockwise_fp8_pretraining_b200 as fp8

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        local = torch.full((2, 3), float(rank))
        # stand-ins for CUDA IPC: the handle carries the rank and the values
        shards = fp8.exchange_shards(local, share=lambda t: ("handle", rank, t.tolist()),
                                     rebuild=lambda h: torch.tensor(h[2]) + 100 * (h[1] + 1))
        results[rank] = ([s.tolist() for s in shards], [s is local for s in shards])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_exchange_gloo_world2():
    """exchange_shards gathers one handle per rank over the process group
    and returns the shards in rank order: this rank's own tensor in its
    place, every other rank's rebuilt from its handle."""
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_exchange_main, args=(world, _free_port(), results), nprocs=world, join=True)
        got = dict(results)
    for rank in range(world):
        values, is_local = got[rank]
        assert is_local == [q == rank for q in range(world)]
        for q in range(world):
            want = float(q) if q == rank else float(q) + 100 * (q + 1)
            assert values[q] == [[want] * 3] * 2
