"""The benchmark's multi-process host logic on CPU (gloo, 2 ranks).

The path shards with no data exchange, so the only cross-rank step is the
reduction of the per-rank timings to their maximum (the job is as slow as its
slowest rank); the reference arm runs on rank 0 alone.
"""
import os
import sys

import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = [1.0 + rank, 10.0 - rank, 3.5, 0.0 if rank else 7.0]
        out[rank] = bench.max_over_ranks(vals, tdist, "cpu")

        class A:
            prefill, steps, warmup, ref_seconds = "tiny", 1, 3, 1.0

        if rank != 0:
            out[10 + rank] = bench.run_reference(A, rank)  # no work off rank 0
    finally:
        tdist.destroy_process_group()


def test_timings_reduce_to_the_max_over_two_gloo_ranks():
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        want = [2.0, 10.0, 3.5, 7.0]
        assert out[0] == want and out[1] == want
        assert out[11] is None


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.0, 2.0], None, "cpu") == [1.0, 2.0]


def test_clock_summary_keeps_only_the_timed_window():
    sys.path.insert(0, ROOT)
    import bench

    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.ok, cs.max_mhz = True, 1965
    # (time, MHz, reasons, util): cold before the region, power-capped inside it
    cs.samples = [(0.0, 1965, 0x0, 90), (0.5, 1965, 0x0, 90), (1.0, 1800, 0x4, 99),
                  (1.1, 1790, 0x4, 99), (1.2, 1810, 0x4, 99), (2.0, 1965, 0x1, 0)]
    s = cs.summary(0.95, 1.25)
    assert s["sm_mhz"] == 1800 and s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    # a region between two samples reports the nearest ones
    s = cs.summary(0.6, 0.7)
    assert s["samples"] == 2 and s["sm_mhz"] in (1965, 1882.5)
    # no window: every sample that is not idle
    assert cs.summary()["samples"] == 5
