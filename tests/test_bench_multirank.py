"""The N-GPU bench path on CPU: two gloo ranks run the bench's rank seeding and
its max-over-ranks timing reduction; the reference arm does no work on ranks
other than 0."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports (r + 1) ms for the step and (10 - r) ms end to end
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], dist, "cpu")
        seed = bench.rank_seed("gqa70b_long", rank)
        dist.barrier()
        q.put((rank, got, seed))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_by_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] == res[1][1] == [2.0, 10.0]
    # rank 0 runs the named workload, rank 1 an independent batch of its shape
    assert res[0][2] is None and res[1][2] is not None


def test_reference_arm_skips_nonzero_ranks():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload = "tiny"
        steps = 1
        warmup = 1

    assert bench.reference_arm(A(), rank=1, world=2) is None


def test_max_over_ranks_without_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1, 2.5]) == [1.0, 2.5]


def test_step_stats_min_median_p90():
    sys.path.insert(0, ROOT)
    import bench

    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    # spans 1..10 ms in scrambled order
    spans = [7, 3, 10, 1, 5, 9, 2, 8, 4, 6]
    ev = {"a": [Ev(0.0) for _ in spans], "b": [Ev(float(s)) for s in spans]}
    st = bench.step_stats(ev, "a", "b")
    assert st == {"min": 1.0, "median": 5.5, "p90": 9.0}  # nearest rank: 9th of 10
    assert bench.step_stats({"a": [], "b": []}, "a", "b") is None


def test_clock_record_keeps_the_timed_window_and_every_reason():
    import bench
    cs = bench.ClockSampler(0)
    cs.thread = object.__new__(type("T", (), {"join": lambda self, timeout=None: None}))
    # (host time, SM MHz, max MHz, reasons bitmask, watts): two samples before,
    # three inside and one after the timed region
    cs.samples = [(0.0, 1965, 1965, 0, 300.0), (1.0, 1965, 1965, 0, 310.0),
                  (2.0, 1900, 1965, 0x4, 900.0), (2.5, 1800, 1965, 0x4 | 0x40, 950.0),
                  (3.0, 1850, 1965, 0, 920.0), (5.0, 1500, 1965, 0x20, 400.0)]
    cs.mark_timed(1.5, 3.2)
    rec = cs.stop()
    assert rec["samples"] == 3 and rec["sm_mhz"] == 1850 and rec["sm_min_mhz"] == 1800
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert rec["window"] == "timed region"
    assert rec["whole_run"]["samples"] == 6
    assert "sw_thermal_slowdown" in rec["whole_run"]["reasons"]
