"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.  Each GPU of a
multi-GPU run is an independent replica of the GEMM (the path has no
exchange step), so the only collective is the max-over-ranks of the timings,
and the whole-job value counts every rank's work in the slowest rank's time.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r timed (r + 1) ms for the step graph and (10 - r) ms end to end
        ms, e2e = bench.max_over_ranks([rank + 1.0, 10.0 - rank])
        value = bench.job_tflops(2.0e12, world, 4, ms)
        out[rank] = (ms, e2e, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, e2e, value = res[r]
        assert ms == 2.0 and e2e == 10.0          # every rank sees the slowest rank's times
        # 2 ranks x 4 steps x 2 TFLOP in 2 ms
        assert value == pytest.approx(2.0e12 * 2 * 4 / 2e-3 / 1e12)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]


def test_reference_arm_rank_other_than_zero_does_no_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    # run_reference returns before touching the oracle or any device on ranks > 0
    class A:
        workload = bench.DEFAULT_WORKLOAD
        steps, warmup, gpus, cpu_seconds = 1, 0, 2, 0.01
    assert bench.run_reference(A) == 0


class _FakeNVML:
    """Stands in for pynvml: a GPU at 1965 MHz (max 1965) whose throttle
    reasons come from a list, one per query."""
    NVML_CLOCK_SM = 1

    def __init__(self, reasons):
        self.reasons = list(reasons)
        self.queries = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        raise RuntimeError("no PCI lookup in the fake")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("gpu", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.queries += 1
        return 1965 if self.queries % 2 else 1905

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons.pop(0) if self.reasons else 0


def test_clock_sampler_reasons_and_in_region_sample(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    fake = _FakeNVML([0x4 | 0x1, 0x40])          # sw_power_cap (+ idle, ignored), then hw_thermal_slowdown
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    clk = bench.ClockSampler(0, period=10.0)     # the thread never samples within the test
    assert clk.ok and clk.max_mhz == 1965
    with clk:
        clk.active = True
        clk.sample_now()                         # as the bench does inside the timed region
        clk.sample_now()
        clk.active = False
    s = clk.summary()
    assert s["samples"] == 2
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["sm_mhz"] == (1965 + 1905) / 2 and s["sm_max_mhz"] == 1965


def test_clock_sampler_takes_one_sample_when_the_region_had_none(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNVML([]))
    clk = bench.ClockSampler(0, period=10.0)
    with clk:
        pass
    s = clk.summary()
    assert s["samples"] == 1 and s["reasons"] == [] and s["sm_mhz"] == 1965


def test_clock_sampler_without_nvml_reports_nothing(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class Broken:
        def nvmlInit(self):
            raise RuntimeError("no driver")
    monkeypatch.setitem(sys.modules, "pynvml", Broken())
    clk = bench.ClockSampler(0, period=10.0)
    assert not clk.ok
    with clk:
        clk.sample_now()
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
