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
