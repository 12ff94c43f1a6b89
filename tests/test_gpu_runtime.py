"""Runtime behaviour of the C ABI on the GPU: profiling timers, and the
bounded waits that turn a stalled pipeline into an error status instead of a
hang.

The stall is made on the host side of the contract: the test hook
mxgemm_debug_inject leaves one pipeline stage unarmed, so the kernel's waits
for it run out (after a short limit set for the test) and the kernel records
a site code and returns.  No fault is involved; the context stays usable and
the next launch on the same handle must be correct again.
"""
import numpy as np
import pytest
import torch

import oracle
from microscaling_block_scaled_b200 import mxgemm, synth

from gpu_util import bits

pytestmark = pytest.mark.gpu

F8, F4 = mxgemm.FMT_MXFP8, mxgemm.FMT_MXFP4


def _operands(fmt, M, N, K, seed):
    A32, B32 = synth.operands(M, N, K, seed=seed, device="cpu")
    qa, sa = mxgemm.quantize(fmt, A32.cuda())
    qb, sb = mxgemm.quantize(fmt, B32.cuda())
    oa, osa = oracle.quantize(fmt, A32.numpy())
    ob, osb = oracle.quantize(fmt, B32.numpy())
    ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
    return (qa, sa, qb, sb), (ref, mag)


def test_profiling_reports_repack_and_gemm_times():
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    fmt, M, N, K = F4, 32, 4096, 4096
    (qa, sa, qb, sb), (ref, mag) = _operands(fmt, M, N, K, seed=61)
    with pytest.raises(mxgemm.MXGemmError):
        h.last_timing()                 # nothing profiled yet
    h.set_profiling(True)
    C = h.run(fmt, qa, sa, qb, sb, K=K)
    rep_ms, gemm_ms = h.last_timing()
    assert 0.0 < rep_ms < 50.0 and 0.0 < gemm_ms < 50.0
    ok, rep = oracle.compare(bits(C), ref, mag)
    assert ok, rep
    h.set_profiling(False)
    h.run(fmt, qa, sa, qb, sb, K=K)
    with pytest.raises(mxgemm.MXGemmError):
        h.last_timing()                 # the last run was not profiled
    h.close()


@pytest.mark.parametrize("fmt,M,N,K", [
    (F4, 32, 1024, 2048),       # swapped decode tile
    (F8, 200, 640, 1536),       # 128-column tiles
    (F8, 512, 8192, 256),       # CTA-pair tiles
], ids=["decode", "mid", "pair"])
def test_stalled_stage_times_out_and_handle_recovers(fmt, M, N, K):
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    (qa, sa, qb, sb), (ref, mag) = _operands(fmt, M, N, K, seed=62)
    h.set_wait_limit(20_000_000)        # 20 ms per wait
    h.debug_inject(1)
    h.run(fmt, qa, sa, qb, sb, K=K)
    st, code = h.check_device_error()
    assert st == mxgemm.ERR_TIMEOUT, (st, code, h.describe(fmt, M, N, K))
    assert code in (1, 2, 3, 4, 5), code
    # the error word was cleared by the read; the next run is normal
    h.set_wait_limit(0)
    C = h.run(fmt, qa, sa, qb, sb, K=K)
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0
    ok, rep = oracle.compare(bits(C), ref, mag)
    assert ok, rep
    h.close()
