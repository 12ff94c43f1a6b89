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
    (F4, 32, 1024, 4096),       # swapped decode tiles, K split over clusters of two
    (F8, 64, 1024, 4096),       # swapped decode tiles, K split over clusters of four
    (F8, 200, 640, 1536),       # 128-column tiles
    (F8, 512, 8192, 256),       # CTA-pair tiles
], ids=["decode", "decode-ksplit4", "mid", "pair"])
def test_stalled_stage_times_out_and_handle_recovers(fmt, M, N, K):
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    if M <= 64:
        # every CTA of every cluster stalls: the reduction waits are never reached
        assert "sched=ksplit" in h.describe(fmt, M, N, K)
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


@pytest.mark.parametrize("prefetch_b", [False, True], ids=["plain", "prefetch_b"])
def test_back_to_back_runs_wait_for_the_previous_gemm(prefetch_b):
    """Two one-launch runs queued back to back with no synchronisation.  The
    second starts as a programmatic dependent of the first, so its CTAs can
    be resident while the first still runs.  It reads the first one's output
    as its A operand (read after write) and writes its C over the first
    one's A operand (write after read): both must see the first GEMM
    complete.  Under the prefetch-B promise only B may be read early.  The
    second GEMM is MXFP4, whose codes are all finite, so any byte pattern of
    the first output is a valid operand."""
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    h.set_prefetch_b(prefetch_b)
    M, N1, K1 = 32, 512, 16384
    N2, K2 = 2048, 4 * N1                   # A2 = the bytes of C1, two E2M1 codes per byte
    assert "scales=fused" in h.describe(F8, M, N1, K1)
    assert "scales=fused" in h.describe(F4, M, N2, K2)
    A1f, B1f = synth.operands(M, N1, K1, seed=71, device="cuda")
    qa1, sa1 = mxgemm.quantize(F8, A1f)
    qb1, sb1 = mxgemm.quantize(F8, B1f)
    _, B2f = synth.operands(M, N2, K2, seed=72, device="cuda")
    qb2, sb2 = mxgemm.quantize(F4, B2f)
    sa2 = torch.full((M, K2 // 32), 120, dtype=torch.uint8, device="cuda")
    # the first GEMM alone, on a copy of its A
    C1_ref = h.run(F8, qa1.clone(), sa1, qb1, sb1, K=K1)
    torch.cuda.synchronize()
    # the chain: C1 starts zeroed; C2 is laid over the first half of A1
    C1 = torch.zeros((M, N1), dtype=torch.bfloat16, device="cuda")
    C2 = qa1.view(-1)[: M * N2 * 2].view(torch.bfloat16).view(M, N2)
    h.run(F8, qa1, sa1, qb1, sb1, C=C1, K=K1)
    h.run(F4, C1.view(torch.uint8), sa2, qb2, sb2, C=C2, K=K2)
    torch.cuda.synchronize()
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, code
    assert np.array_equal(bits(C1), bits(C1_ref)), "the second GEMM wrote A1 before the first one read it"
    # the second GEMM again, alone, from the final C1
    a2 = C1.view(torch.uint8).clone()
    C2_ref = h.run(F4, a2, sa2, qb2, sb2, K=K2)
    torch.cuda.synchronize()
    assert np.array_equal(bits(C2), bits(C2_ref)), "the second GEMM read A before the first one wrote it"
    ref, _, mag = oracle.gemm(F4, K2, a2.cpu().numpy(), sa2.cpu().numpy(), qb2.cpu().numpy(), sb2.cpu().numpy())
    ok, rep = oracle.compare(bits(C2_ref), ref, mag)
    assert ok, rep
    h.close()


def test_capture_needs_a_reserved_workspace():
    """A run whose shape needs a larger workspace than the handle holds cannot
    grow it inside a stream capture: it returns MXGEMM_ERR_CAPTURE and
    launches nothing.  After mxgemm_reserve the same run captures, and the
    replayed graph gives the oracle's result."""
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    fmt, M, N, K = F8, 512, 8192, 512          # CTA-pair plan: repacked scales in the workspace
    (qa, sa, qb, sb), (ref, mag) = _operands(fmt, M, N, K, seed=63)
    C = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = mxgemm.mxgemm_run(h.h, fmt, M, N, K, qa.data_ptr(), sa.data_ptr(), qb.data_ptr(), sb.data_ptr(),
                               C.data_ptr(), s.cuda_stream)
    assert st == mxgemm.ERR_CAPTURE, st
    del g
    h.reserve(fmt, M, N, K)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = mxgemm.mxgemm_run(h.h, fmt, M, N, K, qa.data_ptr(), sa.data_ptr(), qb.data_ptr(), sb.data_ptr(),
                               C.data_ptr(), s.cuda_stream)
    assert st == mxgemm.OK, st
    g.replay()
    torch.cuda.synchronize()
    ok, rep = oracle.compare(bits(C), ref, mag)
    assert ok, rep
    del g
    h.close()
