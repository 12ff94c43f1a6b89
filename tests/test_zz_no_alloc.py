"""mxgemm_run_noalloc: the hot path for callers that cannot allocate device
memory when they run the product (allocator hooks, runtimes that allocate
everything up front).  Its results must match the CPU oracle within the
parity tolerance, match mxgemm_run bit for bit (both compute the same whole
tiles in the same order), and a call must not change the device's free
memory.

Collected last on purpose (file name), so a stop-at-first-failure run has
executed every other test before this one; it also passes on its own in a
fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from microscaling_block_scaled_b200 import mxgemm, synth

pytestmark = pytest.mark.gpu

F8, F4 = mxgemm.FMT_MXFP8, mxgemm.FMT_MXFP4


def _bits(C):
    return C.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def _scratch_bytes(fmt, M, N, K):
    """Repacked-scale bytes of A and B (the library's layout: 128-row blocks
    padded to pairs, K/128 atoms rounded up to 4 (MXFP8) or 8 (MXFP4))."""
    step = 4 if fmt == F8 else 8
    ka = -(-(K // 128) // step) * step
    return (-(-M // 256) + -(-N // 256)) * 2 * ka * 512


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
def test_noalloc_matches_oracle_and_run_on_two_calls_in_a_row(fmt):
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    h.set_schedule(mxgemm.SCHED_DP)        # whole tiles, as the no-allocation path computes them
    # two different shapes back to back: the second call reuses (and must
    # fully rewrite) the scratch the first one left behind; the second shape
    # takes the CTA-pair plan
    shapes = (((200, 520, 768), 51), ((512, 8192, 256), 52))
    inputs = []
    for (M, N, K), seed in shapes:
        A32, B32 = synth.operands(M, N, K, seed=seed)
        qa, sa = mxgemm.quantize(fmt, A32.cuda())
        qb, sb = mxgemm.quantize(fmt, B32.cuda())
        inputs.append(((M, N, K), A32, B32, qa, sa, qb, sb))
    assert "pair=1" in h.describe(fmt, 512, 8192, 256)
    # mxgemm_run first: every kernel the no-allocation calls launch is then
    # loaded, so the free-memory check below sees only what the calls do
    runs = [h.run(fmt, qa, sa, qb, sb, K=K) for (_, _, K), _, _, qa, sa, qb, sb in inputs]
    outs = [torch.empty_like(r) for r in runs]
    (M, N, K), _, _, qa, sa, qb, sb = inputs[0]
    mxgemm.run_noalloc(fmt, qa, sa, qb, sb, C=outs[0], K=K)     # sets the device up
    free0 = _free_bytes()
    for ((M, N, K), _, _, qa, sa, qb, sb), C in zip(inputs, outs):
        mxgemm.run_noalloc(fmt, qa, sa, qb, sb, C=C, K=K)
    free1 = _free_bytes()
    assert free1 == free0, ("device memory changed across no-allocation calls", free0 - free1)
    for ((M, N, K), A32, B32, qa, sa, qb, sb), C, R in zip(inputs, outs, runs):
        oa, osa = oracle.quantize(fmt, A32.numpy())
        ob, osb = oracle.quantize(fmt, B32.numpy())
        ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
        ok, rep = oracle.compare(_bits(C), ref, mag)
        assert ok, ("noalloc differs from the oracle", M, N, K, rep)
        assert np.array_equal(_bits(C), _bits(R)), ("noalloc differs from mxgemm_run", M, N, K)
    h.close()


def test_noalloc_near_the_scratch_limit():
    """A problem whose repacked scales fill most of the fixed scratch: checked
    against mxgemm_run bit for bit and against the oracle on sampled rows."""
    torch.cuda.set_device(0)
    fmt, M, N, K = F4, 1024, 28672, 8192
    need = _scratch_bytes(fmt, M, N, K)
    assert 0.85 * (8 << 20) < need <= (8 << 20), need
    A32, B32 = synth.operands(M, N, K, seed=53, device="cuda")
    qa, sa = mxgemm.quantize(fmt, A32)
    qb, sb = mxgemm.quantize(fmt, B32)
    h = mxgemm.Handle()
    R = h.run(fmt, qa, sa, qb, sb, K=K)
    C = torch.empty_like(R)
    for _ in range(2):
        C.zero_()
        mxgemm.run_noalloc(fmt, qa, sa, qb, sb, C=C, K=K)
        torch.cuda.synchronize()
        assert torch.equal(C.view(torch.int16), R.view(torch.int16))
    rows = np.array([0, 1, 255, 256, 511, 777, M - 1])
    oa, osa = oracle.quantize(fmt, A32[torch.from_numpy(rows).cuda()].cpu().numpy())
    ob, osb = oracle.quantize(fmt, B32.cpu().numpy())
    ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
    ok, rep = oracle.compare(_bits(C)[rows], ref, mag)
    assert ok, rep
    h.close()
    # thirteen more 256-row blocks of B: just past the limit, rejected before any launch
    st = mxgemm.mxgemm_run_noalloc(fmt, M, N + 13 * 256, K, qa.data_ptr(), sa.data_ptr(), qb.data_ptr(),
                                   sb.data_ptr(), C.data_ptr(), 0)
    assert _scratch_bytes(fmt, M, N + 13 * 256, K) > (8 << 20)
    assert st == mxgemm.ERR_TOO_LARGE


def test_noalloc_rejects_too_large_and_bad_args():
    torch.cuda.set_device(0)
    t = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    p = t.data_ptr()
    # 2^20 rows of scales at K = 8192 need far more than the fixed scratch
    st = mxgemm.mxgemm_run_noalloc(mxgemm.FMT_MXFP8, 1 << 20, 1 << 20, 8192, p, p, p, p, p, 0)
    assert st == mxgemm.ERR_TOO_LARGE
    st = mxgemm.mxgemm_run_noalloc(mxgemm.FMT_MXFP8, 4, 4, 100, p, p, p, p, p, 0)
    assert st == mxgemm.ERR_INVALID_ARG
    st = mxgemm.mxgemm_run_noalloc(mxgemm.FMT_MXFP8, 4, 4, 128, p + 4, p, p, p, p, 0)
    assert st == mxgemm.ERR_ALIGNMENT
