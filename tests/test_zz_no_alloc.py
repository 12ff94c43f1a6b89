"""mxgemm_run_noalloc: the hot path for callers that cannot allocate device
memory when they run the product (allocator hooks, runtimes that allocate
everything up front).  It must give the same results as mxgemm_run.

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


def _bits(C):
    return C.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("fmt", [mxgemm.FMT_MXFP8, mxgemm.FMT_MXFP4], ids=["mxfp8", "mxfp4"])
def test_noalloc_matches_run_on_two_calls_in_a_row(fmt):
    torch.cuda.set_device(0)
    h = mxgemm.Handle()
    # two different shapes back to back: the second call reuses (and must
    # fully rewrite) the scratch the first one left behind
    for (M, N, K), seed in (((64, 1024, 1024), 51), ((200, 520, 768), 52)):
        A32, B32 = synth.operands(M, N, K, seed=seed)
        qa, sa = mxgemm.quantize(fmt, A32.cuda())
        qb, sb = mxgemm.quantize(fmt, B32.cuda())
        ref_run = h.run(fmt, qa, sa, qb, sb, K=K)
        got = mxgemm.run_noalloc(fmt, qa, sa, qb, sb, K=K)
        torch.cuda.synchronize()
        # the tolerance the parity tests use, taken around mxgemm_run's result
        # (sum |a b| from the oracle on the oracle's own quantisation)
        oa, osa = oracle.quantize(fmt, A32.numpy())
        ob, osb = oracle.quantize(fmt, B32.numpy())
        _, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
        ok, rep = oracle.compare(_bits(got), _bits(ref_run), mag)
        assert ok, ("noalloc differs from mxgemm_run", M, N, K, rep)
    h.close()


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
