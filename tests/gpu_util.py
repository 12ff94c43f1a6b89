"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare it with the CPU oracle on identical FP32 inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from microscaling_block_scaled_b200 import mxgemm, synth

FMTS = {"mxfp8": mxgemm.FMT_MXFP8, "mxfp4": mxgemm.FMT_MXFP4}

_handle = None


def handle() -> mxgemm.Handle:
    global _handle
    if _handle is None:
        torch.cuda.set_device(0)
        _handle = mxgemm.Handle()
    return _handle


def bits(C: torch.Tensor) -> np.ndarray:
    return C.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_quantize(fmt: int, X: torch.Tensor):
    return mxgemm.quantize(fmt, X.cuda().contiguous())


def assert_parity(got_bits, ref_bits, abssum, what=""):
    ok, rep = oracle.compare(got_bits, ref_bits, abssum)
    assert ok, ("parity failed %s" % what, rep)
    return rep


def full_case(fmt: int, M: int, N: int, K: int, seed: int, kind: str = "normal", schedule=None):
    """Quantise on both sides (must agree bit for bit), run the GEMM on the GPU,
    compare every output element with the oracle."""
    A32, B32 = synth.operands(M, N, K, seed=seed, kind=kind, device="cpu")
    qa, sa = gpu_quantize(fmt, A32)
    qb, sb = gpu_quantize(fmt, B32)
    oa, osa = oracle.quantize(fmt, A32.numpy())
    ob, osb = oracle.quantize(fmt, B32.numpy())
    assert np.array_equal(qa.cpu().numpy(), oa) and np.array_equal(sa.cpu().numpy(), osa), "A quantiser mismatch"
    assert np.array_equal(qb.cpu().numpy(), ob) and np.array_equal(sb.cpu().numpy(), osb), "B quantiser mismatch"
    h = handle()
    if schedule is not None:
        h.set_schedule(*schedule)
    try:
        C = h.run(fmt, qa, sa, qb, sb, K=K)
        torch.cuda.synchronize()
    finally:
        if schedule is not None:
            h.set_schedule(mxgemm.SCHED_AUTO)
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, ("device error word", code)
    ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
    return assert_parity(bits(C), ref, mag, "fmt=%d %dx%dx%d" % (fmt, M, N, K)), C


def sampled_case(fmt: int, M: int, N: int, K: int, seed: int, kind: str = "normal", n_rows: int = 96,
                 n_cols: int = 96, rng_seed: int = 1234):
    """Full-size run with inputs drawn by the CUDA generator; the oracle checks
    the grid of sampled rows x sampled columns (plus the first and last of each),
    quantising only those rows on the host."""
    A32, B32 = synth.operands(M, N, K, seed=seed, kind=kind, device="cuda")
    qa, sa = mxgemm.quantize(fmt, A32)
    qb, sb = mxgemm.quantize(fmt, B32)
    h = handle()
    C = h.run(fmt, qa, sa, qb, sb, K=K)
    torch.cuda.synchronize()
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, ("device error word", code)
    rng = np.random.default_rng(rng_seed)
    rm = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, min(n_rows, M))]))
    rn = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, min(n_cols, N))]))
    a_rows = A32[torch.from_numpy(rm).cuda()].cpu().numpy()
    b_rows = B32[torch.from_numpy(rn).cuda()].cpu().numpy()
    oa, osa = oracle.quantize(fmt, a_rows)
    ob, osb = oracle.quantize(fmt, b_rows)
    assert np.array_equal(qa[torch.from_numpy(rm).cuda()].cpu().numpy(), oa), "A quantiser mismatch"
    assert np.array_equal(sa[torch.from_numpy(rm).cuda()].cpu().numpy(), osa), "A scale mismatch"
    assert np.array_equal(qb[torch.from_numpy(rn).cuda()].cpu().numpy(), ob), "B quantiser mismatch"
    assert np.array_equal(sb[torch.from_numpy(rn).cuda()].cpu().numpy(), osb), "B scale mismatch"
    ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
    got = bits(C[torch.from_numpy(rm).cuda()][:, torch.from_numpy(rn).cuda()])
    rep = assert_parity(got, ref, mag, "sampled fmt=%d %dx%dx%d" % (fmt, M, N, K))
    # properties that hold at any size: finite inputs give a finite output
    assert bool(torch.isfinite(C.float()).all())
    return rep


def rows_cols_points_case(fmt: int, M: int, N: int, K: int, seed: int, kind: str = "normal", n_rows: int = 64,
                          n_cols: int = 64, n_points: int = 65536, rng_seed: int = 4321):
    """Full-size run with inputs drawn by the CUDA generator, checked against
    the oracle on n_rows whole rows of C (every column), n_cols whole columns
    (every row) and n_points random elements.  The first and last row and
    column are always among them, so every output tile of the GEMM has
    checked elements.  Both operands are quantised in full on the host and
    must agree with the device quantiser bit for bit."""
    A32, B32 = synth.operands(M, N, K, seed=seed, kind=kind, device="cuda")
    qa, sa = mxgemm.quantize(fmt, A32)
    qb, sb = mxgemm.quantize(fmt, B32)
    h = handle()
    C = h.run(fmt, qa, sa, qb, sb, K=K)
    torch.cuda.synchronize()
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, ("device error word", code)
    plan = h.describe(fmt, M, N, K)
    got_all = bits(C)
    assert bool(torch.isfinite(C.float()).all())
    del C
    oa, osa = oracle.quantize(fmt, A32.cpu().numpy())
    assert np.array_equal(qa.cpu().numpy(), oa) and np.array_equal(sa.cpu().numpy(), osa), "A quantiser mismatch"
    del A32, qa, sa
    ob, osb = oracle.quantize(fmt, B32.cpu().numpy())
    assert np.array_equal(qb.cpu().numpy(), ob) and np.array_equal(sb.cpu().numpy(), osb), "B quantiser mismatch"
    del B32, qb, sb
    torch.cuda.empty_cache()
    rng = np.random.default_rng(rng_seed)
    rm = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(n_rows, M) - 2, replace=False)]))
    rn = np.unique(np.concatenate([[0, N - 1], rng.choice(N, min(n_cols, N) - 2, replace=False)]))
    ref, _, mag = oracle.gemm(fmt, K, oa[rm], osa[rm], ob, osb)
    assert_parity(got_all[rm], ref, mag, "whole rows fmt=%d %dx%dx%d" % (fmt, M, N, K))
    ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob[rn], osb[rn])
    assert_parity(got_all[:, rn], ref, mag, "whole columns fmt=%d %dx%dx%d" % (fmt, M, N, K))
    pm = rng.integers(0, M, n_points)
    pn = rng.integers(0, N, n_points)
    ref, _, mag = oracle.gemm_points(fmt, K, oa, osa, ob, osb, pm, pn)
    assert_parity(got_all[pm, pn], ref, mag, "random points fmt=%d %dx%dx%d" % (fmt, M, N, K))
    return plan, len(rm), len(rn)


def rows_case(fmt: int, M: int, N: int, K: int, seed: int, n_rows: int = 48, rng_seed: int = 7):
    """CPU-drawn inputs, GPU GEMM through mxgemm_run, oracle on a sample of
    whole output rows (every column of those rows)."""
    A32, B32 = synth.operands(M, N, K, seed=seed, kind="normal", device="cpu")
    qa, sa = gpu_quantize(fmt, A32)
    qb, sb = gpu_quantize(fmt, B32)
    h = handle()
    C = h.run(fmt, qa, sa, qb, sb, K=K)
    torch.cuda.synchronize()
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, ("device error word", code)
    rng = np.random.default_rng(rng_seed)
    rm = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, n_rows)]))
    oa, osa = oracle.quantize(fmt, A32.numpy()[rm])
    ob, osb = oracle.quantize(fmt, B32.numpy())
    assert np.array_equal(qb.cpu().numpy(), ob) and np.array_equal(sb.cpu().numpy(), osb), "B quantiser mismatch"
    ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob, osb)
    got = bits(C)[rm]
    return assert_parity(got, ref, mag, "rows fmt=%d %dx%dx%d" % (fmt, M, N, K)), h.describe(fmt, M, N, K)
