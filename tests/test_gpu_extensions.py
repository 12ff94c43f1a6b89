"""GPU parity of the extensions beyond the MX product, through the C ABI,
against the CPU oracle:

* the BF16-input activation quantiser (bit for bit);
* the fused epilogue act(A B^T + bias) + residual (tolerance of
  oracle.tolerance_fused) on every one-CTA path: swapped decode tiles, plain
  tiles, forced split-K and stream-K;
* the quantised output (the next layer's MX operand): bit for bit with the
  oracle's quantiser applied to the oracle's BF16 result wherever the GPU's
  BF16 result equals the oracle's (everywhere for integer-exact inputs);
* the dense BF16 GEMM (tolerance of the product rule);
* the grouped GEMM with uneven and empty groups, in MXFP8, MXFP4 and BF16.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from microscaling_block_scaled_b200 import mxgemm, synth

from gpu_util import assert_parity, bits, handle

pytestmark = pytest.mark.gpu

F8, F4, BF = mxgemm.FMT_MXFP8, mxgemm.FMT_MXFP4, mxgemm.FMT_BF16
ACTS = [mxgemm.ACT_NONE, mxgemm.ACT_RELU, mxgemm.ACT_SILU, mxgemm.ACT_GELU]


def _bf16(x):
    """float array -> (BF16 bit patterns numpy uint16, CUDA bfloat16 tensor)."""
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.uint16))
    return b, torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)


def _mx_operands(fmt, M, N, K, seed, kind="normal"):
    A32, B32 = synth.operands(M, N, K, seed=seed, kind=kind)
    oa, osa = oracle.quantize(fmt, A32.numpy())
    ob, osb = oracle.quantize(fmt, B32.numpy())
    dev = [torch.from_numpy(x).cuda() for x in (oa, osa, ob, osb)]
    return (oa, osa, ob, osb), dev


def _with_schedule(h, sched, fn):
    if sched is not None:
        h.set_schedule(*sched)
    try:
        return fn()
    finally:
        if sched is not None:
            h.set_schedule(mxgemm.SCHED_AUTO)


def _no_device_error(h):
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, ("device error word", code)


# ------------------------------------------------------ BF16 quantiser

@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("kind", ["normal", "heavy"])
def test_bf16_quantiser_bit_exact(fmt, kind):
    X32, _ = synth.operands(130, 1, 1024, seed=41, kind=kind)
    xb, xt = _bf16(X32.numpy())
    q, s = mxgemm.quantize_bf16(fmt, xt)
    oq, os_ = oracle.quantize_bf16(fmt, xb)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
def test_bf16_quantiser_edge_blocks(fmt):
    r = np.zeros(32 * 8, dtype=np.float32)
    r[32:64] = -0.0
    r[64] = 2.0 ** -130                       # BF16 subnormal amax
    r[96:128] = np.nan
    r[128] = -np.inf
    r[160] = 3.0e38
    r[161] = -2.5e38
    r[192:224] = np.linspace(-9.0, 9.0, 32)
    r[224:256] = 2.0 ** -133                  # smallest BF16 subnormal
    X = np.stack([r, np.random.default_rng(2).standard_normal(r.shape).astype(np.float32)])
    xb, xt = _bf16(X)
    q, s = mxgemm.quantize_bf16(fmt, xt)
    oq, os_ = oracle.quantize_bf16(fmt, xb)
    assert np.array_equal(s.cpu().numpy(), os_), (s.cpu().numpy(), os_)
    assert np.array_equal(q.cpu().numpy(), oq)


# ------------------------------------------------------- fused epilogue

FUSED_PATHS = {
    "swap": ((32, 512, 1024), None),
    "plain": ((200, 384, 768), None),
    "large-m-one-cta": ((640, 1024, 512), None),
    "splitk3": ((100, 640, 2048), (mxgemm.SCHED_SPLITK, 3, 0)),
    "streamk37": ((100, 640, 2048), (mxgemm.SCHED_STREAMK, 1, 37)),
    "swap-splitk3": ((48, 512, 2048), (mxgemm.SCHED_SPLITK, 3, 0)),
    "swap-ksplit4": ((48, 512, 2048), (mxgemm.SCHED_KSPLIT, 4, 0)),
    "swap-dp": ((48, 512, 2048), (mxgemm.SCHED_DP, 1, 0)),
    # 200 decode tiles on 148 CTAs: some CTAs run two tiles, so the epilogue
    # warps apply the operations themselves (the all-warps form is for a
    # CTA's only tile)
    "swap-multitile": ((24, 128 * 200, 256), None),
}


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("act", ACTS, ids=["none", "relu", "silu", "gelu"])
@pytest.mark.parametrize("path", list(FUSED_PATHS))
def test_fused_epilogue(fmt, act, path):
    (M, N, K), sched = FUSED_PATHS[path]
    (oa, osa, ob, osb), (qa, sa, qb, sb) = _mx_operands(fmt, M, N, K, seed=M + N + act)
    rng = np.random.default_rng(act * 10 + M)
    bias_b, bias_t = _bf16(rng.standard_normal(N) * 4)
    res_b, res_t = _bf16(rng.standard_normal((M, N)) * 4)
    h = handle()
    _, ex, mag = oracle.gemm(fmt, K, oa, osa, ob, osb, want_exact=True)
    for use_bias, use_res in ((True, True), (True, False), (False, True)):
        C = _with_schedule(h, sched, lambda: h.run_fused(
            fmt, qa, sa, qb, sb, bias=bias_t if use_bias else None, act=act,
            residual=res_t if use_res else None, K=K))
        torch.cuda.synchronize()
        _no_device_error(h)
        ref, pre = oracle.epilogue(ex, bias_b if use_bias else None, act, res_b if use_res else None)
        tol = oracle.tolerance_fused(ref, mag, pre, res_b if use_res else None)
        ok, rep = oracle.compare_with_tolerance(bits(C), ref, tol)
        assert ok, (path, act, use_bias, use_res, rep)
    plan = _with_schedule(h, sched, lambda: h.describe(fmt, M, N, K))
    if sched is not None:
        assert "sched=" + {mxgemm.SCHED_SPLITK: "splitk", mxgemm.SCHED_STREAMK: "streamk",
                           mxgemm.SCHED_KSPLIT: "ksplit", mxgemm.SCHED_DP: "dp"}[sched[0]] in plan, plan


def test_fused_epilogue_residual_in_place():
    """The residual may be C itself: each element is read before it is written."""
    fmt, M, N, K = F8, 200, 256, 512
    (oa, osa, ob, osb), (qa, sa, qb, sb) = _mx_operands(fmt, M, N, K, seed=5)
    res_b, res_t = _bf16(np.random.default_rng(1).standard_normal((M, N)))
    h = handle()
    C = res_t.clone()
    h.run_fused(fmt, qa, sa, qb, sb, act=mxgemm.ACT_RELU, residual=C, C=C, K=K)
    torch.cuda.synchronize()
    _, ex, mag = oracle.gemm(fmt, K, oa, osa, ob, osb, want_exact=True)
    ref, pre = oracle.epilogue(ex, None, mxgemm.ACT_RELU, res_b)
    ok, rep = oracle.compare_with_tolerance(bits(C), ref, oracle.tolerance_fused(ref, mag, pre, res_b))
    assert ok, rep


# ------------------------------------------------------ quantised output

def _integer_operands(fmt, M, N, K, seed):
    rng = np.random.default_rng(seed)
    vals = np.arange(-8, 9) if fmt == F8 else np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    ai = rng.choice(vals, (M, K))
    bi = rng.choice(vals, (N, K))
    enc = oracle.encode_e4m3 if fmt == F8 else oracle.encode_e2m1
    table = {int(v): enc(float(v)) for v in vals}
    ea = np.vectorize(table.get)(ai).astype(np.uint8)
    eb = np.vectorize(table.get)(bi).astype(np.uint8)
    if fmt == F4:
        ea = (ea[:, 0::2] | (ea[:, 1::2] << 4)).astype(np.uint8)
        eb = (eb[:, 0::2] | (eb[:, 1::2] << 4)).astype(np.uint8)
    # per-block scales 2^-1 .. 2^2: every product is a multiple of 2^-2 and
    # every partial sum stays below 2^21 in magnitude (K <= 2048, |a b| <= 64
    # * 2^4), so all sums are exact in FP32 whatever their order
    sa = rng.integers(126, 130, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(126, 130, (N, K // 32)).astype(np.uint8)
    host = (ea, sa, eb, sb)
    return host, [torch.from_numpy(x).cuda() for x in host]


QPATHS = {
    "swap": ((32, 512, 1024), None),
    "swap16": ((9, 256, 512), None),
    "plain": ((200, 384, 768), None),
    "splitk3": ((100, 640, 2048), (mxgemm.SCHED_SPLITK, 3, 0)),
    "swap-streamk": ((40, 512, 2048), (mxgemm.SCHED_STREAMK, 1, 37)),
    "swap-ksplit2": ((32, 512, 2048), (mxgemm.SCHED_KSPLIT, 2, 0)),
    "swap-multitile": ((24, 128 * 200, 256), None),
}


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("out_fmt", [F8, F4], ids=["to-mxfp8", "to-mxfp4"])
@pytest.mark.parametrize("path", list(QPATHS))
def test_quantised_output_integer_exact(fmt, out_fmt, path):
    """Integer-exact products: the GPU's BF16 result equals the oracle's
    everywhere, so codes and scales must equal the oracle quantiser's output
    on the oracle's C bit for bit."""
    (M, N, K), sched = QPATHS[path]
    (ea, sa, eb, sb), (ta, tsa, tb, tsb) = _integer_operands(fmt, M, N, K, seed=M + out_fmt)
    h = handle()
    Cq, Cs = _with_schedule(h, sched, lambda: h.run_quantized(fmt, ta, tsa, tb, tsb, out_fmt, K=K))
    torch.cuda.synchronize()
    _no_device_error(h)
    ref, _, _ = oracle.gemm(fmt, K, ea, sa, eb, sb)
    oq, os_ = oracle.quantize_bf16(out_fmt, ref)
    assert np.array_equal(Cs.cpu().numpy(), os_)
    assert np.array_equal(Cq.cpu().numpy(), oq)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("out_fmt", [F8, F4], ids=["to-mxfp8", "to-mxfp4"])
@pytest.mark.parametrize("path", ["swap", "plain", "splitk3", "swap-ksplit2"])
@pytest.mark.parametrize("act", [mxgemm.ACT_NONE, mxgemm.ACT_GELU], ids=["none", "gelu"])
def test_quantised_output_normal_inputs(fmt, out_fmt, path, act):
    """Normal inputs (with bias and GELU on one variant): wherever the GPU's
    BF16 result of a 32-run equals the oracle's, that run's codes and scale
    equal the oracle quantiser's bit for bit.  A run whose BF16 values differ
    from the oracle's (within the parity tolerance: a value near a BF16
    rounding boundary) may quantise differently; there the scale may differ
    by one binade and the decoded values by at most a quarter of their
    magnitude plus the block's smallest grid step."""
    (M, N, K), sched = QPATHS[path]
    (oa, osa, ob, osb), (qa, sa, qb, sb) = _mx_operands(fmt, M, N, K, seed=77 + M)
    bias_b, bias_t = _bf16(np.random.default_rng(4).standard_normal(N))
    kw = dict(bias=bias_t, act=act) if act else {}
    h = handle()
    Cq, Cs = _with_schedule(h, sched, lambda: h.run_quantized(fmt, qa, sa, qb, sb, out_fmt, K=K, **kw))
    Cb = _with_schedule(h, sched, lambda: h.run_fused(fmt, qa, sa, qb, sb, K=K, **kw))
    torch.cuda.synchronize()
    _no_device_error(h)
    _, ex, mag = oracle.gemm(fmt, K, oa, osa, ob, osb, want_exact=True)
    ref, pre = oracle.epilogue(ex, bias_b if act else None, act, None)
    ok, rep = oracle.compare_with_tolerance(bits(Cb), ref, oracle.tolerance_fused(ref, mag, pre))
    assert ok, rep
    oq, os_ = oracle.quantize_bf16(out_fmt, ref)
    same = (bits(Cb) == ref).reshape(M, N // 32, 32).all(axis=2)          # runs whose BF16 inputs agree
    assert same.mean() >= 0.5, same.mean()
    gq, gs = Cq.cpu().numpy(), Cs.cpu().numpy()
    assert np.array_equal(gs[same], os_[same])
    per = 32 if out_fmt == F8 else 16
    assert np.array_equal(gq.reshape(M, N // 32, per)[same], oq.reshape(M, N // 32, per)[same])
    # the other runs: a valid quantisation of nearly the same values
    diff = ~same
    assert (np.abs(gs[diff].astype(int) - os_[diff].astype(int)) <= 1).all()
    dg, do = _decode_mx(out_fmt, gq, gs), _decode_mx(out_fmt, oq, os_)
    grid = np.exp2(np.minimum(gs, os_).astype(np.float64) - 127 - (9 if out_fmt == F8 else 1))
    bound = 0.25 * np.maximum(np.abs(dg), np.abs(do)) + np.repeat(grid, 32, axis=1)
    assert (np.abs(dg - do) <= bound).all()


def _decode_mx(fmt, codes, scales):
    """MX codes + E8M0 scales [M][N/32] -> FP64 values [M][N] (oracle decoders)."""
    M = codes.shape[0]
    if fmt == F8:
        dec = np.array([oracle.decode_e4m3(c) for c in range(256)])
        v = dec[codes]
    else:
        dec = np.array([oracle.decode_e2m1(c) for c in range(16)])
        v = np.stack([dec[codes & 0xF], dec[codes >> 4]], axis=2).reshape(M, -1)
    sc = np.array([oracle.decode_e8m0(b) for b in range(256)])[scales]
    return v * np.repeat(sc, 32, axis=1)


def test_quantised_output_rejects_bad_n():
    h = handle()
    t = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    p = t.data_ptr()
    st = mxgemm.mxgemm_run_quantized(h.h, F8, 32, 48, 128, p, p, p, p, 0, 0, 0, F8, p, p, 0)
    assert st == mxgemm.ERR_INVALID_ARG                 # N % 32 != 0
    st = mxgemm.mxgemm_run_quantized(h.h, F8, 32, 64, 128, p, p, p, p, 0, 0, 0, 2, p, p, 0)
    assert st == mxgemm.ERR_INVALID_ARG                 # output format not MX
    st = mxgemm.mxgemm_run_fused(h.h, F8, 32, 64, 128, p, p, p, p, p + 2, 0, 0, p, 0)
    assert st == mxgemm.ERR_ALIGNMENT                   # bias not 16-byte aligned
    st = mxgemm.mxgemm_run_fused(h.h, F8, 32, 64, 128, p, p, p, p, 0, 7, 0, p, 0)
    assert st == mxgemm.ERR_INVALID_ARG                 # unknown activation


# ------------------------------------------------------------ BF16 GEMM

BF16_SHAPES = [(1, 8, 64), (16, 256, 128), (32, 512, 1024), (48, 200, 264), (64, 4104, 512), (65, 128, 64),
               (130, 1000, 1152), (300, 384, 776), (512, 2048, 256)]


@pytest.mark.parametrize("M,N,K", BF16_SHAPES)
def test_bf16_gemm_full(M, N, K):
    rng = np.random.default_rng(M * 3 + N + K)
    ab, at = _bf16(rng.standard_normal((M, K)))
    bb, bt = _bf16(rng.standard_normal((N, K)))
    h = handle()
    C = h.run_bf16(at, bt)
    torch.cuda.synchronize()
    _no_device_error(h)
    ref, _, mag = oracle.gemm_bf16(ab, bb)
    assert_parity(bits(C), ref, mag, "bf16 %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("sched", [(mxgemm.SCHED_SPLITK, 3, 0), (mxgemm.SCHED_STREAMK, 1, 148),
                                   (mxgemm.SCHED_STREAMK, 1, 37), (mxgemm.SCHED_KSPLIT, 4, 0)],
                         ids=["splitk3", "streamk148", "streamk37", "ksplit4"])
@pytest.mark.parametrize("M,N,K", [(40, 1024, 2048), (200, 640, 1536)])
def test_bf16_gemm_forced_schedules(sched, M, N, K):
    rng = np.random.default_rng(7)
    ab, at = _bf16(rng.standard_normal((M, K)))
    bb, bt = _bf16(rng.standard_normal((N, K)))
    h = handle()
    C = _with_schedule(h, sched, lambda: h.run_bf16(at, bt))
    torch.cuda.synchronize()
    _no_device_error(h)
    ref, _, mag = oracle.gemm_bf16(ab, bb)
    assert_parity(bits(C), ref, mag, "bf16 forced %s" % (sched,))
    # the handle describes the BF16 plan under its schedule
    plan = _with_schedule(h, sched, lambda: h.describe(mxgemm.FMT_BF16, M, N, K))
    want = {mxgemm.SCHED_SPLITK: "splitk", mxgemm.SCHED_STREAMK: "streamk", mxgemm.SCHED_KSPLIT: "ksplit"}[sched[0]]
    if not (want == "ksplit" and M > 64):        # the cluster split takes decode tiles only
        assert "fmt=2" in plan and "sched=" + want in plan, plan


def test_bf16_gemm_integer_exact_and_specials():
    rng = np.random.default_rng(8)
    M, N, K = 96, 136, 512
    ai = rng.integers(-16, 17, (M, K)).astype(np.float32)
    bi = rng.integers(-16, 17, (N, K)).astype(np.float32)
    ai[3, 10] = np.nan
    bi[5, 100] = np.inf
    ab, at = _bf16(ai)
    bb, bt = _bf16(bi)
    h = handle()
    C = h.run_bf16(at, bt)
    torch.cuda.synchronize()
    ref, _, mag = oracle.gemm_bf16(ab, bb)
    assert_parity(bits(C), ref, mag, "bf16 integer")
    fin = np.isfinite(oracle.bf16_bits_to_f64(ref))
    assert np.array_equal(bits(C)[fin], ref[fin])


def test_bf16_gemm_64x4096x4096_sampled():
    """The pages' called-out BF16 shape, in the launch configuration the
    benchmark times; every row of C against the oracle on 1024 columns."""
    M, N, K = 64, 4096, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(N, K, generator=g, device="cuda").to(torch.bfloat16)
    h = handle()
    C = h.run_bf16(A, B)
    torch.cuda.synchronize()
    _no_device_error(h)
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(3).integers(0, N, 1022)]))
    ab = A.view(torch.int16).cpu().numpy().view(np.uint16)
    bb = B.view(torch.int16).cpu().numpy().view(np.uint16)[cols]
    ref, _, mag = oracle.gemm_bf16(ab, bb)
    assert_parity(bits(C)[:, cols], ref, mag, "bf16 64x4096x4096")


def test_bf16_rejects_bad_args():
    h = handle()
    t = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    p = t.data_ptr()
    assert mxgemm.mxgemm_run_bf16(h.h, 4, 4, 12, p, p, p, 0) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_run_bf16(h.h, 4, 4, 16, p + 2, p, p, 0) == mxgemm.ERR_ALIGNMENT
    assert mxgemm.mxgemm_run_bf16(None, 4, 4, 16, p, p, p, 0) == mxgemm.ERR_INVALID_ARG


# ------------------------------------------------------------ grouped GEMM

GROUPINGS = {
    "uneven-empty": [0, 37, 300, 0, 1, 128, 0, 259],
    "one-group": [700],
    "empty-ends": [0, 0, 250, 130, 0],
    "tiny": [1, 2, 3, 4, 5, 6, 7, 8],
}


@pytest.mark.parametrize("fmt", [F8, F4, BF], ids=["mxfp8", "mxfp4", "bf16"])
@pytest.mark.parametrize("grouping", list(GROUPINGS))
@pytest.mark.parametrize("N", [256, 200])
def test_grouped_gemm(fmt, grouping, N):
    sizes = GROUPINGS[grouping]
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    M = int(off[-1])
    K = 512
    rng = np.random.default_rng(G * 7 + N + fmt)
    if fmt == BF:
        ab, at = _bf16(rng.standard_normal((M, K)))
        bb, bt = _bf16(rng.standard_normal((G * N, K)))
        bb = bb.reshape(G, N, K)
        sa = sb = osa = osb = None
        oa, ob = ab, bb
    else:
        A32 = rng.standard_normal((M, K)).astype(np.float32)
        B32 = rng.standard_normal((G * N, K)).astype(np.float32)
        oa, osa = oracle.quantize(fmt, A32)
        ob, osb = oracle.quantize(fmt, B32)
        at, sa = torch.from_numpy(oa).cuda(), torch.from_numpy(osa).cuda()
        bt, sb = torch.from_numpy(ob).cuda(), torch.from_numpy(osb).cuda()
        ob = ob.reshape(G, N, -1)
        osb = osb.reshape(G, N, -1)
    h = handle()
    offs = torch.from_numpy(off).cuda()
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    Bv = bt.view(G, N, -1)
    h.run_grouped(fmt, offs, at, sa, Bv, sb, C=C, K=K)
    torch.cuda.synchronize()
    _no_device_error(h)
    ref, mag = oracle.gemm_grouped(fmt, K, off, oa, osa, ob, osb)
    assert_parity(bits(C), ref, mag, "grouped %s N=%d" % (grouping, N))


def test_grouped_plan_and_bad_args():
    plan = mxgemm.mxgemm_describe_grouped_plan(148, F8, 8, 4096, 4096, 4096)
    assert "groups=8" in plan and "pair=0" in plan and "scales=fused" in plan, plan
    h = handle()
    t = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    p = t.data_ptr()
    assert mxgemm.mxgemm_run_grouped(h.h, F8, 0, 10, 64, 128, p, p, p, p, p, p, 0) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_run_grouped(h.h, F8, 2, 10, 64, 100, p, p, p, p, p, p, 0) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_run_grouped(h.h, F8, 2, 10, 64, 128, p + 8, p, p, p, p, p, 0) == mxgemm.ERR_ALIGNMENT
    # no rows at all: nothing to launch
    assert mxgemm.mxgemm_run_grouped(h.h, F8, 2, 0, 64, 128, p, p, p, p, p, p, 0) == mxgemm.OK
