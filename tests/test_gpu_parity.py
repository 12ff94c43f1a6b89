"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Pass rule per element: |C_gpu - C_ref| <= 1 BF16 ulp(C_ref) + 2^-18 * sum_k |a_k b_k|
with identical NaN / +-Inf positions; quantised codes and scales must agree
bit for bit.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from microscaling_block_scaled_b200 import mxgemm, synth

from gpu_util import (assert_parity, bits, full_case, gpu_quantize, handle, rows_case, rows_cols_points_case,
                      sampled_case)

pytestmark = pytest.mark.gpu

F8, F4 = mxgemm.FMT_MXFP8, mxgemm.FMT_MXFP4


# ------------------------------------------------------------- quantiser

@pytest.mark.parametrize("fmt", [F8, F4])
@pytest.mark.parametrize("kind", ["normal", "heavy"])
def test_quantiser_bit_exact(fmt, kind):
    A32, _ = synth.operands(96, 1, 2048, seed=21, kind=kind)
    q, s = mxgemm.quantize(fmt, A32.cuda())
    oq, os_ = oracle.quantize(fmt, A32.numpy())
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("bf16_input", [False, True], ids=["fp32", "bf16"])
@pytest.mark.parametrize("R,K", [(1, 32), (3, 96), (5, 160), (7, 4128), (33, 2080)])
def test_quantiser_ragged_sizes_bit_exact(fmt, bf16_input, R, K):
    """The quantiser covers the input in warp tiles of 32 lanes x 32 bytes,
    four tiles per warp and pass.  Sizes that end inside a tile or inside a
    warp's group of four match the oracle bit for bit, with FP32 and BF16
    input, and leave the bytes past the codes and scales untouched."""
    X32, _ = synth.operands(R, 1, K, seed=R + K, kind="heavy")
    qw = K if fmt == F8 else K // 2
    Qp = torch.full((R * qw + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    Sp = torch.full((R * (K // 32) + 64,), 0x5A, dtype=torch.uint8, device="cuda")
    out = (Qp[:R * qw].view(R, qw), Sp[:R * (K // 32)].view(R, K // 32))
    if bf16_input:
        xb = np.ascontiguousarray(X32.numpy().astype(ml_dtypes.bfloat16).view(np.uint16))
        mxgemm.quantize_bf16(fmt, torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16), out=out)
        oq, os_ = oracle.quantize_bf16(fmt, xb)
    else:
        mxgemm.quantize(fmt, X32.cuda().contiguous(), out=out)
        oq, os_ = oracle.quantize(fmt, X32.numpy())
    torch.cuda.synchronize()
    assert np.array_equal(out[1].cpu().numpy(), os_)
    assert np.array_equal(out[0].cpu().numpy(), oq)
    assert bool((Qp[R * qw:] == 0xA5).all()) and bool((Sp[R * (K // 32):] == 0x5A).all())


@pytest.mark.parametrize("fmt", [F8, F4])
def test_quantiser_edge_blocks_bit_exact(fmt):
    emax = 8 if fmt == F8 else 2
    rows = []
    r = np.zeros(32 * 12, dtype=np.float32)
    r[32:64] = -0.0                                  # negative zeros
    r[64] = np.float32(2.0 ** -140)                  # FP32 subnormal amax
    r[65] = -np.float32(2.0 ** -145)
    r[96:128] = np.nan                               # NaN block
    r[128] = np.inf                                  # Inf block
    r[160] = 1000.0                                  # saturation
    r[161] = -930.0
    # ties in the scaled domain (scale 2^0 when amax is in [2^emax, 2^(emax+1)))
    r[192] = 2.0 ** emax
    if fmt == F8:
        r[193:200] = [1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 15.5 * 2.0 ** -7, -1.0625, 460.0 / 2]
    else:
        r[193:200] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, -5.0]
    r[224] = np.float32(3.0e38)                      # near FP32 max
    r[225] = np.float32(-1.0e-38)
    r[256] = np.float32(2.0 ** -126) * 1.5           # smallest normal binade amax
    r[288:320] = np.linspace(-7.0, 7.0, 32, dtype=np.float32)
    r[320:352] = np.float32(2.0 ** -149)             # smallest subnormal
    rows.append(r)
    X = np.stack(rows + [np.random.default_rng(3).standard_normal(r.shape).astype(np.float32)])
    q, s = mxgemm.quantize(fmt, torch.from_numpy(X).cuda())
    oq, os_ = oracle.quantize(fmt, X)
    assert np.array_equal(s.cpu().numpy(), os_), (s.cpu().numpy(), os_)
    assert np.array_equal(q.cpu().numpy(), oq), np.argwhere(q.cpu().numpy() != oq)[:8]


# ------------------------------------------------------ full comparisons

SMALL = [
    (1, 8, 128), (16, 256, 128), (32, 256, 512), (33, 100, 384), (48, 200, 256), (64, 136, 256),
    (65, 128, 128), (100, 300, 256), (128, 128, 512), (200, 264, 640), (256, 512, 256), (130, 1000, 1152),
]


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_gemm_small_full(fmt, M, N, K):
    full_case(fmt, M, N, K, seed=M * 7 + N + K)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("M,N,K", [(32, 512, 1024), (300, 384, 768)])
def test_gemm_heavy_tails_full(fmt, M, N, K):
    full_case(fmt, M, N, K, seed=4, kind="heavy")


def test_config_mxfp8_32x256x512_full():
    full_case(F8, 32, 256, 512, seed=0)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("sched", [
    (mxgemm.SCHED_DP, 1, 0), (mxgemm.SCHED_SPLITK, 3, 0), (mxgemm.SCHED_SPLITK, 8, 0),
    (mxgemm.SCHED_STREAMK, 1, 0), (mxgemm.SCHED_STREAMK, 1, 7), (mxgemm.SCHED_STREAMK, 1, 37),
    (mxgemm.SCHED_KSPLIT, 2, 0), (mxgemm.SCHED_KSPLIT, 3, 0), (mxgemm.SCHED_KSPLIT, 4, 0),
])
@pytest.mark.parametrize("M,N,K", [(64, 1024, 2048), (200, 640, 1536)])
def test_gemm_forced_schedules(fmt, sched, M, N, K):
    full_case(fmt, M, N, K, seed=9, schedule=sched)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("M,N,K", [
    (1, 4096, 4096), (9, 640, 4096), (33, 300, 4096), (64, 4104, 4096), (48, 1000, 8192),
    (16, 128 * 60, 4096), (64, 4096, 4096), (17, 256, 4608), (17, 256, 4224),
])
def test_gemm_cluster_k_split(fmt, M, N, K):
    """Decode tiles that fill at most half the GPU split each tile's K range
    over a cluster of CTAs; the other ranks write their FP32 partial tiles
    into rank 0's drained ring through distributed shared memory and rank 0
    adds them.  Ragged N, K tails (K = 4224: 33 MXFP8 chunks, two per stage; 16.5 MXFP4
    chunks per row) and one tile column of 1 to 64 rows."""
    h = handle()
    plan = h.describe(fmt, M, N, K)
    field = dict(f.split("=") for f in plan.split())
    kt, tiles = int(field["kt"]), int(field["tiles"])
    want = 4 if kt >= 16 and 4 * tiles <= 148 else 2
    assert field["sched"] == "ksplit" and int(field["ksplit"]) == want, plan
    full_case(fmt, M, N, K, seed=M * 3 + K)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("kc", [1, 2, 4])
@pytest.mark.parametrize("M,N,K", [(32, 512, 1024), (200, 384, 640), (64, 256, 384), (130, 256, 896),
                                   (16, 640, 2560)])
def test_gemm_k_chunks_per_stage(fmt, kc, M, N, K):
    """One, two and four 128-byte K chunks per pipeline stage (2-D and 3-D
    TMA boxes), including K whose last stage is partly past the end of a
    row; four chunks apply to tiles of at most 64 columns."""
    h = handle()
    h.set_kchunks(kc)
    try:
        full_case(fmt, M, N, K, seed=kc * 100 + K)
    finally:
        h.set_kchunks(0)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("M,N,K", [(1024, 5120, 1024), (1000, 5000, 2048), (2048, 4864, 1024)])
def test_gemm_cta_pair_last_wave_split(fmt, M, N, K):
    """CTA-pair plans whose last wave of whole tiles would leave pairs idle
    split that wave's tiles into K ranges (under the MXGEMM_TAIL knob); the
    FP32 partials are summed by the range that finishes last."""
    _, plan = rows_case(fmt, M, N, K, seed=M + K)
    assert "pair=1" in plan and "sched=dptail" in plan, plan
    # the same shape again: the tile counters were left at zero
    _, plan = rows_case(fmt, M, N, K, seed=M + K + 1, n_rows=16)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("kc", [0, 1, 2])
@pytest.mark.parametrize("M,N,K", [(512, 8192, 256), (640, 8448, 384), (1000, 4104, 512)])
def test_gemm_cta_pair_tiles(fmt, kc, M, N, K):
    """Large-M shapes take 256x256 tiles on CTA pairs (cta_group::2); ragged
    M and N, K tails, and one or two K chunks per stage."""
    h = handle()
    h.set_kchunks(kc)
    try:
        _, plan = rows_case(fmt, M, N, K, seed=M + kc)
    finally:
        h.set_kchunks(0)
    assert "pair=1" in plan, plan


# ----------------------------------------------------------- edge cases
#
# Every edge case runs through every execution path of the GEMM: the small
# shape under the automatic plan (one-CTA whole tiles, swapped when M <= 64),
# a shape that takes the CTA pair (cta_group::2, 256x256 tiles), forced
# split-K and stream-K schedules on one-CTA tiles, where the output is the
# FP32 sum of per-worker partials (last-arriver fixup), and decode tiles as
# whole tiles and with their K range split over a cluster (partials summed in
# distributed shared memory).  NaN and +-Inf patterns must come out identical
# on every path.

PATHS = {
    # name: (shape override or None, schedule or None)
    "auto": (None, None),
    "pair": ((512, 8192, 384), None),
    "pair-tail": ((1024, 5120, 1024), None),      # 80 pair tiles: the last wave's 6 tiles split in K
    "splitk3": ((200, 640, 2048), (mxgemm.SCHED_SPLITK, 3, 0)),
    "splitk8": ((200, 640, 2048), (mxgemm.SCHED_SPLITK, 8, 0)),
    "streamk148": ((200, 640, 2048), (mxgemm.SCHED_STREAMK, 1, 148)),
    "streamk37": ((200, 640, 2048), (mxgemm.SCHED_STREAMK, 1, 37)),
    "swap-splitk3": ((40, 1024, 2048), (mxgemm.SCHED_SPLITK, 3, 0)),
    "swap-streamk148": ((40, 1024, 2048), (mxgemm.SCHED_STREAMK, 1, 148)),
    "swap-dp": ((40, 1024, 2048), (mxgemm.SCHED_DP, 1, 0)),
    "ksplit2": ((40, 1024, 2048), (mxgemm.SCHED_KSPLIT, 2, 0)),
    "ksplit4": ((40, 1024, 2048), (mxgemm.SCHED_KSPLIT, 4, 0)),
}


def _shape(path, default):
    return PATHS[path][0] or default


@pytest.fixture(autouse=True)
def _last_wave_split_knob(request, monkeypatch):
    # the last-wave split of CTA-pair plans is a measurement knob: on for the
    # cases that exercise it, unset for all others
    if "tail" in request.node.name or "last_wave" in request.node.name:
        monkeypatch.setenv("MXGEMM_TAIL", "1")
    else:
        monkeypatch.delenv("MXGEMM_TAIL", raising=False)


def _codes_case(fmt, A, SA, B, SB, K, path="auto"):
    h = handle()
    ta = torch.from_numpy(A).cuda()
    tb = torch.from_numpy(B).cuda()
    tsa = torch.from_numpy(SA).cuda()
    tsb = torch.from_numpy(SB).cuda()
    M, N = A.shape[0], B.shape[0]
    sched = PATHS[path][1]
    if sched is not None:
        h.set_schedule(*sched)
    try:
        plan = h.describe(fmt, M, N, K)
        C = h.run(fmt, ta, tsa, tb, tsb, K=K)
        torch.cuda.synchronize()
    finally:
        if sched is not None:
            h.set_schedule(mxgemm.SCHED_AUTO)
    st, code = h.check_device_error()
    assert st == mxgemm.OK and code == 0, ("device error word", code)
    # the path the case is meant to exercise is the one that ran
    if path == "pair":
        assert "pair=1" in plan, plan
    elif path == "pair-tail":
        assert "pair=1" in plan and "sched=dptail" in plan, plan
    elif path.startswith("split") or path.startswith("swap-split"):
        assert "sched=splitk" in plan and "pair=0" in plan, plan
    elif "streamk" in path:
        assert "sched=streamk" in plan and "pair=0" in plan, plan
    elif path.startswith("ksplit"):
        assert "sched=ksplit" in plan and "ksplit=" + path[-1] in plan and "swap=1" in plan, plan
    elif path == "swap-dp":
        assert "sched=dp" in plan, plan
    if path.startswith("swap"):
        assert "swap=1" in plan, plan
    ref, _, mag = oracle.gemm(fmt, K, A, SA, B, SB)
    return bits(C), ref, mag


def _random_codes(rng, fmt, rows, K):
    rb = oracle.row_bytes(fmt, K)
    X = rng.integers(0, 256, (rows, rb), dtype=np.uint8)
    if fmt == F8:
        X[(X & 0x7F) == 0x7F] = 0x35       # no NaN codes here
    return X


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("path", list(PATHS))
def test_gemm_nan_scales_and_zero_blocks(fmt, path):
    rng = np.random.default_rng(17)
    M, N, K = _shape(path, (70, 160, 384))
    A = _random_codes(rng, fmt, M, K)
    B = _random_codes(rng, fmt, N, K)
    SA = rng.integers(110, 140, (M, K // 32), dtype=np.uint8)
    SB = rng.integers(110, 140, (N, K // 32), dtype=np.uint8)
    nan_rows = sorted({3, M - 2})
    nan_cols = sorted({7, N - 3})
    SA[3, 5] = 0xFF                        # NaN scale in A: row 3 all NaN
    SA[M - 2, K // 32 - 1] = 0xFF          # ... and a row in the last tile, last K block
    SB[7, 0] = 0xFF                        # NaN scale in B: column 7 all NaN
    SB[N - 3, K // 64] = 0xFF              # ... and a column in the last tile, mid K
    blk = 32 * oracle.row_bytes(fmt, K) // K
    A[10, 2 * blk:3 * blk] = 0             # an all-zero block
    B[20, :] = 0                           # an all-zero column
    got, ref, mag = _codes_case(fmt, A, SA, B, SB, K, path)
    assert_parity(got, ref, mag, "nan scales (%s)" % path)
    gv = oracle.bf16_bits_to_f64(got)
    for r in nan_rows:
        assert np.isnan(gv[r]).all()
    for c in nan_cols:
        assert np.isnan(gv[:, c]).all()
    keep = np.ones(M, bool)
    keep[nan_rows] = False
    assert (gv[keep, 20] == 0).all()
    assert np.isfinite(gv[np.ix_(keep, [0, 1, 2, 20])]).all()


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("path", list(PATHS))
def test_gemm_overflow_and_underflow_scales(fmt, path):
    """Positive elements (no cancellation) with extreme scales: 2^127 * 2^127
    overflows BF16 to +Inf, 2^-95 * 2^-95 underflows to 0, mixed pairs give
    normal results.  With positive elements every partial sum of a split
    schedule overflows exactly when the total does."""
    rng = np.random.default_rng(23)
    M, N, K = _shape(path, (130, 140, 256))
    if fmt == F8:
        A = rng.integers(0x08, 0x7F, (M, K), dtype=np.uint8)
        B = rng.integers(0x08, 0x7F, (N, K), dtype=np.uint8)
    else:
        na = rng.integers(1, 8, (M, K), dtype=np.uint8)
        nb = rng.integers(1, 8, (N, K), dtype=np.uint8)
        A = (na[:, 0::2] | (na[:, 1::2] << 4)).astype(np.uint8)
        B = (nb[:, 0::2] | (nb[:, 1::2] << 4)).astype(np.uint8)
    SA = np.full((M, K // 32), 0x7F, np.uint8)
    SB = np.full((N, K // 32), 0x7F, np.uint8)
    SA[5, :] = 0xFE
    SA[6, :] = 0x20
    SB[9, :] = 0xFE
    SB[10, :] = 0x20
    SA[M - 1, :] = 0xFE                    # a row of the last tile (the pair's odd CTA)
    SB[N - 1, :] = 0xFE                    # a column of the last tile
    got, ref, mag = _codes_case(fmt, A, SA, B, SB, K, path)
    assert_parity(got, ref, mag, "extreme scales (%s)" % path)
    gv = oracle.bf16_bits_to_f64(got)
    assert np.isposinf(gv[5, 9]) and np.isposinf(gv[5, 0]) and gv[6, 10] == 0.0
    assert np.isfinite(gv[5, 10]) and gv[5, 10] > 0
    assert np.isposinf(gv[M - 1, N - 1]) and np.isposinf(gv[M - 1, 0]) and np.isposinf(gv[0, N - 1])


@pytest.mark.parametrize("path", list(PATHS))
def test_gemm_nan_elements_e4m3(path):
    rng = np.random.default_rng(5)
    M, N, K = _shape(path, (40, 72, 256))
    A = rng.integers(0, 0x70, (M, K), dtype=np.uint8)
    B = rng.integers(0, 0x70, (N, K), dtype=np.uint8)
    A[5, 17] = 0x7F                        # E4M3 NaN element
    B[9, K - 56] = 0xFF
    A[M - 1, K // 2] = 0xFF                # last row, middle of K
    SA = np.full((M, K // 32), 0x7F, np.uint8)
    SB = np.full((N, K // 32), 0x7F, np.uint8)
    got, ref, mag = _codes_case(F8, A, SA, B, SB, K, path)
    assert_parity(got, ref, mag, "nan elements (%s)" % path)
    gv = oracle.bf16_bits_to_f64(got)
    assert np.isnan(gv[5]).all() and np.isnan(gv[:, 9]).all() and np.isnan(gv[M - 1]).all()


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("path", list(PATHS))
def test_gemm_integer_exact(fmt, path):
    """All scales 1 and small integer elements: every output is an exact
    integer (a textbook integer matmul) and must match exactly, whatever the
    order in which the FP32 partial sums are added."""
    rng = np.random.default_rng(8)
    M, N, K = _shape(path, (96, 200, 512))
    vals = np.arange(-16, 17) if fmt == F8 else np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    ai = rng.choice(vals, (M, K))
    bi = rng.choice(vals, (N, K))
    enc = oracle.encode_e4m3 if fmt == F8 else oracle.encode_e2m1
    table = {int(v): enc(float(v)) for v in vals}
    ea = np.vectorize(table.get)(ai).astype(np.uint8)
    eb = np.vectorize(table.get)(bi).astype(np.uint8)
    if fmt == F4:
        ea = (ea[:, 0::2] | (ea[:, 1::2] << 4)).astype(np.uint8)
        eb = (eb[:, 0::2] | (eb[:, 1::2] << 4)).astype(np.uint8)
    S1 = np.full((M, K // 32), 0x7F, np.uint8)
    S2 = np.full((N, K // 32), 0x7F, np.uint8)
    got, ref, mag = _codes_case(fmt, ea, S1, eb, S2, K, path)
    exact = ai.astype(np.int64) @ bi.astype(np.int64).T
    small = np.abs(exact) <= 256           # exactly representable in BF16
    assert np.array_equal(oracle.bf16_bits_to_f64(got)[small], exact[small].astype(np.float64))
    assert np.array_equal(got, ref)        # exact FP32 sums: the one BF16 rounding is the oracle's


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("path", list(PATHS))
def test_gemm_fp32_subnormal_results(fmt, path):
    """Results, partial sums and single products in the FP32-subnormal range
    (below 2^-126): the tensor pipe's FP32 accumulation keeps them (no flush
    to zero), so they match the oracle exactly and fall under the ordinary
    pass rule."""
    M, N, K = _shape(path, (64, 256, 256))
    enc = oracle.encode_e4m3 if fmt == F8 else oracle.encode_e2m1
    one, neg1 = enc(1.0), enc(-1.0)
    big = enc(1.125) if fmt == F8 else enc(1.5)
    tiny = 0x01                                     # smallest subnormal code: 2^-9 (E4M3), 0.5 (E2M1)
    A = np.zeros((M, K), np.uint8)
    B = np.zeros((N, K), np.uint8)
    SA = np.full((M, K // 32), 62, np.uint8)
    SB = np.full((N, K // 32), 62, np.uint8)
    B[:, 0] = one
    B[:, 32] = one
    B[:, 64] = tiny
    A[0, 0] = one                                   # one product of 2^-130
    A[1, 0], A[1, 32] = big, neg1                   # (1.125 - 1) 2^-125 or (1.5 - 1) 2^-126: a subnormal difference
    SA[1, :] = 67 if fmt == F8 else 66
    A[2, 64] = tiny                                 # smallest elements: 2^-18 * 2^-112 / 0.25 * 2^-130
    SA[2, :] = 80 if fmt == F8 else 62
    A[3, 0], A[3, K - 32] = one, one                # a subnormal part added to a normal one
    SA[3, K // 32 - 1] = 167
    B[:, K - 32] = one
    A[4, 0], A[4, 32], A[4, 64] = one, one, one     # subnormal products summed
    if fmt == F4:
        A = (A[:, 0::2] | (A[:, 1::2] << 4)).astype(np.uint8)
        B = (B[:, 0::2] | (B[:, 1::2] << 4)).astype(np.uint8)
    got, ref, mag = _codes_case(fmt, A, SA, B, SB, K, path)
    assert_parity(got, ref, mag, "subnormal results (%s)" % path)
    rv = oracle.bf16_bits_to_f64(ref)
    assert (np.abs(rv[[0, 1, 2, 4], 0]) < 2.0 ** -126).all() and (rv[[0, 1, 2, 4], 0] != 0).all()
    assert np.array_equal(got[:5], ref[:5])


# -------------------------------------------------------- entry points

@pytest.mark.parametrize("fmt,M,N,K", [(F4, 48, 512, 1024), (F4, 32, 512, 1024), (F8, 16, 384, 512)],
                         ids=["repack-plan", "fused-plan", "fused-plan-mxfp8"])
def test_repack_then_gemm_equals_run_and_host_path(fmt, M, N, K):
    """mxgemm_run (one launch with the scale conversion fused into the GEMM,
    or repack + GEMM, per the plan), mxgemm_repack + mxgemm_gemm and the
    host-buffer path give bit-identical C."""
    A32, B32 = synth.operands(M, N, K, seed=31)
    qa, sa = mxgemm.quantize(fmt, A32.cuda())
    qb, sb = mxgemm.quantize(fmt, B32.cuda())
    h = handle()
    C1 = h.run(fmt, qa, sa, qb, sb, K=K)
    C2 = torch.empty_like(C1)
    h.repack(fmt, M, N, K, sa, sb)
    h.gemm(fmt, M, N, K, qa, qb, C2)
    C3 = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    h.run_host(fmt, M, N, K, qa.cpu().pin_memory(), sa.cpu().pin_memory(), qb.cpu().pin_memory(),
               sb.cpu().pin_memory(), C3)
    torch.cuda.synchronize()
    assert torch.equal(C1.view(torch.int16), C2.view(torch.int16))
    assert torch.equal(C1.view(torch.int16).cpu(), C3.view(torch.int16))


@pytest.mark.parametrize("fmt,M,N,K,same_plans", [(F8, 4096, 4096, 1024, True), (F4, 3000, 6004, 1024, False)],
                         ids=["mxfp8-2x2-blocks", "mxfp4-ragged-blocks"])
def test_host_path_in_blocks(fmt, M, N, K, same_plans):
    """With 32 MB or more of copies, mxgemm_run_host uploads row bands of A
    and B, computes each block of C once its bands have landed and
    downloads it while later bands upload (three streams).  4096 x 4096 runs
    as 2 x 2 blocks of 2048 x 2048; 3000 x 6004 as 2 x 2 ragged blocks
    (1536 / 1464 rows by 3072 / 2932 columns).  Two calls with different
    inputs on one handle, so a GEMM that started before its bands landed
    would read the first call's operands: each call matches the oracle on
    whole rows and whole columns on both sides of every block boundary, and
    where each block runs the same kind of plan as the whole product (CTA
    pairs), mxgemm_run bit for bit."""
    h = handle()
    rows = sorted({0, 1, 1535, 1536, 2047, 2048, M - 2, M - 1})
    cols = sorted({0, 3, 2047, 2048, 3071, 3072, N - 2, N - 1})
    for seed in (61, 62):
        A32, B32 = synth.operands(M, N, K, seed=seed, kind="normal", device="cpu")
        qa, sa = gpu_quantize(fmt, A32)
        qb, sb = gpu_quantize(fmt, B32)
        oa, osa = oracle.quantize(fmt, A32.numpy())
        ob, osb = oracle.quantize(fmt, B32.numpy())
        assert np.array_equal(qa.cpu().numpy(), oa) and np.array_equal(sa.cpu().numpy(), osa)
        assert np.array_equal(qb.cpu().numpy(), ob) and np.array_equal(sb.cpu().numpy(), osb)
        C = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        C.fill_(float("nan"))
        h.run_host(fmt, M, N, K, qa.cpu().pin_memory(), sa.cpu().pin_memory(), qb.cpu().pin_memory(),
                   sb.cpu().pin_memory(), C)
        st, code = h.check_device_error()
        assert st == mxgemm.OK and code == 0, ("device error word", code)
        got = C.view(torch.int16).numpy().view(np.uint16)
        ref, _, mag = oracle.gemm(fmt, K, oa[rows], osa[rows], ob, osb)
        assert_parity(got[rows], ref, mag, "host path whole rows, seed %d" % seed)
        ref, _, mag = oracle.gemm(fmt, K, oa, osa, ob[cols], osb[cols])
        assert_parity(got[:, cols], ref, mag, "host path whole columns, seed %d" % seed)
        assert bool(torch.isfinite(C.float()).all())
        if same_plans:
            C1 = h.run(fmt, qa, sa, qb, sb, K=K)
            torch.cuda.synchronize()
            assert np.array_equal(bits(C1), got)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("sched", [
    (mxgemm.SCHED_SPLITK, 3, 0), (mxgemm.SCHED_STREAMK, 1, 0), (mxgemm.SCHED_STREAMK, 1, 37),
])
def test_fused_scales_with_split_schedules(fmt, sched):
    """The GEMM's own scale conversion under split-K and stream-K, where a
    CTA's work spans several tiles and K ranges."""
    M, N, K = 32, 1536, 2048
    h = handle()
    h.set_schedule(*sched)
    try:
        plan = h.describe(fmt, M, N, K)
    finally:
        h.set_schedule(mxgemm.SCHED_AUTO)
    assert "scales=fused" in plan, plan
    full_case(fmt, M, N, K, seed=77, schedule=sched)


def test_gemm_rejects_shape_not_repacked():
    h = handle()
    t = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    st = mxgemm.mxgemm_repack(h.h, F8, 4, 4, 128, t.data_ptr(), t.data_ptr(), 0)
    assert st == mxgemm.OK
    st = mxgemm.mxgemm_gemm(h.h, F8, 4, 8, 128, t.data_ptr(), t.data_ptr(), t.data_ptr(), 0)
    assert st == mxgemm.ERR_INVALID_ARG
    st = mxgemm.mxgemm_run(h.h, F8, 4, 4, 100, t.data_ptr(), t.data_ptr(), t.data_ptr(), t.data_ptr(),
                           t.data_ptr(), 0)
    assert st == mxgemm.ERR_INVALID_ARG
    st = mxgemm.mxgemm_run(h.h, F8, 4, 4, 128, t.data_ptr() + 8, t.data_ptr(), t.data_ptr(), t.data_ptr(),
                           t.data_ptr(), 0)
    assert st == mxgemm.ERR_ALIGNMENT


# ----------------------------------------------- the pages' workloads

@pytest.mark.parametrize("fmt,M,N,K,seed", [
    (F4, 32, 14336, 4096, 1),
    (F8, 64, 4096, 4096, 2),
    (F4, 64, 4096, 4096, 2),
])
def test_decode_workloads_sampled(fmt, M, N, K, seed):
    sampled_case(fmt, M, N, K, seed, n_rows=M, n_cols=1024)


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("M,N,K", [(2048, 28672, 8192), (8192, 8192, 8192), (4096, 4096, 14336)])
def test_prefill_workloads_rows_cols_points(fmt, M, N, K):
    """The prefill workloads at full size, in the launch configuration the
    benchmark times: 64 whole rows, 64 whole columns and 65 536 random
    elements of C against the oracle."""
    plan, nr, nc = rows_cols_points_case(fmt, M, N, K, seed=3)
    assert "pair=1" in plan, plan
    assert nr == 64 and nc == 64


@pytest.mark.parametrize("fmt", [F8, F4], ids=["mxfp8", "mxfp4"])
@pytest.mark.parametrize("M", list(synth.SWEEP_M))
def test_shape_sweep_heavy_tailed_sampled(fmt, M):
    """The shape sweep: M in {16 .. 8192} x the five (N, K) pairs, both
    formats, heavy-tailed inputs (N(0,1) * 2^U(-20, 20) per 32-block, exact
    zero blocks included) from seed 4.  Every run is checked on a sampled
    grid of rows x columns against the oracle, quantiser outputs bit for bit
    on the sampled rows."""
    for N, K in synth.SWEEP_NK:
        sampled_case(fmt, M, N, K, seed=synth.SWEEP_SEED, kind="heavy", n_rows=min(M, 48), n_cols=48,
                     rng_seed=M * 7 + N + K)
        torch.cuda.empty_cache()
