"""The host planner of the GEMM, on CPU: mxgemm_describe_plan_for needs no GPU.

The planner decides, from the shape and the SM count alone, the operand
swap for decode shapes, the output tile width, the K chunks per pipeline
stage, the ring depth, CTA pairs for large M, the schedule (whole tiles or
split K) and whether mxgemm_run converts the scales inside the GEMM.  These
tests pin those decisions and the invariants every plan must keep.
"""
import ctypes

import numpy as np
import pytest

from microscaling_block_scaled_b200 import build as mxbuild
from microscaling_block_scaled_b200 import mxgemm

F8, F4 = mxgemm.FMT_MXFP8, mxgemm.FMT_MXFP4
B200_SMS = 148


@pytest.fixture(scope="module", autouse=True)
def _library():
    mxbuild.build()
    mxgemm.load()


@pytest.fixture(autouse=True)
def _default_planner(monkeypatch):
    # the planner's measurement knobs stay unset
    monkeypatch.delenv("MXGEMM_BN", raising=False)
    monkeypatch.delenv("MXGEMM_PAIR", raising=False)
    monkeypatch.delenv("MXGEMM_BAND", raising=False)
    monkeypatch.delenv("MXGEMM_TAIL", raising=False)


def plan(fmt, M, N, K, sms=B200_SMS):
    text = mxgemm.mxgemm_describe_plan_for(sms, fmt, M, N, K)
    out = {}
    for field in text.split():
        k, v = field.split("=")
        out[k] = int(v) if v.lstrip("-").isdigit() else v
    return out


def cdiv(a, b):
    return -(-a // b)


def test_decode_shape_plan():
    p = plan(F4, 32, 14336, 4096)
    assert p == {"fmt": 1, "swap": 1, "pair": 0, "BN": 32, "kc": 2, "stages": 5, "tiles": 112, "kt": 8,
                 "workers": 112, "grid": 112, "sched": "dp", "partial_bytes": 0, "scales": "fused"}


@pytest.mark.parametrize("M,swap,bn", [(1, 1, 16), (16, 1, 16), (17, 1, 32), (32, 1, 32), (33, 1, 64),
                                       (64, 1, 64), (65, 0, 128), (200, 0, 128)])
def test_swap_and_tile_width_follow_M(M, swap, bn):
    p = plan(F8, M, 4096, 1024)
    assert (p["swap"], p["BN"]) == (swap, bn)


@pytest.mark.parametrize("M,N,pair", [
    (512, 8192, 1),     # 2 x 32 = 64 pair tiles: the smallest grid that fills the GPU
    (512, 8000, 1),     # ragged N, still 64 tiles
    (512, 7936, 0),     # 62 pair tiles
    (511, 8192, 0),     # M below 512
    (512, 8190, 0),     # N not a multiple of 8 (16-byte rows of C for the TMA store)
    (4096, 4096, 1),
    (64, 65536, 0),     # decode shapes never pair
])
def test_cta_pairs_for_large_M(M, N, pair):
    p = plan(F8, M, N, 1024)
    assert p["pair"] == pair
    if pair:
        assert p["BN"] == 256 and p["scales"] == "repack" and p["sched"] in ("dp", "dptail")
        assert p["band"] == min(8, cdiv(M, 256))      # tile order: bands of at most 8 tile rows
        assert p["tiles"] == cdiv(M, 256) * cdiv(N, 256)
        assert p["grid"] == 2 * min(p["tiles"], B200_SMS // 2)


@pytest.fixture
def _tail_knob(monkeypatch):
    monkeypatch.setenv("MXGEMM_TAIL", "1")


def test_pair_plans_keep_whole_tiles_by_default():
    p = plan(F8, 4096, 4096, 8192)
    assert p["sched"] == "dp" and p["workers"] == p["tiles"] and "tail_split" not in p


@pytest.mark.usefixtures("_tail_knob")
@pytest.mark.parametrize("M,N,full,split", [
    (4096, 4096, 222, 2),      # 256 tiles on 74 pairs: 3 whole waves, 34 tiles split in two
    (2048, 28672, 888, 4),     # 896 tiles: 12 waves, 8 tiles split in four (at most four)
    (8192, 8192, None, 1),     # 1024 tiles: the last wave has 62 of 74 pairs busy: whole tiles
    (512, 8192, None, 1),      # 64 tiles, one wave
])
def test_pair_plans_split_the_last_wave(M, N, full, split):
    p = plan(F8, M, N, 8192)
    tiles, pairs = p["tiles"], B200_SMS // 2
    if split == 1:
        assert p["sched"] == "dp" and p["workers"] == tiles and p["partial_bytes"] == 0
        return
    rest = tiles - full
    assert p["sched"] == "dptail" and p["tail_first"] == full and p["tail_split"] == split
    assert full == tiles // pairs * pairs and rest * split <= pairs
    assert p["workers"] == full + rest * split
    assert p["partial_bytes"] == rest * split * 2 * 128 * 256 * 4


def test_pair_grid_on_a_small_device():
    p = plan(F8, 512, 8192, 256, sms=2)
    assert p["pair"] == 1 and p["grid"] == 2


@pytest.mark.parametrize("fmt,M,K,kc", [
    (F4, 128, 128, 1),      # 64-byte rows: one partial chunk
    (F8, 128, 128, 1),      # one 128-byte chunk
    (F8, 128, 256, 2),
    (F4, 128, 512, 2),
    (F8, 64, 512, 2),       # 64-column decode tiles: two chunks (four fit only two stages)
    (F4, 64, 4096, 2),
    (F8, 64, 384, 2),       # ... and two with fewer than four
    (F4, 32, 4096, 2),
])
def test_k_chunks_per_stage(fmt, M, K, kc):
    assert plan(fmt, M, 1024, K)["kc"] == kc


def test_cluster_split_for_decode_tiles_that_fill_at_most_half_the_gpu():
    # the 64x4096x4096 decode shapes: 32 tiles, each K range over a cluster
    # of CTAs with at least four K steps each, no global partials
    for fmt, kt, ks in ((F8, 16, 4), (F4, 8, 2), (mxgemm.FMT_BF16, 32, 4)):
        p = plan(fmt, 64, 4096, 4096)
        assert (p["sched"], p["ksplit"], p["tiles"], p["kt"]) == ("ksplit", ks, 32, kt), p
        assert p["workers"] == p["grid"] == 32 * ks and p["partial_bytes"] == 0
    # 2 tiles, 32 K steps: four-way
    p = plan(F8, 32, 256, 8192)
    assert (p["sched"], p["ksplit"], p["workers"]) == ("ksplit", 4, 8)
    # 37..74 tiles: two-way
    p = plan(F8, 16, 128 * 60, 2048)
    assert (p["sched"], p["ksplit"], p["workers"]) == ("ksplit", 2, 120) and p["kt"] == 8
    # fewer than four K steps per CTA: whole tiles
    for M, N, K in [(32, 256, 512), (16, 128 * 60, 1024), (32, 1024, 1024)]:
        q = plan(F8, M, N, K)
        assert q["sched"] == "dp" and "ksplit" not in q, q
    # more than half the GPU: whole tiles
    for M, N, K in [(32, 14336, 4096), (16, 14336, 4096), (32, 4096 * 8, 8192)]:
        r = plan(F8, M, N, K)
        assert r["sched"] == "dp" and "ksplit" not in r, r


def test_global_split_k_for_few_row_tiles_with_many_k_steps():
    # not a decode tile (M > 64): 2 tiles of 128 x 128, 64 K steps: two-way
    # split with FP32 partials of 128 x BN in global memory
    p = plan(F8, 128, 256, 16384)
    assert p["sched"] == "splitk" and p["tiles"] == 2 and p["workers"] == 4 and p["grid"] == 4
    assert p["partial_bytes"] == 2 * p["workers"] * 128 * p["BN"] * 4
    q = plan(F8, 128, 256, 4096)           # 16 K steps: whole tiles
    assert q["sched"] == "dp" and q["partial_bytes"] == 0


def test_fused_scales_need_a_deep_one_cta_ring():
    for fmt, M, N, K in [(F4, 32, 14336, 4096), (F8, 32, 256, 512), (F8, 200, 640, 1536),
                         (F8, 64, 4096, 4096), (F4, 64, 4096, 4096), (F8, 4096, 4096, 4096)]:
        p = plan(fmt, M, N, K)
        assert (p["scales"] == "fused") == (p["pair"] == 0 and p["stages"] >= 4), p
    # the 64x4096x4096 decode shape: two chunks per stage, four stages, one launch
    p = plan(F8, 64, 4096, 4096)
    assert p["kc"] == 2 and p["stages"] == 4 and p["scales"] == "fused" and p["sched"] == "ksplit"


def test_plan_invariants_over_random_shapes():
    rng = np.random.default_rng(2024)
    for _ in range(400):
        fmt = int(rng.integers(0, 2))
        M = int(rng.choice([rng.integers(1, 65), rng.integers(65, 9000)]))
        N = int(rng.integers(1, 40000))
        K = 128 * int(rng.integers(1, 200))
        sms = int(rng.choice([148, 132, 2, 16]))
        p = plan(fmt, M, N, K, sms)
        assert 1 <= p["grid"] <= sms and p["workers"] >= p["tiles"]
        row_bytes = K if fmt == F8 else K // 2
        if p["pair"]:
            assert p["tiles"] == cdiv(M, 256) * cdiv(N, 256) and p["grid"] % 2 == 0
            assert p["scales"] == "repack"
            if p["sched"] == "dptail":
                rest = p["tiles"] - p["tail_first"]
                assert 0 < rest and p["workers"] == p["tail_first"] + rest * p["tail_split"]
                assert rest * p["tail_split"] <= p["grid"] // 2 and 2 <= p["tail_split"] <= 4
                assert p["partial_bytes"] == rest * p["tail_split"] * 2 * 128 * 256 * 4
                continue
        else:
            P, Q = (N, M) if p["swap"] else (M, N)
            assert p["swap"] == (1 if M <= 64 else 0)
            assert p["tiles"] == cdiv(P, 128) * cdiv(Q, p["BN"])
        assert p["kt"] == cdiv(cdiv(row_bytes, 128), p["kc"])
        assert p["stages"] >= 2
        if p["sched"] == "dp":
            assert p["workers"] == p["tiles"] and p["partial_bytes"] == 0
        elif p["sched"] == "ksplit":
            # one wave of clusters, each CTA of a cluster with >= 2 K steps
            ks = p["ksplit"]
            assert p["swap"] == 1 and p["BN"] <= 64 and ks in (2, 4)
            assert p["workers"] == p["grid"] == p["tiles"] * ks <= sms and p["kt"] >= 4 * ks
            assert p["partial_bytes"] == 0
        else:
            assert p["partial_bytes"] == 2 * p["workers"] * 128 * p["BN"] * 4
            assert p["workers"] <= p["tiles"] * p["kt"]


def test_describe_plan_for_rejects_bad_arguments():
    lib = mxgemm.load()
    buf = ctypes.create_string_buffer(256)
    assert lib.mxgemm_describe_plan_for(1, F8, 32, 256, 512, buf, 256) == mxgemm.ERR_INVALID_ARG
    assert lib.mxgemm_describe_plan_for(148, F8, 32, 256, 500, buf, 256) == mxgemm.ERR_INVALID_ARG
    assert lib.mxgemm_describe_plan_for(148, F8, 0, 256, 512, buf, 256) == mxgemm.ERR_INVALID_ARG
    assert lib.mxgemm_describe_plan_for(148, 3, 32, 256, 512, buf, 256) == mxgemm.ERR_INVALID_ARG
    assert lib.mxgemm_describe_plan_for(148, mxgemm.FMT_BF16, 32, 256, 100, buf, 256) == mxgemm.ERR_INVALID_ARG
    assert lib.mxgemm_describe_plan_for(148, F8, 32, 256, 512, buf, 0) == mxgemm.ERR_INVALID_ARG
    assert lib.mxgemm_describe_plan_for(148, F8, 32, 256, 512, None, 256) == mxgemm.ERR_INVALID_ARG
    # a short buffer is filled and NUL-terminated
    small = ctypes.create_string_buffer(16)
    assert lib.mxgemm_describe_plan_for(148, F8, 32, 256, 512, small, 16) == mxgemm.OK
    assert small.value == b"fmt=0 swap=1 pa"
