"""Pins for the CPU oracle: checks against what the formats and the
mathematics fix, never against the oracle itself.

Independent sources used here:
  * closed-form value sets of the formats (E2M1 magnitudes, E4M3 max 448 and
    NaN code, E8M0 2^(e-127) and NaN);
  * ml_dtypes' float8_e4m3fn / float4_e2m1fn / float8_e8m0fnu / bfloat16
    types (a separate implementation of the same encodings);
  * exact rational arithmetic (fractions.Fraction) for tiny GEMMs;
  * numpy int64 matmul for the integer special case;
  * hand-worked examples in tests/golden/hand_sums.json.
"""
import json
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_sums.json")
FMT = {"mxfp8": oracle.FMT_MXFP8, "mxfp4": oracle.FMT_MXFP4}


# ----------------------------------------------------------------- helpers

def _bf16_table():
    bits = np.arange(0x10000, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << 16).view(np.float32).astype(np.float64)
    fin = np.isfinite(vals) & ~((bits & 0x8000) != 0)  # non-negative finite
    pos_bits = bits[fin]
    pos_vals = vals[fin]
    order = np.argsort(pos_vals, kind="stable")
    pos_vals, pos_bits = pos_vals[order], pos_bits[order]
    # drop the duplicate +0 / keep one entry per value
    keep = np.concatenate([[True], np.diff(pos_vals) > 0])
    return pos_vals[keep], pos_bits[keep]


_BF_VALS, _BF_BITS = _bf16_table()
_BF_MAX = Fraction(float(_BF_VALS[-1]))
_BF_HALF_ULP_MAX = Fraction(2) ** 119  # ulp at the top binade is 2^120


def nearest_bf16_bits(x) -> int:
    """Round an exact value (Fraction or float) to BF16 by searching the table
    of all BF16 values: nearest value, ties to the even code, +-inf past
    max + half an ulp.  An implementation independent of the oracle's."""
    if isinstance(x, float) and math.isnan(x):
        return 0x7FC0
    x = Fraction(x)
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    if a >= _BF_MAX + _BF_HALF_ULP_MAX:
        return sign | 0x7F80
    i = int(np.searchsorted(_BF_VALS, float(a)))
    cands = []
    for j in (i - 1, i, i + 1):
        if 0 <= j < len(_BF_VALS):
            cands.append((abs(Fraction(float(_BF_VALS[j])) - a), int(_BF_BITS[j]) & 1, int(_BF_BITS[j])))
    cands.sort()
    best = cands[0]
    if len(cands) > 1 and cands[1][0] == best[0] and cands[1][2] != best[2]:
        best = min(cands[0], cands[1], key=lambda c: c[1])  # even code wins
    return sign | best[2]


def e4m3_values():
    return np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def e2m1_values():
    return np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def e8m0_values():
    return np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)


def _expand(rows):
    out = []
    for r in rows:
        bs = []
        for code, cnt in r:
            bs += [int(code, 16)] * cnt
        out.append(bs)
    return np.array(out, dtype=np.uint8)


# --------------------------------------------------------------- decoders

def test_e2m1_value_set_closed_form():
    vals = [oracle.decode_e2m1(c) for c in range(16)]
    assert sorted(set(abs(v) for v in vals)) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert vals[0] == 0.0 and vals[8] == 0.0
    assert vals[:8] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert vals[8:] == [-v for v in vals[:8]]


def test_e2m1_matches_ml_dtypes():
    ref = e2m1_values()
    for c in range(16):
        assert oracle.decode_e2m1(c) == ref[c]


def test_e4m3_special_codes():
    assert oracle.decode_e4m3(0x7E) == 448.0
    assert oracle.decode_e4m3(0xFE) == -448.0
    assert math.isnan(oracle.decode_e4m3(0x7F)) and math.isnan(oracle.decode_e4m3(0xFF))
    assert oracle.decode_e4m3(0x01) == 2.0 ** -9
    assert oracle.decode_e4m3(0x08) == 2.0 ** -6
    assert oracle.decode_e4m3(0x38) == 1.0
    assert oracle.decode_e4m3(0x00) == 0.0 and oracle.decode_e4m3(0x80) == 0.0
    finite = [oracle.decode_e4m3(c) for c in range(256) if not math.isnan(oracle.decode_e4m3(c))]
    assert len(finite) == 254 and max(finite) == 448.0 and min(finite) == -448.0


def test_e4m3_matches_ml_dtypes_all_codes():
    ref = e4m3_values()
    for c in range(256):
        v = oracle.decode_e4m3(c)
        if math.isnan(ref[c]):
            assert math.isnan(v)
        else:
            assert v == ref[c], hex(c)


def test_e8m0_codes():
    assert oracle.decode_e8m0(0x7F) == 1.0
    assert oracle.decode_e8m0(0x00) == 2.0 ** -127
    assert oracle.decode_e8m0(0xFE) == 2.0 ** 127
    assert math.isnan(oracle.decode_e8m0(0xFF))
    ref = e8m0_values()
    for b in range(255):
        assert oracle.decode_e8m0(b) == ref[b]


# --------------------------------------------------------------- encoders

def test_e4m3_encode_roundtrips_every_code():
    for c in range(256):
        v = oracle.decode_e4m3(c)
        if math.isnan(v):
            assert oracle.encode_e4m3(v) == 0x7F
            continue
        got = oracle.encode_e4m3(v)
        assert got == c, (hex(c), hex(got))


def test_e2m1_encode_roundtrips_every_code():
    for c in range(16):
        assert oracle.encode_e2m1(oracle.decode_e2m1(c)) == c


@pytest.mark.parametrize("x,code", [
    (0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
    (5.0, 0x6), (5.5, 0x7), (6.0, 0x7), (7.0, 0x7), (100.0, 0x7), (0.2, 0x0),
    (0.26, 0x1), (-0.25, 0x8), (-5.0, 0xE), (-1e-30, 0x8),
])
def test_e2m1_ties_and_saturation(x, code):
    assert oracle.encode_e2m1(x) == code


@pytest.mark.parametrize("x,code", [
    (448.0, 0x7E), (460.0, 0x7E), (464.0, 0x7E), (1e9, 0x7E), (-1e9, 0xFE),
    (2.0 ** -10, 0x00),            # half of the smallest subnormal: tie to even 0
    (3 * 2.0 ** -10, 0x02),        # 1.5 subnormal steps: tie to even 2
    (-2.0 ** -12, 0x80),           # negative value rounding to zero keeps its sign
    (1.0625, 0x38),                # 1 + 1/16: tie between 1 and 1.125 -> even (1)
    (1.1875, 0x3A),                # 1 + 3/16: tie between 1.125 and 1.25 -> even (1.25)
    (15.5 * 2.0 ** -7, 0x20),      # 1.9375 * 2^-4: tie between 1.875*2^-4 (0x1F) and 2^-3 (0x20)
    (15.0 * 2.0 ** -10, 0x08),     # 7.5 subnormal steps: tie between 0x07 and 2^-6 (0x08) -> even
])
def test_e4m3_ties_and_saturation(x, code):
    assert oracle.encode_e4m3(x) == code


def test_e4m3_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(123)
    x = np.concatenate([
        rng.standard_normal(20000) * 50.0,
        rng.standard_normal(20000) * 2.0 ** -7,
        np.clip(rng.standard_normal(5000) * 300.0, -447.9, 447.9),
    ])
    x = x[np.abs(x) < 448.0].astype(np.float32).astype(np.float64)
    ref = x.astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([oracle.encode_e4m3(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(7)
    x = rng.uniform(-6.0, 6.0, 20000)
    x = np.concatenate([x, np.arange(-24, 25) / 4.0])  # every quarter: all ties
    ref = x.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.array([oracle.encode_e2m1(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)


# -------------------------------------------------------------- quantiser

def _independent_quantize(fmt, X):
    """The OCP MX rule written with numpy + ml_dtypes casts (not the oracle):
    scale exponent from frexp of the block amax, elements cast by ml_dtypes
    after clipping to the format's max (saturation)."""
    R, K = X.shape
    emax, vmax = (8, 448.0) if fmt == oracle.FMT_MXFP8 else (2, 6.0)
    Xb = X.astype(np.float64).reshape(R, K // 32, 32)
    amax = np.abs(Xb).max(axis=2)
    _, ex = np.frexp(amax)
    s = np.where(amax > 0, ex - 1 - emax, -127)
    s = np.clip(s, -127, 127)
    S = (s + 127).astype(np.uint8)
    q = np.clip(Xb * np.exp2(-s)[..., None], -vmax, vmax).reshape(R, K)
    if fmt == oracle.FMT_MXFP8:
        Q = q.astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    else:
        nib = q.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
        Q = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return Q, S


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
@pytest.mark.parametrize("kind", ["normal", "heavy"])
def test_quantize_matches_independent_rule(fmt, kind):
    from microscaling_block_scaled_b200 import synth
    A, _ = synth.operands(16, 1, 256, seed=11, kind=kind)
    X = A.numpy()
    Q, S = oracle.quantize(fmt, X)
    Qr, Sr = _independent_quantize(fmt, X)
    assert np.array_equal(S, Sr)
    # ml_dtypes maps a negative value that rounds to zero to +0 or -0 the same
    # way IEEE does (sign kept), so codes compare exactly.
    assert np.array_equal(Q, Qr)


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_quantize_amax_lands_in_top_binade_and_is_idempotent(fmt):
    from microscaling_block_scaled_b200 import synth
    A, _ = synth.operands(8, 1, 512, seed=5, kind="heavy")
    X = A.numpy()
    Q, S = oracle.quantize(fmt, X)
    emax = 8 if fmt == oracle.FMT_MXFP8 else 2
    dec = (e4m3_values()[Q] if fmt == oracle.FMT_MXFP8 else
           np.stack([e2m1_values()[Q & 0xF], e2m1_values()[Q >> 4]], axis=-1).reshape(8, 512))
    blocks = np.abs(dec.reshape(8, 16, 32)).max(axis=2)
    nz = np.abs(X.reshape(8, 16, 32)).max(axis=2) > 0
    assert np.all(blocks[nz] >= 2.0 ** emax) and np.all(blocks[nz] < 2.0 ** (emax + 1))
    assert np.all(S[~nz] == 0)
    # idempotence: the dequantised values quantise back to the same codes
    deq = (dec.reshape(8, 16, 32) * e8m0_values()[S][..., None]).reshape(8, 512).astype(np.float32)
    Q2, S2 = oracle.quantize(fmt, deq)
    assert np.array_equal(S2, S) and np.array_equal(Q2, Q)


def test_quantize_edge_blocks():
    X = np.zeros((1, 160), dtype=np.float32)
    X[0, 32:64] = -0.0                        # all -0: zero block, sign kept
    X[0, 64] = np.float32(2.0 ** -140)        # FP32 subnormal amax
    X[0, 96:128] = np.float32(np.nan)         # non-finite block
    X[0, 128] = 1000.0                        # saturating block
    X[0, 129] = 930.0                         # 465 in the scaled domain -> 448
    Q, S = oracle.quantize(oracle.FMT_MXFP8, X)
    assert S[0, 0] == 0x00 and np.all(Q[0, :32] == 0x00)
    assert S[0, 1] == 0x00 and np.all(Q[0, 32:64] == 0x80)
    # floor(log2 2^-140) - 8 = -148 -> clamped to -127; 2^-140 * 2^127 = 2^-13 -> rounds to 0
    assert S[0, 2] == 0x00 and Q[0, 64] == 0x00
    assert S[0, 3] == 0xFF and np.all(Q[0, 96:128] == 0)
    # amax 1000: floor(log2) = 9, scale 2^1, 1000/2 = 500 -> saturates to 448
    assert S[0, 4] == 0x80 and Q[0, 128] == 0x7E and Q[0, 129] == 0x7E


# ---------------------------------------------------------- BF16 rounding

def test_bf16_rne_against_table_search():
    rng = np.random.default_rng(99)
    xs = list(rng.standard_normal(3000) * np.exp2(rng.uniform(-140, 130, 3000)))
    # exact ties and near-ties around random BF16 values
    for b in rng.integers(0x0001, 0x7F7F, 1500):
        v = float(((np.uint32(b) << 16).view(np.float32)))
        up = float(((np.uint32(b + 1) << 16).view(np.float32)))
        mid = (v + up) / 2
        xs += [mid, -mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)]
    xs += [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** -126,
           float(_BF_MAX), float(_BF_MAX + _BF_HALF_ULP_MAX), np.nextafter(float(_BF_MAX + _BF_HALF_ULP_MAX), 0),
           1e300, -1e300, float("inf"), float("-inf")]
    for x in xs:
        x = float(x)
        if math.isinf(x):
            assert oracle.bf16_rne(x) == (0x7F80 if x > 0 else 0xFF80)
            continue
        got = oracle.bf16_rne(x)
        want = nearest_bf16_bits(x)
        if x == 0:
            want = 0x8000 if math.copysign(1, x) < 0 else 0
        assert got == want, (x, hex(got), hex(want))
    assert oracle.bf16_rne(float("nan")) & 0x7FFF == 0x7FC0


# ------------------------------------------------------------------- GEMM

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_gemm_hand_sums(case):
    fmt = FMT[case["fmt"]]
    K = case["K"]
    A, B = _expand(case["A"]), _expand(case["B"])
    SA = np.array([[int(x, 16) for x in r] for r in case["SA"]], dtype=np.uint8)
    SB = np.array([[int(x, 16) for x in r] for r in case["SB"]], dtype=np.uint8)
    C, ex, _ = oracle.gemm(fmt, K, A, SA, B, SB, want_exact=True)
    for i, row in enumerate(case["C_bf16"]):
        for j, want in enumerate(row):
            if want == "nan":
                assert (C[i, j] & 0x7FFF) > 0x7F80
                assert math.isnan(ex[i, j])
            else:
                assert C[i, j] == int(want, 16), (case["name"], i, j, hex(C[i, j]))
                assert ex[i, j] == case["C_value"][i][j]


def _fraction_gemm(fmt, K, A, SA, B, SB):
    """Exact rational C = A * B^T with ml_dtypes decoding."""
    e8 = e8m0_values()
    if fmt == oracle.FMT_MXFP8:
        da = e4m3_values()[A]
        db = e4m3_values()[B]
    else:
        t = e2m1_values()
        da = np.stack([t[A & 0xF], t[A >> 4]], axis=-1).reshape(A.shape[0], K)
        db = np.stack([t[B & 0xF], t[B >> 4]], axis=-1).reshape(B.shape[0], K)
    M, N = da.shape[0], db.shape[0]
    out = []
    for m in range(M):
        row = []
        for n in range(N):
            tot = Fraction(0)
            for k in range(K):
                sa = Fraction(float(e8[SA[m, k // 32]]))
                sb = Fraction(float(e8[SB[n, k // 32]]))
                tot += sa * sb * Fraction(float(da[m, k])) * Fraction(float(db[n, k]))
            row.append(tot)
        out.append(row)
    return out


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_gemm_brute_force_exact_rationals(fmt):
    rng = np.random.default_rng(2024 + fmt)
    M, N, K = 3, 4, 96
    rb = oracle.row_bytes(fmt, K)
    A = rng.integers(0, 256, (M, rb), dtype=np.uint8)
    B = rng.integers(0, 256, (N, rb), dtype=np.uint8)
    if fmt == oracle.FMT_MXFP8:   # keep elements finite (no NaN code)
        A[(A & 0x7F) == 0x7F] = 0x11
        B[(B & 0x7F) == 0x7F] = 0x22
    SA = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
    SB = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
    C, ex, mag = oracle.gemm(fmt, K, A, SA, B, SB, want_exact=True)
    exact = _fraction_gemm(fmt, K, A, SA, B, SB)
    for m in range(M):
        for n in range(N):
            assert int(C[m, n]) == nearest_bf16_bits(exact[m][n])
            # the FP64 sum is exact up to the cross-block rounding
            assert abs(Fraction(ex[m, n]) - exact[m][n]) <= Fraction(mag[m, n]) * Fraction(2) ** -50


def test_gemm_integer_special_case_vs_numpy_matmul():
    rng = np.random.default_rng(5)
    M, N, K = 5, 7, 256
    ai = rng.integers(-16, 17, (M, K))
    bi = rng.integers(-16, 17, (N, K))
    enc = {v: oracle.encode_e4m3(float(v)) for v in range(-16, 17)}
    A = np.vectorize(enc.get)(ai).astype(np.uint8)
    B = np.vectorize(enc.get)(bi).astype(np.uint8)
    SA = np.full((M, K // 32), 0x7F, np.uint8)
    SB = np.full((N, K // 32), 0x7F, np.uint8)
    C, ex, _ = oracle.gemm(oracle.FMT_MXFP8, K, A, SA, B, SB, want_exact=True)
    ref = ai.astype(np.int64) @ bi.astype(np.int64).T
    assert np.array_equal(ex, ref.astype(np.float64))
    want = np.vectorize(lambda v: nearest_bf16_bits(int(v)))(ref)
    assert np.array_equal(C.astype(np.int64), want)
    # and the E2M1 integers {0, +-1, +-2, +-3, +-4, +-6}
    vals = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    ai = rng.choice(vals, (M, K))
    bi = rng.choice(vals, (N, K))
    e2 = {v: oracle.encode_e2m1(float(v)) for v in vals}
    na = np.vectorize(e2.get)(ai).astype(np.uint8)
    nb = np.vectorize(e2.get)(bi).astype(np.uint8)
    A = (na[:, 0::2] | (na[:, 1::2] << 4)).astype(np.uint8)
    B = (nb[:, 0::2] | (nb[:, 1::2] << 4)).astype(np.uint8)
    C, ex, _ = oracle.gemm(oracle.FMT_MXFP4, K, A, SA, B, SB, want_exact=True)
    ref = ai.astype(np.int64) @ bi.astype(np.int64).T
    assert np.array_equal(ex, ref.astype(np.float64))


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_scale_increment_doubles_exactly_that_block(fmt):
    rng = np.random.default_rng(77)
    M, N, K = 2, 3, 128
    rb = oracle.row_bytes(fmt, K)
    A = rng.integers(0, 256, (M, rb), dtype=np.uint8)
    B = rng.integers(0, 256, (N, rb), dtype=np.uint8)
    if fmt == oracle.FMT_MXFP8:
        A[(A & 0x7F) == 0x7F] = 0x3C
        B[(B & 0x7F) == 0x7F] = 0x3C
    SA = np.full((M, K // 32), 0x7F, np.uint8)
    SB = np.full((N, K // 32), 0x7F, np.uint8)
    _, base, _ = oracle.gemm(fmt, K, A, SA, B, SB, want_exact=True)
    # contribution of block j alone: zero every other block's A elements
    for j in range(K // 32):
        Aj = np.zeros_like(A)
        lo, hi = j * 32 * rb // K, (j + 1) * 32 * rb // K
        Aj[:, lo:hi] = A[:, lo:hi]
        _, contrib, _ = oracle.gemm(fmt, K, Aj, SA, B, SB, want_exact=True)
        SA2 = SA.copy()
        SA2[0, j] += 1
        _, bumped, _ = oracle.gemm(fmt, K, A, SA2, B, SB, want_exact=True)
        assert np.array_equal(bumped[0], base[0] + contrib[0])   # row 0 gains that block once more
        assert np.array_equal(bumped[1], base[1])                # other rows unchanged


def test_points_agree_with_full_and_transpose_symmetry():
    from microscaling_block_scaled_b200 import synth
    A32, B32 = synth.operands(9, 13, 256, seed=3)
    for fmt in (oracle.FMT_MXFP8, oracle.FMT_MXFP4):
        A, SA = oracle.quantize(fmt, A32.numpy())
        B, SB = oracle.quantize(fmt, B32.numpy())
        C, _, mag = oracle.gemm(fmt, 256, A, SA, B, SB)
        CT, _, _ = oracle.gemm(fmt, 256, B, SB, A, SA)
        assert np.array_equal(C, CT.T)
        im, in_ = np.meshgrid(np.arange(9), np.arange(13), indexing="ij")
        P, _, pm = oracle.gemm_points(fmt, 256, A, SA, B, SB, im.ravel(), in_.ravel())
        assert np.array_equal(P, C.ravel()) and np.array_equal(pm, mag.ravel())


def test_tolerance_ulp_rule():
    bits = np.array([0x3F80, 0x0000, 0x0001, 0x4300, 0xC300, 0x7F80, 0x3F7F], dtype=np.uint16)
    u = oracle.bf16_ulp(bits)
    assert u[0] == 2.0 ** -7          # 1.0
    assert u[1] == 2.0 ** -133 and u[2] == 2.0 ** -133
    assert u[3] == 2.0 ** 0 and u[4] == 2.0 ** 0   # +-128
    assert np.isinf(u[5])
    assert u[6] == 2.0 ** -8          # just below 1.0


def test_compare_accepts_and_rejects_by_the_rule():
    """The parity comparison itself: within 1 ulp + 2^-18 * sum|ab| passes,
    2 ulp with no magnitude term fails, and the NaN / +Inf / -Inf positions
    must match exactly (an Inf of the wrong sign, or a NaN for a finite
    value, fails)."""
    one, one_up, one_up2 = 0x3F80, 0x3F81, 0x3F82       # 1, 1 + 2^-7, 1 + 2^-6
    pinf, ninf, qnan = 0x7F80, 0xFF80, 0x7FC0
    z = np.zeros(1)
    ok, _ = oracle.compare(np.array([one_up], np.uint16), np.array([one], np.uint16), z)
    assert ok                                            # exactly 1 ulp
    ok, rep = oracle.compare(np.array([one_up2], np.uint16), np.array([one], np.uint16), z)
    assert not ok and rep["n_bad"] == 1                  # 2 ulp
    ok, _ = oracle.compare(np.array([one_up2], np.uint16), np.array([one], np.uint16), np.array([2.0 ** 11]))
    assert ok                                            # 2^-18 * 2^11 = 2^-7 of extra slack
    for got, ref, want in [(qnan, qnan, True), (pinf, pinf, True), (ninf, ninf, True),
                           (pinf, ninf, False), (qnan, one, False), (one, qnan, False), (pinf, one, False)]:
        ok, rep = oracle.compare(np.array([got], np.uint16), np.array([ref], np.uint16), z)
        assert ok == want, (hex(got), hex(ref), rep)


# ------------------------------------------- MX quantisation of BF16 output

def test_quantize_bf16_hand_worked_block():
    # one block of a row: 1.0, 2.0, then 30 zeros.  amax 2 = 2^1.
    #  MXFP8: scale exponent 1 - 8 = -7 (byte 120); 1 * 2^7 = 128 = 2^7 -> E4M3
    #  exponent field 7 + 7 = 14, mantissa 0 -> 0x70; 256 -> field 15 -> 0x78.
    #  MXFP4: scale exponent 1 - 2 = -1 (byte 126); 1 * 2 = 2.0 -> E2M1 0b0100,
    #  2 * 2 = 4.0 -> 0b0110; packed low nibble first -> 0x64.
    bits = np.zeros((1, 32), dtype=np.uint16)
    bits[0, 0], bits[0, 1] = 0x3F80, 0x4000
    Q8, S8 = oracle.quantize_bf16(oracle.FMT_MXFP8, bits)
    assert S8.tolist() == [[120]] and Q8[0, 0] == 0x70 and Q8[0, 1] == 0x78 and not Q8[0, 2:].any()
    Q4, S4 = oracle.quantize_bf16(oracle.FMT_MXFP4, bits)
    assert S4.tolist() == [[126]] and Q4[0, 0] == 0x64 and not Q4[0, 1:].any()


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_quantize_bf16_matches_ml_dtypes_widening_and_independent_rule(fmt):
    rng = np.random.default_rng(31)
    # BF16 bit patterns of finite values over a wide exponent range, some
    # blocks zero, some negative zero
    v = (rng.standard_normal((12, 256)) * np.exp2(rng.integers(-30, 30, (12, 1)))).astype(np.float32)
    v[3, 64:96] = 0.0
    v[5, 0:32] = -0.0
    bits = v.astype(ml_dtypes.bfloat16).view(np.uint16)
    Q, S = oracle.quantize_bf16(fmt, bits)
    widened = bits.view(ml_dtypes.bfloat16).astype(np.float32)
    Qr, Sr = _independent_quantize(fmt, widened)
    assert np.array_equal(S, Sr) and np.array_equal(Q, Qr)


def test_quantize_bf16_exact_round_trip_for_representable_blocks():
    # BF16 values with at most 3 mantissa bits, within 2^8 of the block's
    # amax binade and with significand at most 1.75 (the block amax scales to
    # 2^8 times its significand, and 1.875 * 2^8 = 480 would saturate to 448)
    # are E4M3 values times the block scale: MXFP8 reproduces them.
    rng = np.random.default_rng(32)
    mant = rng.integers(8, 15, (4, 64)).astype(np.float64) / 8.0          # 1.mmm, mmm <= 110
    expo = rng.integers(-5, 3, (4, 64)).astype(np.float64)
    sign = np.where(rng.random((4, 64)) < 0.5, -1.0, 1.0)
    x = (sign * mant * np.exp2(expo)).astype(np.float32)
    bits = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(bits.view(ml_dtypes.bfloat16).astype(np.float32), x)   # exact in BF16
    Q, S = oracle.quantize_bf16(oracle.FMT_MXFP8, bits)
    dec = e4m3_values()[Q].reshape(4, 2, 32) * e8m0_values()[S][..., None]
    assert np.array_equal(dec.reshape(4, 64), x.astype(np.float64))
