"""Pins of the oracle's extensions beyond the MX product (CPU only).

* Dense BF16 GEMM (the pages' BF16 comparison suite): BF16 decoding against
  ml_dtypes for all 65 536 patterns, an integer special case against numpy
  int64 matmul, an exact-rational brute force rounded by the table search of
  test_oracle_pins, and transpose symmetry.
* Fused epilogue (the roadmap's GEMM epilogue fusion): the activations at
  textbook points (the standard normal CDF Phi(1) = 0.8413447460685429,
  Phi(2) = 0.9772498680518208, Phi(-10) = 7.619853024160527e-24; the logistic
  function at +-1), against scipy's independent ndtr / expit on a grid, an
  integer bias + ReLU + residual case against numpy int64 arithmetic, and the
  one rounding of act(pre) + residual against exact rationals.
* Grouped product: uneven and empty groups against numpy int64 matmul per
  group, and against one oracle call per group.
"""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import scipy.special

import oracle
from test_oracle_pins import nearest_bf16_bits


def _bf16_bits(x):
    return np.asarray(x, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


# ------------------------------------------------------------ BF16 GEMM

def test_bf16_decode_all_patterns_against_ml_dtypes():
    bits = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(ml_dtypes.bfloat16).astype(np.float64)
    for b in range(0, 0x10000, 97):                 # the scalar entry on a spread of codes
        got = oracle.decode_bf16(b)
        assert (math.isnan(got) and math.isnan(ref[b])) or got == ref[b], hex(b)
    # all codes through the product path: A = [x], B = [1.0]
    one = _bf16_bits([[1.0]])
    C, ex, _ = oracle.gemm_bf16(bits.reshape(-1, 1), one, want_exact=True)
    fin = np.isfinite(ref)
    assert np.array_equal(ex[fin, 0], ref[fin])
    assert np.isnan(ex[np.isnan(ref), 0]).all()


def test_bf16_gemm_integer_case_vs_numpy():
    rng = np.random.default_rng(3)
    M, N, K = 19, 23, 200
    ai = rng.integers(-60, 61, (M, K))
    bi = rng.integers(-60, 61, (N, K))
    C, ex, mag = oracle.gemm_bf16(_bf16_bits(ai), _bf16_bits(bi), want_exact=True)
    exact = ai.astype(np.int64) @ bi.astype(np.int64).T
    assert np.array_equal(ex, exact.astype(np.float64))
    assert np.array_equal(mag, (np.abs(ai).astype(np.int64) @ np.abs(bi).astype(np.int64).T).astype(np.float64))
    for (m, n) in [(0, 0), (3, 7), (M - 1, N - 1)]:
        assert C[m, n] == nearest_bf16_bits(int(exact[m, n]))


def test_bf16_gemm_brute_force_exact_rationals():
    rng = np.random.default_rng(11)
    M, N, K = 3, 4, 40
    a = _bf16_bits(rng.standard_normal((M, K)) * np.exp2(rng.integers(-30, 30, (M, K))))
    b = _bf16_bits(rng.standard_normal((N, K)) * np.exp2(rng.integers(-30, 30, (N, K))))
    C, _, _ = oracle.gemm_bf16(a, b)
    av = a.view(ml_dtypes.bfloat16).astype(np.float64)
    bv = b.view(ml_dtypes.bfloat16).astype(np.float64)
    for m in range(M):
        for n in range(N):
            s = sum(Fraction(float(av[m, k])) * Fraction(float(bv[n, k])) for k in range(K))
            assert C[m, n] == nearest_bf16_bits(s), (m, n)


def test_bf16_gemm_transpose_symmetry():
    rng = np.random.default_rng(5)
    a = _bf16_bits(rng.standard_normal((7, 64)))
    b = _bf16_bits(rng.standard_normal((9, 64)))
    C1, _, _ = oracle.gemm_bf16(a, b)
    C2, _, _ = oracle.gemm_bf16(b, a)
    assert np.array_equal(C1, C2.T)


# ------------------------------------------------------- fused epilogue

@pytest.mark.parametrize("act,x,y", [
    (oracle.ACT_RELU, -3.0, 0.0), (oracle.ACT_RELU, 2.5, 2.5), (oracle.ACT_RELU, 0.0, 0.0),
    (oracle.ACT_SILU, 0.0, 0.0), (oracle.ACT_SILU, 1.0, 0.7310585786300049),
    (oracle.ACT_SILU, -1.0, -0.2689414213699951),
    (oracle.ACT_GELU, 0.0, 0.0), (oracle.ACT_GELU, 1.0, 0.8413447460685429),
    (oracle.ACT_GELU, -1.0, -(1.0 - 0.8413447460685429)), (oracle.ACT_GELU, 2.0, 2 * 0.9772498680518208),
    (oracle.ACT_GELU, -10.0, -10 * 7.619853024160527e-24), (oracle.ACT_NONE, -7.25, -7.25),
])
def test_activation_textbook_values(act, x, y):
    assert oracle.activation(act, x) == pytest.approx(y, rel=1e-12, abs=0.0)


def test_activation_special_values():
    assert math.isnan(oracle.activation(oracle.ACT_RELU, float("nan")))
    assert math.copysign(1.0, oracle.activation(oracle.ACT_RELU, -0.0)) == -1.0   # x < 0 is false for -0
    assert math.isnan(oracle.activation(oracle.ACT_SILU, float("nan")))
    assert math.isnan(oracle.activation(oracle.ACT_GELU, float("nan")))
    assert oracle.activation(oracle.ACT_GELU, 40.0) == 40.0
    assert oracle.activation(oracle.ACT_SILU, -800.0) == 0.0


@pytest.mark.parametrize("act,ref", [
    (oracle.ACT_SILU, lambda x: x * scipy.special.expit(x)),
    (oracle.ACT_GELU, lambda x: x * scipy.special.ndtr(x)),
])
def test_activation_against_scipy(act, ref):
    xs = np.concatenate([np.linspace(-30, 30, 1201), -np.geomspace(1e-6, 37, 200), np.geomspace(1e-6, 37, 200)])
    for x in xs:
        y = ref(x)
        got = oracle.activation(act, float(x))
        assert got == pytest.approx(y, rel=1e-12, abs=1e-300), x


def test_epilogue_integer_bias_relu_residual_vs_numpy():
    rng = np.random.default_rng(9)
    M, N = 13, 40
    exact = rng.integers(-200, 200, (M, N)).astype(np.float64)
    bias = rng.integers(-50, 50, N)
    res = rng.integers(-50, 50, (M, N))
    C, pre = oracle.epilogue(exact, _bf16_bits(bias), oracle.ACT_RELU, _bf16_bits(res))
    want = np.maximum(exact.astype(np.int64) + bias, 0) + res
    assert np.array_equal(pre, exact + bias)
    assert np.array_equal(oracle.bf16_bits_to_f64(C), want.astype(np.float64))   # |want| <= 300: exact in BF16
    C0, pre0 = oracle.epilogue(exact)
    assert np.array_equal(oracle.bf16_bits_to_f64(C0), exact) and np.array_equal(pre0, exact)


def test_epilogue_rounds_once():
    # pre = 1 + 2^-8 (a BF16 midpoint) and residual 2^-30: one rounding of the
    # exact sum goes up to 1 + 2^-7, rounding pre first would go to 1 (even)
    exact = np.array([[1.0 + 2.0 ** -8]])
    res = _bf16_bits([[2.0 ** -30]])
    C, _ = oracle.epilogue(exact, None, oracle.ACT_NONE, res)
    assert C[0, 0] == nearest_bf16_bits(Fraction(1) + Fraction(1, 256) + Fraction(1, 2 ** 30))
    assert oracle.bf16_bits_to_f64(C)[0, 0] == 1.0 + 2.0 ** -7
    rng = np.random.default_rng(21)
    exact = rng.standard_normal((6, 8)) * 10
    bias = _bf16_bits(rng.standard_normal(8))
    res = _bf16_bits(rng.standard_normal((6, 8)))
    C, pre = oracle.epilogue(exact, bias, oracle.ACT_RELU, res)
    bv = bias.view(ml_dtypes.bfloat16).astype(np.float64)
    rv = res.view(ml_dtypes.bfloat16).astype(np.float64)
    for m in range(6):
        for n in range(8):
            p = Fraction(float(exact[m, n])) + Fraction(float(bv[n]))
            v = (p if p >= 0 else Fraction(0)) + Fraction(float(rv[m, n]))
            assert C[m, n] == nearest_bf16_bits(v)


def test_fused_tolerance_reduces_to_the_product_rule():
    ref = _bf16_bits([[1.0, -3.0]])
    mag = np.array([[10.0, 0.0]])
    t = oracle.tolerance_fused(ref, mag, np.zeros((1, 2)))
    assert np.allclose(t, oracle.bf16_ulp(ref) + 1.25 * 2.0 ** -18 * mag)
    t2 = oracle.tolerance_fused(ref, mag, np.array([[4.0, -8.0]]), _bf16_bits([[2.0, 2.0]]))
    assert np.allclose(t2 - t, 2.0 ** -19 * np.array([[6.0, 10.0]]))


# --------------------------------------------------------- grouped product

def _int_codes_f8(vals):
    table = {int(v): oracle.encode_e4m3(float(v)) for v in range(-16, 17)}
    return np.vectorize(table.get)(vals).astype(np.uint8)


def test_grouped_uneven_and_empty_groups_vs_numpy():
    rng = np.random.default_rng(12)
    K, N = 256, 40
    sizes = [0, 5, 130, 0, 1, 77, 0]
    off = np.concatenate([[0], np.cumsum(sizes)])
    M = int(off[-1])
    G = len(sizes)
    ai = rng.integers(-16, 17, (M, K))
    bi = rng.integers(-16, 17, (G, N, K))
    A = _int_codes_f8(ai)
    B = _int_codes_f8(bi)
    SA = np.full((M, K // 32), 0x7F, np.uint8)
    SB = np.full((G, N, K // 32), 0x7F, np.uint8)
    C, mag = oracle.gemm_grouped(oracle.FMT_MXFP8, K, off, A, SA, B, SB)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        want = ai[r0:r1].astype(np.int64) @ bi[g].astype(np.int64).T
        got = oracle.bf16_bits_to_f64(C[r0:r1])
        small = np.abs(want) <= 256
        assert np.array_equal(got[small], want[small].astype(np.float64))
        c1, _, m1 = oracle.gemm(oracle.FMT_MXFP8, K, A[r0:r1], SA[r0:r1], B[g], SB[g])
        assert np.array_equal(C[r0:r1], c1) and np.array_equal(mag[r0:r1], m1)


def test_grouped_bf16_vs_numpy():
    rng = np.random.default_rng(14)
    K, N = 48, 24
    off = np.array([0, 3, 3, 20, 21])
    ai = rng.integers(-30, 31, (21, K))
    bi = rng.integers(-30, 31, (4, N, K))
    C, _ = oracle.gemm_grouped(oracle.FMT_BF16, K, off, _bf16_bits(ai), None, _bf16_bits(bi), None)
    for g in range(4):
        want = ai[off[g]:off[g + 1]].astype(np.int64) @ bi[g].astype(np.int64).T
        for (m, n), w in np.ndenumerate(want):
            assert C[off[g] + m, n] == nearest_bf16_bits(int(w))
