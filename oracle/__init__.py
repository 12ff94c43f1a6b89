"""CPU oracle for the MX block-scaled NT matrix multiply (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the CUDA library and its Python binding) never does.

The arithmetic lives in ``mx_oracle.c`` (plain C, FP64, one BF16 rounding at
the end); this module compiles it with gcc on first use and exposes numpy
wrappers.  See ``mx_oracle.c`` for what each function follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB = os.path.join(_HERE, "libmx_oracle.so")

FMT_MXFP8 = 0
FMT_MXFP4 = 1
FMT_BF16 = 2

_lib = None


def build(force: bool = False) -> str:
    """Compile ``mx_oracle.c`` into ``libmx_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.mxo_decode_e4m3.restype = ctypes.c_double
        lib.mxo_decode_e4m3.argtypes = [ctypes.c_uint8]
        lib.mxo_decode_e2m1.restype = ctypes.c_double
        lib.mxo_decode_e2m1.argtypes = [ctypes.c_uint8]
        lib.mxo_decode_e8m0.restype = ctypes.c_double
        lib.mxo_decode_e8m0.argtypes = [ctypes.c_uint8]
        lib.mxo_encode_e4m3.restype = ctypes.c_uint8
        lib.mxo_encode_e4m3.argtypes = [ctypes.c_double]
        lib.mxo_encode_e2m1.restype = ctypes.c_uint8
        lib.mxo_encode_e2m1.argtypes = [ctypes.c_double]
        lib.mxo_bf16_rne.restype = ctypes.c_uint16
        lib.mxo_bf16_rne.argtypes = [ctypes.c_double]
        lib.mxo_quantize.restype = None
        lib.mxo_quantize.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.mxo_gemm.restype = None
        lib.mxo_gemm.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.mxo_gemm_points.restype = None
        lib.mxo_gemm_points.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.mxo_decode_bf16.restype = ctypes.c_double
        lib.mxo_decode_bf16.argtypes = [ctypes.c_uint16]
        lib.mxo_gemm_bf16.restype = None
        lib.mxo_gemm_bf16.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.mxo_activation.restype = ctypes.c_double
        lib.mxo_activation.argtypes = [ctypes.c_int, ctypes.c_double]
        lib.mxo_epilogue.restype = None
        lib.mxo_epilogue.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.mxo_num_threads.restype = ctypes.c_int
        lib.mxo_num_threads.argtypes = []
        del u8p
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def row_bytes(fmt: int, K: int) -> int:
    return K if fmt == FMT_MXFP8 else K // 2


# ---------------------------------------------------------------- scalars

def decode_e4m3(code: int) -> float:
    return _load().mxo_decode_e4m3(code)


def decode_e2m1(nibble: int) -> float:
    return _load().mxo_decode_e2m1(nibble)


def decode_e8m0(byte: int) -> float:
    return _load().mxo_decode_e8m0(byte)


def encode_e4m3(v: float) -> int:
    return _load().mxo_encode_e4m3(v)


def encode_e2m1(v: float) -> int:
    return _load().mxo_encode_e2m1(v)


def bf16_rne(v: float) -> int:
    return _load().mxo_bf16_rne(v)


def num_threads() -> int:
    return _load().mxo_num_threads()


# ----------------------------------------------------------------- arrays

def quantize(fmt: int, X: np.ndarray):
    """OCP MX quantisation of FP32 ``X`` [R][K] -> (codes, E8M0 scales)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    R, K = X.shape
    assert K % 32 == 0
    Q = np.zeros((R, row_bytes(fmt, K)), dtype=np.uint8)
    S = np.zeros((R, K // 32), dtype=np.uint8)
    _load().mxo_quantize(fmt, R, K, _ptr(X), _ptr(Q), _ptr(S))
    return Q, S


def quantize_bf16(fmt: int, C_bits: np.ndarray):
    """OCP MX quantisation of a BF16 matrix given by its bit patterns [R][K]
    (uint16): each value widens exactly to FP32, then ``quantize`` applies.
    This is the form in which a GEMM's BF16 result becomes the MX operand of
    the next layer (one E8M0 scale per 32 consecutive values of a row, as
    the 5ulink.com page's support matrix fixes for MX operands)."""
    b = np.ascontiguousarray(C_bits, dtype=np.uint16).astype(np.uint32) << 16
    return quantize(fmt, b.view(np.float32))


def gemm(fmt: int, K: int, A: np.ndarray, SA: np.ndarray, B: np.ndarray, SB: np.ndarray,
         want_exact: bool = False):
    """C = A * B^T for MX operands.  Returns (C_bf16_bits [M][N] uint16,
    exact FP64 [M][N] or None, sum|a*b| FP64 [M][N])."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    SA = np.ascontiguousarray(SA, dtype=np.uint8)
    SB = np.ascontiguousarray(SB, dtype=np.uint8)
    M, N = A.shape[0], B.shape[0]
    assert A.shape[1] == row_bytes(fmt, K) and B.shape[1] == row_bytes(fmt, K)
    assert SA.shape == (M, K // 32) and SB.shape == (N, K // 32)
    C = np.zeros((M, N), dtype=np.uint16)
    ex = np.zeros((M, N), dtype=np.float64) if want_exact else None
    mag = np.zeros((M, N), dtype=np.float64)
    _load().mxo_gemm(fmt, M, N, K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB), _ptr(C),
                     _ptr(ex) if ex is not None else None, _ptr(mag))
    return C, ex, mag


def gemm_points(fmt: int, K: int, A, SA, B, SB, im: np.ndarray, in_: np.ndarray,
                want_exact: bool = False):
    """Selected elements C[im[i], in_[i]].  Returns (bf16 bits, exact or None, sum|a*b|)."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    SA = np.ascontiguousarray(SA, dtype=np.uint8)
    SB = np.ascontiguousarray(SB, dtype=np.uint8)
    im = np.ascontiguousarray(im, dtype=np.int64)
    in_ = np.ascontiguousarray(in_, dtype=np.int64)
    n = im.shape[0]
    assert in_.shape[0] == n
    assert im.size == 0 or (im.min() >= 0 and im.max() < A.shape[0])
    assert in_.size == 0 or (in_.min() >= 0 and in_.max() < B.shape[0])
    C = np.zeros(n, dtype=np.uint16)
    ex = np.zeros(n, dtype=np.float64) if want_exact else None
    mag = np.zeros(n, dtype=np.float64)
    _load().mxo_gemm_points(fmt, A.shape[0], B.shape[0], K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB),
                            n, _ptr(im), _ptr(in_), _ptr(C),
                            _ptr(ex) if ex is not None else None, _ptr(mag))
    return C, ex, mag


ACT_NONE, ACT_RELU, ACT_SILU, ACT_GELU = 0, 1, 2, 3


def decode_bf16(bits: int) -> float:
    return _load().mxo_decode_bf16(bits)


def activation(act: int, x: float) -> float:
    return _load().mxo_activation(act, x)


def gemm_bf16(A_bits: np.ndarray, B_bits: np.ndarray, want_exact: bool = False):
    """C = A * B^T for dense BF16 operands given as bit patterns (uint16 [M][K],
    [N][K]).  Returns (C_bf16_bits [M][N], exact FP64 or None, sum|a*b|)."""
    A = np.ascontiguousarray(A_bits, dtype=np.uint16)
    B = np.ascontiguousarray(B_bits, dtype=np.uint16)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K
    C = np.zeros((M, N), dtype=np.uint16)
    ex = np.zeros((M, N), dtype=np.float64) if want_exact else None
    mag = np.zeros((M, N), dtype=np.float64)
    _load().mxo_gemm_bf16(M, N, K, _ptr(A), _ptr(B), _ptr(C), _ptr(ex) if ex is not None else None, _ptr(mag))
    return C, ex, mag


def epilogue(exact: np.ndarray, bias_bits=None, act: int = ACT_NONE, residual_bits=None):
    """The fused epilogue from the unrounded product: C = bf16(act(exact +
    bias) + residual), one rounding.  Returns (C_bits, pre) with pre =
    exact + bias (FP64)."""
    exact = np.ascontiguousarray(exact, dtype=np.float64)
    M, N = exact.shape
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    r = None if residual_bits is None else np.ascontiguousarray(residual_bits, dtype=np.uint16)
    assert b is None or b.shape == (N,)
    assert r is None or r.shape == (M, N)
    C = np.zeros((M, N), dtype=np.uint16)
    pre = np.zeros((M, N), dtype=np.float64)
    _load().mxo_epilogue(M, N, _ptr(exact), _ptr(b) if b is not None else None, act,
                         _ptr(r) if r is not None else None, _ptr(C), _ptr(pre))
    return C, pre


def gemm_grouped(fmt: int, K: int, offsets, A, SA, B, SB):
    """Grouped product: group g's rows [off[g], off[g+1]) of A times its own
    B[g] (one plain product per group; empty groups contribute nothing).
    fmt FMT_BF16 takes BF16 bit patterns and ignores SA / SB.  Returns
    (C_bits [M_total][N], sum|a*b| [M_total][N])."""
    off = [int(x) for x in offsets]
    G = len(off) - 1
    M_total, N = A.shape[0], B.shape[1]
    C = np.zeros((M_total, N), dtype=np.uint16)
    mag = np.zeros((M_total, N), dtype=np.float64)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        if r1 <= r0:
            continue
        if fmt == FMT_BF16:
            c, _, m = gemm_bf16(A[r0:r1], B[g])
        else:
            c, _, m = gemm(fmt, K, A[r0:r1], SA[r0:r1], B[g], SB[g])
        C[r0:r1] = c
        mag[r0:r1] = m
    return C, mag


def tolerance_fused(ref_bits: np.ndarray, abssum: np.ndarray, pre: np.ndarray, residual_bits=None) -> np.ndarray:
    """Per-element bound for the fused epilogue: 1 BF16 ulp of the result +
    the product's bound 2^-18 * sum|a b| carried through the activation (whose
    slope is at most 1.13 for GELU, 1.1 for SiLU, 1 for ReLU; 1.25 here) +
    2^-19 * (|pre| + |residual|) for the FP32 rounding of the bias add, the
    activation's evaluation and the residual add (each a few FP32 ulps)."""
    res = 0.0 if residual_bits is None else np.abs(bf16_bits_to_f64(residual_bits))
    with np.errstate(invalid="ignore"):
        extra = (2.0 ** -19) * (np.abs(pre) + res)
    extra = np.where(np.isfinite(extra), extra, 0.0)
    return bf16_ulp(ref_bits) + 1.25 * (2.0 ** -18) * abssum + extra


def compare_with_tolerance(got_bits: np.ndarray, ref_bits: np.ndarray, tol: np.ndarray):
    """compare() with an explicit per-element tolerance."""
    got = bf16_bits_to_f64(got_bits)
    ref = bf16_bits_to_f64(ref_bits)
    nan_g, nan_r = np.isnan(got), np.isnan(ref)
    inf_g, inf_r = np.isinf(got), np.isinf(ref)
    pattern_ok = bool(np.array_equal(nan_g, nan_r)) and bool(
        np.array_equal(inf_g & (got > 0), inf_r & (ref > 0))) and bool(
        np.array_equal(inf_g & (got < 0), inf_r & (ref < 0)))
    fin = ~(nan_r | inf_r) & ~(nan_g | inf_g)
    with np.errstate(invalid="ignore"):
        err = np.abs(got - ref)
    bad = fin & ~(err <= tol)
    rep = {"n": int(got.size), "pattern_ok": pattern_ok, "n_bad": int(bad.sum()),
           "max_err_over_tol": float((err[fin] / tol[fin]).max()) if fin.any() else 0.0}
    if bad.any():
        idx = np.argwhere(bad)[:5]
        rep["first_bad"] = [(tuple(int(x) for x in i), float(got[tuple(i)]), float(ref[tuple(i)]),
                             float(tol[tuple(i)])) for i in idx]
    return pattern_ok and not bad.any(), rep


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float64 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_ulp(bits: np.ndarray) -> np.ndarray:
    """One BF16 ulp of each value: 2^(floor(log2|c|) - 7) for normal values,
    2^-133 for zero and subnormals; inf / nan give inf / nan."""
    v = np.abs(bf16_bits_to_f64(bits))
    out = np.full(v.shape, 2.0 ** -133, dtype=np.float64)
    normal = np.isfinite(v) & (v >= 2.0 ** -126)
    e = np.floor(np.log2(np.where(normal, v, 1.0)))
    # log2 of an exact power of two is exact; guard against a rounded-up log2
    # just below a power of two by checking the binade explicitly.
    e = np.where(normal & (2.0 ** e > v), e - 1, e)
    out = np.where(normal, 2.0 ** (e - 7), out)
    out = np.where(np.isfinite(v), out, v)
    return out


def tolerance(ref_bits: np.ndarray, abssum: np.ndarray) -> np.ndarray:
    """Per-element bound: 1 BF16 ulp of C_ref + 2^-18 * sum_k |a_k b_k|."""
    return bf16_ulp(ref_bits) + (2.0 ** -18) * abssum


def compare(got_bits: np.ndarray, ref_bits: np.ndarray, abssum: np.ndarray):
    """Element-wise parity check.  Returns (ok, report dict)."""
    got = bf16_bits_to_f64(got_bits)
    ref = bf16_bits_to_f64(ref_bits)
    nan_g, nan_r = np.isnan(got), np.isnan(ref)
    inf_g, inf_r = np.isinf(got), np.isinf(ref)
    pattern_ok = bool(np.array_equal(nan_g, nan_r)) and bool(
        np.array_equal(inf_g & (got > 0), inf_r & (ref > 0))) and bool(
        np.array_equal(inf_g & (got < 0), inf_r & (ref < 0)))
    fin = ~(nan_r | inf_r) & ~(nan_g | inf_g)
    tol = tolerance(ref_bits, abssum)
    with np.errstate(invalid="ignore"):      # inf - inf where both are infinite: not compared
        err = np.abs(got - ref)
    bad = fin & ~(err <= tol)
    rep = {
        "n": int(got.size),
        "pattern_ok": pattern_ok,
        "n_bad": int(bad.sum()),
        "max_err_over_tol": float((err[fin] / tol[fin]).max()) if fin.any() else 0.0,
        "max_abs_err": float(err[fin].max()) if fin.any() else 0.0,
        "n_exact": int((fin & (err == 0)).sum()),
    }
    if bad.any():
        idx = np.argwhere(bad)[:5]
        rep["first_bad"] = [(tuple(int(x) for x in i), float(got[tuple(i)]), float(ref[tuple(i)]),
                             float(tol[tuple(i)])) for i in idx]
    return pattern_ok and not bad.any(), rep
