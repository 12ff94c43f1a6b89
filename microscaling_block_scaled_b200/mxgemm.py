"""Python binding of ``libmxgemm.so`` (ctypes; argument marshalling only).

Every function named ``mxgemm_*`` here calls the C entry point of the same
name declared in ``include/mxgemm.h``; the ``Handle`` class and the
``quantize`` / ``run`` helpers only turn torch tensors into pointers, sizes
and the current CUDA stream.  There is no fallback: if the shared library is
missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmxgemm.so")

FMT_MXFP8 = 0
FMT_MXFP4 = 1
FMT_BF16 = 2
FMT_NAMES = {"mxfp8": FMT_MXFP8, "mxfp4": FMT_MXFP4, "bf16": FMT_BF16}

ACT_NONE, ACT_RELU, ACT_SILU, ACT_GELU = 0, 1, 2, 3

SCHED_AUTO, SCHED_DP, SCHED_SPLITK, SCHED_STREAMK, SCHED_KSPLIT = 0, 1, 2, 3, 4

OK = 0
ERR_INVALID_ARG = 1
ERR_ALIGNMENT = 2
ERR_UNSUPPORTED_DEVICE = 3
ERR_OOM = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_TOO_LARGE = 7
ERR_CAPTURE = 8

# Entry points and their C signatures (restype, argtypes).
_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
SIGNATURES = {
    "mxgemm_create": (ctypes.c_int, [ctypes.POINTER(_vp)]),
    "mxgemm_destroy": (ctypes.c_int, [_vp]),
    "mxgemm_run": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxgemm_reserve": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64]),
    "mxgemm_repack": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp]),
    "mxgemm_gemm": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "mxgemm_run_host": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxgemm_quantize": (ctypes.c_int, [ctypes.c_int, _i64, _i64, _vp, _vp, _vp, _vp]),
    "mxgemm_set_schedule": (ctypes.c_int, [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mxgemm_set_kchunks": (ctypes.c_int, [_vp, ctypes.c_int]),
    "mxgemm_describe_plan": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, ctypes.c_char_p, ctypes.c_size_t]),
    "mxgemm_describe_plan_for": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, ctypes.c_char_p,
                                                ctypes.c_size_t]),
    "mxgemm_check_device_error": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_int)]),
    "mxgemm_set_wait_limit": (ctypes.c_int, [_vp, ctypes.c_uint64]),
    "mxgemm_debug_inject": (ctypes.c_int, [_vp, ctypes.c_int]),
    "mxgemm_run_fused": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, ctypes.c_int,
                                        _vp, _vp, _vp]),
    "mxgemm_run_quantized": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp,
                                            ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, _vp]),
    "mxgemm_quantize_bf16": (ctypes.c_int, [ctypes.c_int, _i64, _i64, _vp, _vp, _vp, _vp]),
    "mxgemm_run_bf16": (ctypes.c_int, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "mxgemm_run_grouped": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp]),
    "mxgemm_describe_grouped_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, _i64,
                                                    ctypes.c_char_p, ctypes.c_size_t]),
    "mxgemm_run_noalloc": (ctypes.c_int, [ctypes.c_int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxgemm_set_profiling": (ctypes.c_int, [_vp, ctypes.c_int]),
    "mxgemm_last_timing": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
    "mxgemm_set_prefetch_b": (ctypes.c_int, [_vp, ctypes.c_int]),
    "mxgemm_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mxgemm_version": (ctypes.c_char_p, []),
}

_lib = None


class MXGemmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError("libmxgemm.so not found at %s: run `python -m microscaling_block_scaled_b200.build`"
                               % path)
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().mxgemm_status_string(status).decode()


def version() -> str:
    return load().mxgemm_version().decode()


def _check(fn: str, status: int) -> None:
    if status != OK:
        raise MXGemmError(fn, status)


def row_bytes(fmt: int, K: int) -> int:
    return K if fmt == FMT_MXFP8 else (K // 2 if fmt == FMT_MXFP4 else 2 * K)


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return int(t.data_ptr())


# ------------------------------------------------------------- raw calls

def mxgemm_create() -> int:
    h = _vp()
    _check("mxgemm_create", load().mxgemm_create(ctypes.byref(h)))
    return h.value


def mxgemm_destroy(h: int) -> None:
    _check("mxgemm_destroy", load().mxgemm_destroy(h))


def mxgemm_run(h, fmt, M, N, K, A, SA, B, SB, C, stream) -> int:
    return load().mxgemm_run(h, fmt, M, N, K, A, SA, B, SB, C, stream)


def mxgemm_reserve(h, fmt, M, N, K) -> int:
    return load().mxgemm_reserve(h, fmt, M, N, K)


def mxgemm_repack(h, fmt, M, N, K, SA, SB, stream) -> int:
    return load().mxgemm_repack(h, fmt, M, N, K, SA, SB, stream)


def mxgemm_gemm(h, fmt, M, N, K, A, B, C, stream) -> int:
    return load().mxgemm_gemm(h, fmt, M, N, K, A, B, C, stream)


def mxgemm_run_host(h, fmt, M, N, K, A, SA, B, SB, C, stream) -> int:
    return load().mxgemm_run_host(h, fmt, M, N, K, A, SA, B, SB, C, stream)


def mxgemm_run_noalloc(fmt, M, N, K, A, SA, B, SB, C, stream) -> int:
    return load().mxgemm_run_noalloc(fmt, M, N, K, A, SA, B, SB, C, stream)


def run_noalloc(fmt, A, SA, B, SB, C=None, K=None, stream=None):
    """mxgemm_run_noalloc on torch CUDA tensors (no handle, no device
    allocation inside the library); returns C (bfloat16 [M][N])."""
    import torch
    M, N = A.shape[0], B.shape[0]
    if K is None:
        K = SA.shape[1] * 32
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check("mxgemm_run_noalloc", mxgemm_run_noalloc(fmt, M, N, K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB), _ptr(C),
                                                    _stream_ptr(stream)))
    return C


def mxgemm_run_fused(h, fmt, M, N, K, A, SA, B, SB, bias, act, residual, C, stream) -> int:
    return load().mxgemm_run_fused(h, fmt, M, N, K, A, SA, B, SB, bias, act, residual, C, stream)


def mxgemm_run_quantized(h, fmt, M, N, K, A, SA, B, SB, bias, act, residual, out_fmt, Cq, Cs, stream) -> int:
    return load().mxgemm_run_quantized(h, fmt, M, N, K, A, SA, B, SB, bias, act, residual, out_fmt, Cq, Cs, stream)


def mxgemm_quantize_bf16(fmt, R, K, X, Q, S, stream) -> int:
    return load().mxgemm_quantize_bf16(fmt, R, K, X, Q, S, stream)


def mxgemm_run_bf16(h, M, N, K, A, B, C, stream) -> int:
    return load().mxgemm_run_bf16(h, M, N, K, A, B, C, stream)


def mxgemm_run_grouped(h, fmt, G, M_total, N, K, offsets, A, SA, B, SB, C, stream) -> int:
    return load().mxgemm_run_grouped(h, fmt, G, M_total, N, K, offsets, A, SA, B, SB, C, stream)


def mxgemm_describe_grouped_plan(num_sms, fmt, G, M_total, N, K) -> str:
    buf = ctypes.create_string_buffer(256)
    _check("mxgemm_describe_grouped_plan",
           load().mxgemm_describe_grouped_plan(num_sms, fmt, G, M_total, N, K, buf, 256))
    return buf.value.decode()


def mxgemm_quantize(fmt, R, K, X, Q, S, stream) -> int:
    return load().mxgemm_quantize(fmt, R, K, X, Q, S, stream)


def mxgemm_set_schedule(h, schedule, splits=1, workers=0) -> int:
    return load().mxgemm_set_schedule(h, schedule, splits, workers)


def mxgemm_set_kchunks(h, kc) -> int:
    return load().mxgemm_set_kchunks(h, kc)


def mxgemm_describe_plan(h, fmt, M, N, K) -> str:
    buf = ctypes.create_string_buffer(256)
    _check("mxgemm_describe_plan", load().mxgemm_describe_plan(h, fmt, M, N, K, buf, 256))
    return buf.value.decode()


def mxgemm_describe_plan_for(num_sms, fmt, M, N, K) -> str:
    """The plan text for a device with ``num_sms`` SMs and the automatic
    schedule; needs no handle and no GPU."""
    buf = ctypes.create_string_buffer(256)
    _check("mxgemm_describe_plan_for", load().mxgemm_describe_plan_for(num_sms, fmt, M, N, K, buf, 256))
    return buf.value.decode()


def mxgemm_check_device_error(h) -> tuple[int, int]:
    code = ctypes.c_int(0)
    st = load().mxgemm_check_device_error(h, ctypes.byref(code))
    return st, code.value


def mxgemm_set_wait_limit(h, ns: int) -> int:
    return load().mxgemm_set_wait_limit(h, ns)


def mxgemm_debug_inject(h, mode: int) -> int:
    return load().mxgemm_debug_inject(h, mode)


def mxgemm_set_profiling(h, on: int) -> int:
    return load().mxgemm_set_profiling(h, on)


def mxgemm_set_prefetch_b(h, on: int) -> int:
    return load().mxgemm_set_prefetch_b(h, on)


def mxgemm_last_timing(h) -> tuple[int, float, float]:
    rep, gem = ctypes.c_float(0.0), ctypes.c_float(0.0)
    st = load().mxgemm_last_timing(h, ctypes.byref(rep), ctypes.byref(gem))
    return st, rep.value, gem.value


# ------------------------------------------------------- torch helpers

def quantize(fmt: int, X, stream=None, out=None):
    """OCP MX quantisation of an FP32 CUDA tensor [R][K] on the device.
    Returns (codes uint8 [R][row_bytes], scales uint8 [R][K/32]), written into
    `out` = (codes, scales) when given."""
    import torch
    assert X.is_cuda and X.dtype == torch.float32 and X.is_contiguous()
    R, K = X.shape
    if out is None:
        Q = torch.empty((R, row_bytes(fmt, K)), dtype=torch.uint8, device=X.device)
        S = torch.empty((R, K // 32), dtype=torch.uint8, device=X.device)
    else:
        Q, S = out
    _check("mxgemm_quantize", mxgemm_quantize(fmt, R, K, _ptr(X), _ptr(Q), _ptr(S), _stream_ptr(stream)))
    return Q, S


def quantize_bf16(fmt: int, X, stream=None, out=None):
    """OCP MX quantisation of a BF16 CUDA tensor [R][K] (the activation
    quantiser).  Returns (codes uint8 [R][row_bytes], scales uint8 [R][K/32])."""
    import torch
    assert X.is_cuda and X.dtype == torch.bfloat16 and X.is_contiguous()
    R, K = X.shape
    if out is None:
        Q = torch.empty((R, row_bytes(fmt, K)), dtype=torch.uint8, device=X.device)
        S = torch.empty((R, K // 32), dtype=torch.uint8, device=X.device)
    else:
        Q, S = out
    _check("mxgemm_quantize_bf16", mxgemm_quantize_bf16(fmt, R, K, _ptr(X), _ptr(Q), _ptr(S), _stream_ptr(stream)))
    return Q, S


def _optr(t) -> int:
    return 0 if t is None else _ptr(t)


class Handle:
    """Owns one ``mxgemm_handle`` (workspace, schedule) on the current device."""

    def __init__(self):
        self.h = mxgemm_create()

    def close(self):
        if self.h:
            mxgemm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_schedule(self, schedule: int, splits: int = 1, workers: int = 0):
        _check("mxgemm_set_schedule", mxgemm_set_schedule(self.h, schedule, splits, workers))

    def reserve(self, fmt, M, N, K):
        """Grow the workspace for this shape now (before a stream capture)."""
        _check("mxgemm_reserve", mxgemm_reserve(self.h, fmt, M, N, K))

    def set_kchunks(self, kc: int):
        _check("mxgemm_set_kchunks", mxgemm_set_kchunks(self.h, kc))

    def describe(self, fmt, M, N, K) -> str:
        return mxgemm_describe_plan(self.h, fmt, M, N, K)

    def run(self, fmt, A, SA, B, SB, C=None, K=None, stream=None):
        """C = A * B^T for MX operands on the device; returns C (bfloat16 [M][N])."""
        import torch
        M, N = A.shape[0], B.shape[0]
        if K is None:
            K = SA.shape[1] * 32
        if C is None:
            C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
        _check("mxgemm_run", mxgemm_run(self.h, fmt, M, N, K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB), _ptr(C),
                                        _stream_ptr(stream)))
        return C

    def run_fused(self, fmt, A, SA, B, SB, bias=None, act=ACT_NONE, residual=None, C=None, K=None, stream=None):
        """C = bf16(act(A * B^T + bias) + residual) with the operations in the
        GEMM's epilogue; bias BF16 [N] / residual BF16 [M][N] or None."""
        import torch
        M, N = A.shape[0], B.shape[0]
        if K is None:
            K = SA.shape[1] * 32
        if C is None:
            C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
        _check("mxgemm_run_fused", mxgemm_run_fused(self.h, fmt, M, N, K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB),
                                                    _optr(bias), act, _optr(residual), _ptr(C), _stream_ptr(stream)))
        return C

    def run_quantized(self, fmt, A, SA, B, SB, out_fmt, bias=None, act=ACT_NONE, residual=None, out=None, K=None,
                      stream=None):
        """The fused-epilogue product written as the next layer's MX operand:
        returns (codes uint8 [M][row_bytes(out_fmt, N)], scales uint8 [M][N/32])."""
        import torch
        M, N = A.shape[0], B.shape[0]
        if K is None:
            K = SA.shape[1] * 32
        if out is None:
            Cq = torch.empty((M, row_bytes(out_fmt, N)), dtype=torch.uint8, device=A.device)
            Cs = torch.empty((M, N // 32), dtype=torch.uint8, device=A.device)
        else:
            Cq, Cs = out
        _check("mxgemm_run_quantized",
               mxgemm_run_quantized(self.h, fmt, M, N, K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB), _optr(bias), act,
                                    _optr(residual), out_fmt, _ptr(Cq), _ptr(Cs), _stream_ptr(stream)))
        return Cq, Cs

    def run_bf16(self, A, B, C=None, stream=None):
        """Dense BF16 C = A * B^T (A [M][K], B [N][K] bfloat16 CUDA tensors)."""
        import torch
        M, K = A.shape
        N = B.shape[0]
        if C is None:
            C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
        _check("mxgemm_run_bf16", mxgemm_run_bf16(self.h, M, N, K, _ptr(A), _ptr(B), _ptr(C), _stream_ptr(stream)))
        return C

    def run_grouped(self, fmt, offsets, A, SA, B, SB, C=None, K=None, stream=None):
        """Grouped GEMM: offsets int64 [G+1] CUDA tensor, A [M_total][..], B
        [G][N][..]; C[off[g]:off[g+1]] = A[off[g]:off[g+1]] * B[g]^T.  SA / SB
        are ignored (may be None) for fmt FMT_BF16."""
        import torch
        G = offsets.shape[0] - 1
        M_total = A.shape[0]
        N = B.shape[1]
        if K is None:
            K = SA.shape[1] * 32 if fmt != FMT_BF16 else A.shape[1]
        if C is None:
            C = torch.empty((M_total, N), dtype=torch.bfloat16, device=A.device)
        _check("mxgemm_run_grouped",
               mxgemm_run_grouped(self.h, fmt, G, M_total, N, K, _ptr(offsets), _ptr(A), _optr(SA), _ptr(B),
                                  _optr(SB), _ptr(C), _stream_ptr(stream)))
        return C

    def repack(self, fmt, M, N, K, SA, SB, stream=None):
        _check("mxgemm_repack", mxgemm_repack(self.h, fmt, M, N, K, _ptr(SA), _ptr(SB), _stream_ptr(stream)))

    def gemm(self, fmt, M, N, K, A, B, C, stream=None):
        _check("mxgemm_gemm", mxgemm_gemm(self.h, fmt, M, N, K, _ptr(A), _ptr(B), _ptr(C), _stream_ptr(stream)))

    def run_host(self, fmt, M, N, K, A, SA, B, SB, C, stream=None):
        """Host (CPU, ideally pinned) tensors in, C written to the host tensor ``C``."""
        _check("mxgemm_run_host", mxgemm_run_host(self.h, fmt, M, N, K, _ptr(A), _ptr(SA), _ptr(B), _ptr(SB),
                                                  _ptr(C), _stream_ptr(stream)))

    def check_device_error(self) -> tuple[int, int]:
        return mxgemm_check_device_error(self.h)

    def set_wait_limit(self, ns: int):
        _check("mxgemm_set_wait_limit", mxgemm_set_wait_limit(self.h, ns))

    def debug_inject(self, mode: int):
        _check("mxgemm_debug_inject", mxgemm_debug_inject(self.h, mode))

    def set_profiling(self, on: bool):
        _check("mxgemm_set_profiling", mxgemm_set_profiling(self.h, 1 if on else 0))

    def set_prefetch_b(self, on: bool):
        """Promise that B of later runs is not written by the work queued
        before them (constant weights); see mxgemm_set_prefetch_b."""
        _check("mxgemm_set_prefetch_b", mxgemm_set_prefetch_b(self.h, 1 if on else 0))

    def last_timing(self) -> tuple[float, float]:
        """(repack_ms, gemm_ms) of the last profiled run on this handle."""
        st, rep, gem = mxgemm_last_timing(self.h)
        _check("mxgemm_last_timing", st)
        return rep, gem
