"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/mxgemm.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from microscaling_block_scaled_b200 import build as mxbuild
from microscaling_block_scaled_b200 import mxgemm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxgemm.h")


@pytest.fixture(scope="module")
def lib():
    mxbuild.build()
    return mxgemm.load()


def declared_names():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MXGEMM_API\s+(?:int|const char \*)\s*(mxgemm_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_names()
    for required in ("mxgemm_create", "mxgemm_run", "mxgemm_destroy", "mxgemm_quantize", "mxgemm_repack",
                     "mxgemm_gemm", "mxgemm_run_host"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_names():
        assert hasattr(lib, name), name
        assert name in mxgemm.SIGNATURES, name


def test_status_strings(lib):
    assert mxgemm.status_string(mxgemm.OK) == "ok"
    assert "bounded wait" in mxgemm.status_string(mxgemm.ERR_TIMEOUT)
    assert mxgemm.status_string(999) == "unknown status"
    assert "capture" in mxgemm.status_string(mxgemm.ERR_CAPTURE)
    assert re.match(r"^\d+\.\d+\.\d+$", mxgemm.version())


def test_run_rejects_null_handle(lib):
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf)
    assert mxgemm.mxgemm_run(None, 0, 1, 1, 128, p, p, p, p, p, None) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_gemm(None, 0, 1, 1, 128, p, p, p, None) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_repack(None, 0, 1, 1, 128, p, p, None) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_set_schedule(None, 0, 1, 0) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_debug_inject(None, 1) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_set_profiling(None, 1) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_set_prefetch_b(None, 1) == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_last_timing(None)[0] == mxgemm.ERR_INVALID_ARG
    assert mxgemm.mxgemm_reserve(None, 0, 1, 1, 128) == mxgemm.ERR_INVALID_ARG


@pytest.mark.parametrize("fmt,R,K,align,expect", [
    (2, 4, 64, 0, mxgemm.ERR_INVALID_ARG),      # unknown format
    (0, 0, 64, 0, mxgemm.ERR_INVALID_ARG),      # empty
    (0, 4, 48, 0, mxgemm.ERR_INVALID_ARG),      # K not a multiple of 32
    (1, 4, 64, 1, mxgemm.ERR_ALIGNMENT),        # misaligned pointer
])
def test_quantize_validates_before_launch(lib, fmt, R, K, align, expect):
    buf = ctypes.create_string_buffer(4096 + 64)
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    X = base + align
    assert mxgemm.mxgemm_quantize(fmt, R, K, X, base + 1024, base + 2048, None) == expect


def test_quantize_rejects_null(lib):
    assert mxgemm.mxgemm_quantize(0, 4, 64, None, None, None, None) == mxgemm.ERR_INVALID_ARG


def test_create_without_gpu_reports_unsupported(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = lib.mxgemm_create(ctypes.byref(h))
    assert st in (mxgemm.ERR_UNSUPPORTED_DEVICE, mxgemm.ERR_CUDA)
    assert not h.value
    assert lib.mxgemm_destroy(None) == mxgemm.OK
