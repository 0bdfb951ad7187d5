"""CPU checks of the C-ABI library: it builds, loads without a GPU, and
exports every function include/sqint8.h declares."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from w8a8_int8_quantized_sq_b200 import build as sq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sqint8.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(",
                                 src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(sq_build.build())


def test_header_declares_the_four_layer_calls():
    names = declared_functions()
    for n in ("sq_quant_per_token", "w8a8_scaled_mm", "w8a8_gs128_mm", "w8a16_mm"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_exports(lib):
    import w8a8_int8_quantized_sq_b200 as sq
    assert set(sq.EXPORTS) == set(declared_functions())


def test_shape_and_null_checks_without_gpu(lib):
    # argument checks run before any CUDA call
    lib.w8a8_scaled_mm.restype = ctypes.c_int
    lib.w8a8_scaled_mm.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 3 + [
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert lib.w8a8_scaled_mm(None, None, None, None, None, 4, 32, 200, None, 0, None) == 2
    assert lib.w8a8_scaled_mm(None, None, None, None, None, 4, 24, 256, None, 0, None) == 2
    assert lib.w8a8_scaled_mm(None, None, None, None, None, 4, 32, 256, None, 0, None) == 1
    assert lib.w8a8_scaled_mm(None, None, None, None, None, 0, 32, 256, None, 0, None) == 0
    lib.sq_status_string.restype = ctypes.c_char_p
    lib.sq_status_string.argtypes = [ctypes.c_int]
    assert lib.sq_status_string(6) == b"kernel wait timed out"


def _sig(lib, name, nargs_ptr, nargs_i64, tail):
    f = getattr(lib, name)
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * nargs_ptr + [ctypes.c_int64] * nargs_i64 + tail
    return f


def test_next_rows_argument_checks_without_gpu(lib):
    """Shape, null and alignment checks of the next rows' entry points run
    before any CUDA call (status codes: 1 null, 2 shape, 3 alignment)."""
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    bad = ctypes.c_void_p(0x1001)      # not 16-byte aligned
    ok = ctypes.c_void_p(0x100000)     # aligned (never dereferenced: checks fail first)

    rms = lib.sq_rmsnorm_quant
    rms.restype = ctypes.c_int
    rms.argtypes = [vp, vp, ctypes.c_float, i64, vp, vp, vp, i64, i64, vp]
    assert rms(ok, ok, 1e-6, 0, ok, ok, None, 4, 200, None) == 2        # K % 128
    assert rms(ok, ok, 1e-6, 0, ok, ok, None, 4, 24576 + 128, None) == 2  # K > 24576
    assert rms(ok, ok, 0.0, 0, ok, ok, None, 4, 256, None) == 2         # eps <= 0
    assert rms(ok, ok, 1e-6, 64, ok, ok, None, 4, 256, None) == 2       # group 64
    assert rms(ok, ok, 1e-6, 0, ok, ok, None, 0, 256, None) == 0        # M = 0: no-op
    assert rms(None, ok, 1e-6, 0, ok, ok, None, 4, 256, None) == 1
    assert rms(bad, ok, 1e-6, 0, ok, ok, None, 4, 256, None) == 3

    for name in ("sq_quant_per_group", "sq_quant_fp8_per_group"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [vp, vp, vp, vp, i64, i64, vp]
        assert f(ok, None, ok, ok, 4, 200, None) == 2
        assert f(ok, None, ok, ok, 0, 256, None) == 0
        assert f(None, None, ok, ok, 4, 256, None) == 1
        assert f(ok, bad, ok, ok, 4, 256, None) == 3

    fb = lib.sq_quant_fp8_block
    fb.restype = ctypes.c_int
    fb.argtypes = [vp, vp, vp, vp, i64, i64, vp]
    assert fb(ok, None, ok, ok, 200, 256, None) == 2     # N % 128
    assert fb(ok, None, ok, ok, 0, 256, None) == 0
    assert fb(ok, None, None, ok, 128, 256, None) == 1

    for name in ("w8a8_pg128_mm", "fp8_block_mm"):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = [vp] * 5 + [i64] * 3 + [vp, sz, vp]
        assert f(ok, ok, ok, ok, ok, 4, 128, 200, None, 0, None) == 2   # K % 128
        assert f(ok, ok, ok, ok, ok, 0, 128, 256, None, 0, None) == 0
        assert f(None, ok, ok, ok, ok, 4, 128, 256, None, 0, None) == 1
        assert f(ok, bad, ok, ok, ok, 4, 128, 256, None, 0, None) == 3
    fm = lib.fp8_block_mm
    assert fm(ok, ok, ok, ok, ok, 4, 144, 256, None, 0, None) == 2     # N % 128

    wg = lib.w8a16_group_mm
    wg.restype = ctypes.c_int
    wg.argtypes = [vp] * 4 + [i64] * 3 + [vp, sz, vp]
    assert wg(ok, ok, ok, ok, 4, 24, 256, None, 0, None) == 2          # N % 16
    assert wg(ok, ok, ok, ok, 0, 128, 256, None, 0, None) == 0
    assert wg(ok, ok, None, ok, 4, 128, 256, None, 0, None) == 1

    pk = lib.sq_mma_peak
    pk.restype = ctypes.c_int
    pk.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp]
    d = ctypes.c_double()
    assert pk(3, 1024, None, ctypes.byref(d)) == 2      # unknown kind
    assert pk(0, 1, None, ctypes.byref(d)) == 2         # too few MMAs
    assert pk(0, 1024, None, None) == 1

    st = lib.sq_selftest_wait_timeout
    st.restype = ctypes.c_int
    st.argtypes = [i64, vp, vp]
    assert st(0, ok, None) == 2 and st(1000, None, None) == 1
