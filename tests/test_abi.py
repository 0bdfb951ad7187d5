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
