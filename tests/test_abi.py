"""The C ABI library builds, loads and exports what include/maple_moe.h declares.

These run without a GPU: only argument validation that returns before any
CUDA call is exercised; no kernel is launched.
"""
import ctypes as C
import os
import re
import subprocess

import pytest

import ternary_weight_moe_forward_b200 as tw
from ternary_weight_moe_forward_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "maple_moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(maple_moe_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return tw.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("maple_moe_create", "maple_moe_route", "maple_moe_forward", "maple_moe_destroy",
              "maple_moe_pack_ternary", "maple_moe_stack_forward", "maple_moe_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", tw.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)
    assert set(tw.EXPORTED) <= exported


def test_library_links_no_oracle(lib):
    out = subprocess.run(["nm", "-D", tw.LIB_PATH], capture_output=True, text=True, check=True).stdout
    assert "orc_" not in out
    deps = subprocess.run(["ldd", tw.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in deps


def test_status_strings(lib):
    assert tw.maple_moe_status_string(0) == "ok"
    assert "unsupported" in tw.maple_moe_status_string(tw.MAPLE_ERR_UNSUPPORTED_SHAPE)
    assert tw.maple_moe_status_string(-99) == "unknown status"


def test_argument_errors_before_any_cuda_call(lib):
    assert lib.maple_moe_destroy(None) == tw.MAPLE_OK
    assert lib.maple_moe_expert_path(None, 1, C.byref(C.c_int32())) != tw.MAPLE_OK
    assert lib.maple_moe_create(None, None, None, None) == tw.MAPLE_ERR_INVALID_ARG
    w = tw.maple_moe_weights()
    h = C.c_void_p()
    for shape in ((300, 16, 2, 128), (256, 12, 2, 128), (256, 16, 0, 128), (256, 16, 2, 100), (256, 16, 33, 128),
                  (256, 2048, 2, 128)):
        cfg = tw.maple_moe_config(*shape, 8, 0, 0)
        assert lib.maple_moe_create(C.byref(cfg), C.byref(w), None, C.byref(h)) == tw.MAPLE_ERR_UNSUPPORTED_SHAPE
    cfg = tw.maple_moe_config(256, 16, 2, 128, 0, 0, 0)
    assert lib.maple_moe_create(C.byref(cfg), C.byref(w), None, C.byref(h)) == tw.MAPLE_ERR_UNSUPPORTED_SHAPE
    cfg = tw.maple_moe_config(256, 16, 2, 128, 8, 0, 0)
    assert lib.maple_moe_create(C.byref(cfg), C.byref(w), None, C.byref(h)) == tw.MAPLE_ERR_INVALID_ARG  # NULL weights
    cfg = tw.maple_moe_config(256, 16, 2, 128, 8, 65, 0)   # decode kernel serves at most 64 tokens
    assert lib.maple_moe_create(C.byref(cfg), C.byref(w), None, C.byref(h)) == tw.MAPLE_ERR_UNSUPPORTED_SHAPE
    for flags in (0x80, tw.MAPLE_CFG_FORCE_TC | tw.MAPLE_CFG_DECODE_ONLY):   # unknown, conflicting
        cfg = tw.maple_moe_config(256, 16, 2, 128, 8, 0, flags)
        assert lib.maple_moe_create(C.byref(cfg), C.byref(w), None, C.byref(h)) == tw.MAPLE_ERR_INVALID_ARG
    assert lib.maple_moe_forward(None, None, 1, None, None, None) == tw.MAPLE_ERR_INVALID_ARG
    assert lib.maple_moe_route(None, None, 1, None, None, None, None) == tw.MAPLE_ERR_INVALID_ARG
    assert lib.maple_moe_pack_ternary(None, 4, 15, None, None, None) == tw.MAPLE_ERR_INVALID_ARG
    assert lib.maple_moe_pack_ternary(None, 0, 16, None, None, None) == tw.MAPLE_OK
    assert lib.maple_moe_stack_forward(None, 1, None, 1, None) == tw.MAPLE_ERR_INVALID_ARG
    f = C.c_uint32()
    assert lib.maple_moe_device_flags(None, C.byref(f), 0) == tw.MAPLE_ERR_INVALID_ARG


def test_bad_handle_is_rejected(lib):
    junk = (C.c_uint32 * 64)()
    assert lib.maple_moe_forward(C.addressof(junk), None, 1, None, None, None) == tw.MAPLE_ERR_INVALID_ARG
    assert lib.maple_moe_destroy(C.addressof(junk)) == tw.MAPLE_ERR_INVALID_ARG
