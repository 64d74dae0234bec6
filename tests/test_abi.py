"""The C-ABI library loads and exports every symbol include/slim.h declares;
host-only calls behave as documented (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "slim.h")
LIB = os.path.join(ROOT, "sparse_int4_linear_b200", "libslim.so")


def declared_functions(path):
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(slim_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def clib():
    if not os.path.exists(LIB):
        from sparse_int4_linear_b200 import build
        build.build()
    lib = ctypes.CDLL(LIB)
    lib.slim_layer_bytes.restype = ctypes.c_size_t
    lib.slim_layer_bytes.argtypes = [ctypes.c_int] * 4
    lib.slim_status_string.restype = ctypes.c_char_p
    lib.slim_workspace_bytes.restype = ctypes.c_size_t
    lib.slim_workspace_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int]
    return lib


def test_header_declares_the_expected_calls():
    names = declared_functions(HEADER)
    for must in ["slim_pack", "slim_linear", "slim_layer_bytes", "slim_layer_init", "slim_workspace_bytes",
                 "slim_linear_host", "slim_sync_status", "slim_status_string", "slim_unpack_dec"]:
        assert must in names


def test_every_declared_symbol_is_exported(clib):
    for name in declared_functions(HEADER):
        assert hasattr(clib, name), name


def test_debug_library_exports_the_same_symbols():
    """The index-checking debug build (SLIM_DEBUG) is the same C ABI."""
    dbg = os.path.join(ROOT, "sparse_int4_linear_b200", "libslim_debug.so")
    if not os.path.exists(dbg):
        pytest.skip("libslim_debug.so not built (python -m sparse_int4_linear_b200.build --debug)")
    lib = ctypes.CDLL(dbg)
    for name in declared_functions(HEADER):
        assert hasattr(lib, name), name
    lib.slim_status_string.restype = ctypes.c_char_p
    assert b"debug" in lib.slim_status_string(-10)


def test_layer_bytes_shapes(clib):
    assert clib.slim_layer_bytes(256, 256, 16, 128) > 256 * 256 * 3 // 8
    assert clib.slim_layer_bytes(4096, 4096, 128, 128) >= 4096 * 4096 * 3 // 8 + 4096 * 32 * 2
    # bad shapes -> 0
    assert clib.slim_layer_bytes(100, 256, 16, 128) == 0      # K % 128
    assert clib.slim_layer_bytes(256, 256, 16, 64) == 0       # group
    assert clib.slim_layer_bytes(256, 0, 16, 128) == 0        # N
    assert clib.slim_layer_bytes(256, 256, -1, 128) == 0      # r
    assert clib.slim_layer_bytes(256, 256, 0, 128) > 0        # r = 0 allowed


def test_status_strings(clib):
    for code in range(-10, 1):
        assert clib.slim_status_string(code)
    assert clib.slim_status_string(0) == b"ok"


def test_uninitialised_descriptor_is_rejected_on_host(clib):
    blank = ctypes.create_string_buffer(256)
    clib.slim_linear.restype = ctypes.c_int
    rc = clib.slim_linear(blank, ctypes.c_void_p(16), 1, ctypes.c_void_p(4096), None, ctypes.c_size_t(0), None)
    assert rc == -9
    clib.slim_pack.restype = ctypes.c_int
    assert clib.slim_pack(None, None, None, None, None) == -9
    assert clib.slim_workspace_bytes(None, 4) == 0
    assert clib.slim_abi_version() == 3
    clib.slim_layer_set_adapter_bits.restype = ctypes.c_int
    assert clib.slim_layer_set_adapter_bits(None, 4) == -9
    assert clib.slim_layer_set_adapter_bits(blank, 4) == -9
    clib.slim_unpack_adapters.restype = ctypes.c_int
    assert clib.slim_unpack_adapters(blank, None, None, None, None, None) == -9


def test_grouped_layer_sizes(clib):
    """Grouped layers (several linears on one X): G = 1 is the plain layer; the
    fused adapter factor L grows with G; group row counts other than the last
    must be multiples of 256; at most 8 groups."""
    arr = lambda xs: (ctypes.c_int32 * len(xs))(*xs)
    clib.slim_grouped_layer_bytes.restype = ctypes.c_size_t
    clib.slim_grouped_layer_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                                              ctypes.c_int, ctypes.c_int]
    g = clib.slim_grouped_layer_bytes
    assert g(4096, 1, arr([4096]), 128, 128) == clib.slim_layer_bytes(4096, 4096, 128, 128)
    three = g(4096, 3, arr([4096, 4096, 4096]), 128, 128)
    assert three > clib.slim_layer_bytes(4096, 3 * 4096, 128, 128)      # L and its image are 3x wider
    assert g(4096, 2, arr([11008, 11008]), 128, 128) > 0               # 11008 = 43 x 256
    assert g(4096, 2, arr([1000, 24]), 16, 128) == 0                  # first group not a multiple of 256
    assert g(4096, 2, arr([1024, 24]), 16, 128) > 0                   # the last group may be ragged
    assert g(4096, 9, arr([256] * 9), 16, 128) == 0                   # more than 8 groups
    assert g(4096, 0, arr([256]), 16, 128) == 0
    assert g(4096, 2, arr([256, 0]), 16, 128) == 0
