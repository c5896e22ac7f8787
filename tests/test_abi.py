"""The C-ABI library loads and exports every function include/spot.h declares
(no compute calls: runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spot.h")


def declared_functions(path=HEADER):
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spot_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_long_spot_b200 import build
    return ctypes.CDLL(build.build())


def test_header_declares_the_path_entry_points():
    names = declared_functions()
    for n in ("spot_append_selector_keys", "spot_select", "spot_sparse_decode",
              "spot_decode_step", "spot_workspace_size", "spot_read_device_status",
              "spot_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.spot_status_string.restype = ctypes.c_char_p
    assert lib.spot_status_string(0) == b"ok"
    assert lib.spot_status_string(3) == b"workspace too small"
    assert lib.spot_status_string(99) == b"unknown status"


def test_host_validation_without_device(lib):
    # Argument errors are caught on the host before any CUDA call.
    import block_sparse_long_spot_b200 as spot
    L = spot.lib()
    desc = spot.layer_desc(32, 8, 16)
    prm = spot.select_params()
    P = ctypes.c_void_p
    # null desc
    assert L.spot_select(None, ctypes.byref(prm), *([None] * 5), 64, *([None] * 2), 1,
                         None, None, 64, None, 0, None) == 1
    # unsupported head_dim
    bad = spot.layer_desc(32, 8, 16, head_dim=96)
    assert L.spot_select(ctypes.byref(bad), ctypes.byref(prm), *([None] * 5), 64,
                         *([None] * 2), 1, None, None, 64, None, 0, None) == 2
    # group too large (16 query heads per KV head)
    bad = spot.layer_desc(32, 2, 16)
    assert L.spot_sparse_decode(ctypes.byref(bad), *([None] * 4), 64, None, None, None, 64, 1,
                                0.1, None, None, None, 0, None) == 2
    # batch 0 is a no-op
    assert L.spot_sparse_decode(ctypes.byref(desc), *([None] * 4), 64, None, None, None, 64, 0,
                                0.1, None, None, None, 0, None) == 0
    # bad temperature
    prm_bad = spot.select_params(temperature=0.0)
    q = P(256)
    assert L.spot_select(ctypes.byref(desc), ctypes.byref(prm_bad), q, None, q, None, q, 64, q, q,
                         1, q, q, 64, q, 1 << 20, None) == 1
    # misaligned pointer
    assert L.spot_select(ctypes.byref(desc), ctypes.byref(prm), P(258), None, q, None, q, 64, q,
                         q, 1, q, q, 64, q, 1 << 20, None) == 1
