"""CPU checks of the C ABI: the library loads, exports every entry point bts.h declares, and the host-only
calls (workspace sizing, argument validation before any launch) behave as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "bts.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:bt|bsa)_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from ball_tree_sparse_b200 import build
    return ctypes.CDLL(build.build())


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n


def test_binding_covers_the_header():
    import ball_tree_sparse_b200 as b
    assert sorted(b.EXPORTED) == _declared()
    for n in _declared():
        assert callable(getattr(b, n)), n


def test_workspace_size_host_only():
    import ball_tree_sparse_b200 as b
    s1 = b.bt_build_workspace_size([0, 1024], 32)
    s2 = b.bt_build_workspace_size([0, 1 << 20], 128)
    assert 0 < s1 < s2
    assert b.bt_build_workspace_size([0, 0], 32) == 0        # empty cloud
    assert b.bt_build_workspace_size([0, 10], 0) == 0        # m < 1
    assert b.bt_build_workspace_size([0, 10], 2048) == 0     # m too large
    assert b.bt_build_workspace_size(list(range(66)), 1) == 0  # more than 64 clouds
    # a batch needs at least the sum of its clouds' key and list arrays
    off = np.cumsum([0, 300, 5000, 7])
    assert b.bt_build_workspace_size(off, 16) >= 4 * 4 * (512 + 8192 + 16)


def test_argument_errors_before_any_launch(lib):
    # NULL pointers and bad shapes return without touching the device (no GPU here)
    P = ctypes.c_void_p
    lib.bt_build.argtypes = [P, ctypes.c_int64, ctypes.c_int32, P, P, ctypes.c_size_t, P]
    assert lib.bt_build(None, 1024, 32, None, None, 0, None) == 1          # BT_ERR_ARG
    lib.bt_ball_attention.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int, P, P]
    one = ctypes.c_void_p(16)
    assert lib.bt_ball_attention(one, one, one, None, 128, 128, 32, 2, 48, 1, one, None) == 2  # d = 48
    assert lib.bt_ball_attention(one, one, one, None, 100, 100, 32, 2, 32, 1, one, None) == 2  # npad % m
    assert lib.bt_ball_attention(one, one, one, None, 128, 64, 32, 2, 32, 1, one, None) == 1  # rows < npad
    lib.bt_gather.argtypes = [P, P, ctypes.c_int64, ctypes.c_int32, P, P]
    assert lib.bt_gather(one, one, 10, 0, one, None) == 1                   # row_bytes < 1
