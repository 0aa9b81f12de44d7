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
    lib.bt_build_segmented_ex.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, P, P, P, ctypes.c_size_t,
                                          ctypes.c_uint32, P]
    offs = (ctypes.c_int64 * 2)(0, 1024)
    assert lib.bt_build_segmented_ex(one, offs, 1, 32, one, None, one, 1 << 30, 2, None) == 1  # unknown flag bit
    assert lib.bt_build_segmented_ex(None, offs, 1, 32, one, None, one, 1 << 30, 1, None) == 1
    lib.bt_gather.argtypes = [P, P, ctypes.c_int64, ctypes.c_int32, P, P]
    assert lib.bt_gather(one, one, 10, 0, one, None) == 1                   # row_bytes < 1
    i64, i32 = ctypes.c_int64, ctypes.c_int32
    lib.bt_pool_mean.argtypes = [P, P, i64, i64, i32, i32, ctypes.c_int, P, P, P]
    assert lib.bt_pool_mean(one, one, 96, 96, 8, 3, 1, one, None, None) == 2   # stride not a power of two
    assert lib.bt_pool_mean(one, one, 96, 96, 8, 64, 1, one, None, None) == 2  # stride does not divide npad
    assert lib.bt_pool_mean(one, None, 128, 100, 8, 2, 1, one, None, None) == 1  # no perm, rows < npad
    assert lib.bt_pool_mean(None, one, 128, 128, 8, 2, 1, one, None, None) == 1
    lib.bt_coarse_workspace_size.argtypes = [i64, i32, i32, i32, ctypes.c_int]
    lib.bt_coarse_workspace_size.restype = ctypes.c_size_t
    assert lib.bt_coarse_workspace_size(1024, 2, 32, 4, 1) >= 4 * 256 * 2 * 32 * 2 + 256 * 4
    assert lib.bt_coarse_workspace_size(1024, 2, 32, 3, 1) == 0
    lib.bt_coarse_ball_attention.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, ctypes.c_int, i32, P, P,
                                             ctypes.c_size_t, P]
    assert lib.bt_coarse_ball_attention(one, one, one, one, 1024, 1024, 128, 2, 32, 1, 16, one, one, 1 << 30,
                                        None) == 2                          # 64 coarse tokens, ball of 128
    assert lib.bt_coarse_ball_attention(one, one, one, one, 1024, 1024, 32, 2, 32, 1, 4, one, None, 0,
                                        None) == 4                          # no workspace


def test_binding_constants_match_the_header():
    # the status names, dtype codes, batch limit and build flags the binding passes through the ABI
    text = open(os.path.join(ROOT, "include", "bts.h")).read()
    enum = dict((k, int(v)) for k, v in re.findall(r"\b(BT_[A-Z_0-9]+)\s*=\s*(\d+)", text))
    defines = dict((k, int(v)) for k, v in re.findall(r"#define\s+(BT_[A-Z_0-9]+)\s+(\d+)u?\b", text))
    b = pytest.importorskip("ball_tree_sparse_b200")
    assert {v: k for k, v in b.STATUS.items()} == {k: v for k, v in enum.items() if k.startswith("BT_OK") or
                                                   k.startswith("BT_ERR_")}
    assert (b.BT_F32, b.BT_BF16) == (enum["BT_F32"], enum["BT_BF16"])
    assert b.MAX_CLOUDS == defines["BT_MAX_CLOUDS"]
    assert b.BT_BUILD_NARROW == defines["BT_BUILD_NARROW"]


def test_projection_calls_check_arguments_before_any_launch(lib):
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    one = ctypes.c_void_p(16)
    lib.bt_qkv_project.argtypes = [P, i64, i32, P, i32, i32, ctypes.c_int, P, P, i64, P, P, P, P]
    assert lib.bt_qkv_project(None, 128, 64, one, 2, 32, 1, None, None, 0, one, one, one, None) == 1  # no X
    assert lib.bt_qkv_project(one, 128, 64, one, 2, 32, 1, one, None, 128, one, one, one, None) == 1  # perm, no inv
    assert lib.bt_qkv_project(one, 128, 0, one, 2, 32, 1, None, None, 0, one, one, one, None) == 1     # C < 1
    assert lib.bt_qkv_project(one, 128, 64, one, 2, 32, 7, None, None, 0, one, one, one, None) == 1    # dtype
    assert lib.bt_qkv_project(one, 128, 64, one, 2048, 32, 1, None, None, 0, one, one, one, None) == 7  # 3Hd too big
    lib.bt_ball_attention_tree.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, ctypes.c_int, P, P]
    assert lib.bt_ball_attention_tree(one, one, one, None, 256, 256, 128, 2, 32, 1, one, None) == 1  # perm required
    assert lib.bt_ball_attention_tree(one, one, one, one, 200, 256, 128, 2, 32, 1, one, None) == 2   # npad % m
    assert lib.bt_ball_attention_tree(one, one, one, one, 256, 256, 128, 2, 64, 1, one, None) == 7   # d = 64
    assert lib.bt_ball_attention_tree(one, one, one, one, 256, 256, 128, 3, 32, 1, one, None) == 7   # odd H
    assert lib.bt_ball_attention_tree(one, one, one, one, 64, 64, 32, 2, 32, 1, one, None) == 7      # npad < 128
    lib.bt_projected_workspace_size.argtypes = [i64, i64, i32, i32, ctypes.c_int]
    lib.bt_projected_workspace_size.restype = ctypes.c_size_t
    ws = lib.bt_projected_workspace_size(1024, 1000, 8, 32, 1)
    assert ws >= 3 * 1024 * 8 * 32 * 2 + 1000 * 4          # Q, K, V in slot order and the inverse slot map
    assert lib.bt_projected_workspace_size(1024, 1000, 8, 32, 5) == 0
    lib.bt_projected_ball_attention.argtypes = [P, P, i64, i64, i32, P, i32, i32, i32, ctypes.c_int, P, P,
                                                ctypes.c_size_t, P]
    assert lib.bt_projected_ball_attention(one, one, 1024, 1000, 64, one, 128, 8, 48, 1, one, one, ws,
                                           None) == 2       # d = 48
    assert lib.bt_projected_ball_attention(one, one, 1024, 1000, 64, one, 128, 8, 32, 1, one, one, ws - 1,
                                           None) == 4       # workspace too small
    assert lib.bt_projected_ball_attention(one, one, 1024, 1000, 64, one, 128, 8, 32, 1, one, ctypes.c_void_p(272),
                                           ws, None) == 1   # workspace not 256-byte aligned
