"""The allocation-free build entry point against the workspace one (bit-exact permutations).

bt_build_noalloc serves callers that cannot allocate device memory at build time (inside a CUDA
graph capture region, under a framework that owns all device allocations, on a host with a memory
budget fixed at start-up).  Its scratch is a static array inside the library that every call reuses,
so this test makes two calls in a row, of different inputs, and checks that the second is not
disturbed by what the first left behind.  Collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")


def _noalloc_c(coords, m, perm, status):
    lib = ctypes.CDLL(bts.LIB_PATH)
    f = lib.bt_build_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f(ctypes.c_void_p(coords.data_ptr()), coords.shape[0], m, ctypes.c_void_p(perm.data_ptr()),
             ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_build_twice():
    # Calls in a row on the shared scratch, each checked bit-exact against bt_build:
    #  - two multi-kernel (record-path) builds of 65,536 slots with different inputs and leaf sizes, so the
    #    second runs on the counters, histograms and look-back words the first left behind;
    #  - the index-list path (leaf size 96, not a power of two) after them;
    #  - a one-launch cluster build (16,384 slots), then a multi-kernel build again.
    cases = [(workloads.uniform_cloud(65536, 11), 128),
             (workloads.tied_cloud(65536, 12, levels=5), 64),
             (workloads.uniform_cloud(96 * 2 ** 9, 13, scale=(3.0, 1.0, 0.5)), 96),
             (workloads.uniform_cloud(16384, 14), 128),
             (workloads.tied_cloud(65536, 15, levels=9), 128)]
    for pts, m in cases:
        c = torch.from_numpy(pts).cuda()
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        perm = torch.full((len(pts),), -7, dtype=torch.int32, device="cuda")
        assert _noalloc_c(c, m, perm, status) == 0
        want = bts.bt_build(c, m)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(perm, want), f"{len(pts)} points, m = {m}"


def test_noalloc_rejects_too_many_points():
    c = torch.zeros((131072, 3), device="cuda")
    perm = torch.empty(131072, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc_c(c, 128, perm, status) == 7  # BT_ERR_UNSUPPORTED, nothing enqueued
