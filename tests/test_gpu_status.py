"""Per-stream device status and captured launches of the ball-attention kernel.

Device-found errors are recorded in a status word of the stream a call was enqueued on, so that callers
on different streams neither see nor clear each other's errors.  The head-pair attention kernel hands
out its work from device counters; a launch captured into a CUDA graph gets a counter pair of its own,
and replays of the graph must give the eager result.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _qkv(n, H, seed):
    return [_bf(t) for t in workloads.random_qkv(n, H, 32, workloads.BF16, seed)]


def test_errors_stay_on_their_stream():
    n, m, H = 4096, 128, 8
    Q, K, V = _qkv(n, H, 3)
    good = torch.randperm(n, generator=torch.Generator().manual_seed(1)).to(torch.int32).cuda()
    bad = good.clone()
    bad[77] = n + 5  # not a row of Q/K/V
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        with torch.cuda.stream(s1):
            bts.bt_ball_attention(Q, K, V, bad, m)
        with torch.cuda.stream(s2):
            bts.bt_ball_attention(Q, K, V, good, m)
    assert bts.bt_last_device_status(s2) == 0
    assert bts.bt_last_device_status(s1) == 8  # BT_ERR_INTERNAL
    assert bts.bt_last_device_status(s1) == 0  # taken and cleared
    assert bts.bt_attention_device_status(s2) == 0  # the earlier name reads the same word


def test_build_error_reaches_the_stream_word():
    # non-finite coordinates on each build shape: the workspace word and the stream word both say so, and a
    # clean build on another stream at the same time reports nothing
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for n, m in [(16384, 128), (65536, 128), (96 * 64, 96)]:
        pts = workloads.uniform_cloud(n, 8)
        pts[n // 2, 1] = np.inf
        c_bad = torch.from_numpy(pts).cuda()
        c_good = torch.from_numpy(workloads.uniform_cloud(n, 9)).cuda()
        ws1, ws2 = bts.workspace([0, n], m), bts.workspace([0, n], m)
        torch.cuda.synchronize()
        with torch.cuda.stream(s1):
            bts.bt_build(c_bad, m, ws=ws1)
        with torch.cuda.stream(s2):
            bts.bt_build(c_good, m, ws=ws2)
        assert bts.bt_last_device_status(s2) == 0
        assert bts.bt_last_device_status(s1) == 3  # BT_ERR_NONFINITE
        assert bts.bt_build_device_status(ws1, s1) == 3
        assert bts.bt_last_device_status(s1) == 0


def test_captured_attention_replays_equal_eager():
    n, m, H = 16384, 128, 8
    Q, K, V = _qkv(n, H, 4)
    Q2, K2, V2 = _qkv(n, H, 5)
    perm = bts.bt_build(torch.from_numpy(workloads.uniform_cloud(n, 6)).cuda(), m)
    want = bts.bt_ball_attention(Q, K, V, perm, m)
    want2 = bts.bt_ball_attention(Q2, K2, V2, perm, m)
    out, out2 = torch.zeros_like(Q), torch.zeros_like(Q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        bts.bt_ball_attention(Q, K, V, perm, m, out=out)
    with torch.cuda.graph(g2, stream=s):
        bts.bt_ball_attention(Q2, K2, V2, perm, m, out=out2)
    for _ in range(3):
        out.zero_()
        out2.zero_()
        g.replay()
        g2.replay()
        # eager launches in between take eager counter pairs
        bts.bt_ball_attention(Q, K, V, perm, m)
        torch.cuda.synchronize()
        assert torch.equal(out, want) and torch.equal(out2, want2)
    assert bts.bt_last_device_status(s) == 0
