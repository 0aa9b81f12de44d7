"""Ball attention captured after the library's captured-launch counter pairs are used up.

Each launch of the head-pair kernel captured into a CUDA graph keeps a counter pair of its own (4,096 per
device); later captured launches run on a fixed schedule without counters.  This test captures more
launches than that, so every capture after it in this process takes the fixed schedule: it is collected
late on purpose.  The fixed schedule must give the eager result.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")

CAPTURED_PAIRS = 4096


def test_fixed_schedule_after_captured_pairs_run_out():
    n, m, H = 8192, 128, 4
    q, k, v = workloads.random_qkv(n, H, 32, workloads.BF16, 21)
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(t).view(np.int16)).cuda().view(torch.bfloat16)
               for t in (q, k, v))
    perm = bts.bt_build(torch.from_numpy(workloads.uniform_cloud(n, 22)).cuda(), m)
    want = bts.bt_ball_attention(Q, K, V, perm, m)
    out = torch.zeros_like(Q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    for _ in range(CAPTURED_PAIRS + 2):  # the last captures have no counters left
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            bts.bt_ball_attention(Q, K, V, perm, m, out=out)
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, want)
