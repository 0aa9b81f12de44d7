"""GPU parity of ball attention against the float64 oracle.

Tolerances (max-abs): 1e-4 for float32 inputs, 2e-2 for bfloat16 inputs and
outputs.  The outputs' RMS is well below 1 (V ~ N(0,1) averaged over up to
128 keys gives about 0.15), so every bf16 comparison also bounds
max_abs / RMS(O_oracle) by REL_BF16 = 0.08.  Derivation: the bf16 path rounds
each weight P to bf16 (relative error at most 2^-9) and each output to bf16
(at most 2^-9 of |O|); with |V| at most about 4.5 inside a ball and |O| below
1 that is at most 2^-9 * 4.5 + 2^-9 = 0.011 absolute, 0.077 of an RMS of
0.143.  Measured: about 0.02 on a few thousand outputs, 0.05 at the tail of
the 16.7 million outputs of the full 65,536-point layer.  The ratio of every
comparison is printed.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")

TOL = {workloads.F32: 1e-4, workloads.BF16: 2e-2}
REL_BF16 = 0.08


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _qkv_dev(q, k, v, dtype):
    if dtype == workloads.BF16:
        return [_dev(t.view(np.int16)).view(torch.bfloat16) for t in (q, k, v)]
    return [_dev(t) for t in (q, k, v)]


def _out_np(o):
    if o.dtype == torch.bfloat16:
        return o.float().cpu().numpy().astype(np.float64)
    return o.cpu().numpy().astype(np.float64)


def _compare(orc, q, k, v, m, perm, dtype, balls=None):
    Q, K, V = _qkv_dev(q, k, v, dtype)
    o = bts.bt_ball_attention(Q, K, V, None if perm is None else _dev(perm), m,
                              npad=None if perm is None else len(perm))
    assert bts.bt_last_device_status() == 0
    got = _out_np(o)
    want = orc.ball_attention(q, k, v, m, perm, balls=balls)
    if balls is not None:
        slots = np.concatenate([np.arange(b * m, (b + 1) * m) for b in balls])
        rows = slots if perm is None else perm[slots]
        rows = rows[rows >= 0]
        got, want = got[rows], want[rows]
    return _check(got, want, dtype)


def _check(got, want, dtype):
    err = np.abs(got - want).max()
    rms = np.sqrt((want ** 2).mean())
    print(f"parity: max_abs {err:.3e} rms {rms:.3e} max_abs/rms {err / rms:.3e}")
    assert err <= TOL[dtype], f"max abs err {err} (rms {rms})"
    if dtype == workloads.BF16:
        assert err / rms <= REL_BF16, f"max abs err {err} is {err / rms:.3f} of the output rms {rms}"
    return err, rms


def test_tiny_fp32(orc):
    wl = workloads.tiny()
    perm = bts.bt_build(_dev(wl.coords), wl.m).cpu().numpy()
    L = wl.layers[0]
    _compare(orc, L.q, L.k, L.v, wl.m, perm, workloads.F32)


@pytest.mark.parametrize("m,d,H", [(128, 32, 8), (128, 64, 2), (64, 32, 3), (32, 64, 2), (16, 32, 4)])
def test_tensor_core_path(orc, m, d, H):
    n = m * 64
    pts = workloads.uniform_cloud(n, m + d)
    perm = bts.bt_build(_dev(pts), m).cpu().numpy()
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, m * d + H)
    _compare(orc, q, k, v, m, perm, workloads.BF16)


@pytest.mark.parametrize("m,d", [(128, 32), (32, 64)])
def test_tensor_core_identity_order(orc, m, d):
    n, H = m * 40, 2
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 77)
    _compare(orc, q, k, v, m, None, workloads.BF16)


def test_tensor_core_partial_tile(orc):
    # m = 32 with 3 balls: one 128-slot tile, its last 32 slots beyond npad
    n, m, H, d = 96, 32, 2, 32
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 5)
    _compare(orc, q, k, v, m, None, workloads.BF16)


@pytest.mark.parametrize("m,d,dtype", [(8, 32, workloads.BF16), (256, 32, workloads.BF16), (100, 64, workloads.BF16),
                                       (1, 32, workloads.F32), (256, 64, workloads.F32), (32, 32, workloads.F32)])
def test_cuda_core_path(orc, m, d, dtype):
    n, H = m * 16, 2
    q, k, v = workloads.random_qkv(n, H, d, dtype, m + d)
    g = np.random.Generator(np.random.PCG64(m))
    perm = g.permutation(n).astype(np.int32)
    _compare(orc, q, k, v, m, perm, dtype)


def test_masked_ragged(orc):
    wl = workloads.ragged(batch=4, n_min=200, n_max=5000)
    perm, _ = bts.bt_build_segmented(_dev(wl.coords), wl.offsets, wl.m)
    perm = perm.cpu().numpy()
    assert (perm < 0).any()
    L = wl.layers[0]
    _compare(orc, L.q, L.k, L.v, wl.m, perm, workloads.BF16)
    # the same with a cuda-core ball size
    perm16, _ = bts.bt_build_segmented(_dev(wl.coords), wl.offsets, 8)
    _compare(orc, L.q, L.k, L.v, 8, perm16.cpu().numpy(), workloads.BF16)


def test_all_dummy_ball_writes_nothing(orc):
    # balls with 2 real points, 1 real point and none; row 131 is named by no slot and must stay untouched
    n, m, H, d = 132, 128, 2, 32
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 9)
    perm = np.full(512, -1, np.int32)
    perm[:130] = np.arange(130)
    perm[256] = 130
    Q, K, V = _qkv_dev(q, k, v, workloads.BF16)
    out = torch.full_like(Q, 7.0)
    bts.bt_ball_attention(Q, K, V, _dev(perm), m, out=out)
    got = _out_np(out)
    want = orc.ball_attention(q, k, v, m, perm)
    assert np.abs(got[:131] - want[:131]).max() <= 2e-2
    assert np.all(got[131] == 7.0)


def test_gauss_mix_layers(orc):
    wl = workloads.gauss_mix()
    c = _dev(wl.coords)
    for L in wl.layers:
        cc = bts.bt_rotate_z(c) if L.rotated else c
        perm, _ = bts.bt_build_segmented(cc, wl.offsets, wl.m)
        perm = perm.cpu().numpy()
        balls = np.random.Generator(np.random.PCG64(1)).choice(len(perm) // wl.m, 48, replace=False)
        _compare(orc, L.q, L.k, L.v, wl.m, perm, workloads.BF16, balls=balls)


def test_box_cluster_full_size_sampled(orc):
    wl = workloads.box_cluster()
    L = wl.layers[1]
    rot = bts.bt_rotate_z(_dev(wl.coords))
    perm = bts.bt_build(rot, wl.m).cpu().numpy()
    balls = np.random.Generator(np.random.PCG64(2)).choice(len(perm) // wl.m, 32, replace=False)
    _compare(orc, L.q, L.k, L.v, wl.m, perm, workloads.BF16, balls=balls)


def test_m_equals_n_is_full_attention(orc):
    # one ball holding every point is plain softmax attention over all rows
    n, H, d = 128, 2, 32
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 31)
    Q, K, V = _qkv_dev(q, k, v, workloads.BF16)
    o = _out_np(bts.bt_ball_attention(Q, K, V, None, n))
    assert np.abs(o - orc.full_attention(q, k, v)).max() <= 2e-2


def test_m1_is_v():
    n, H, d = 64, 2, 32
    q, k, v = workloads.random_qkv(n, H, d, workloads.F32, 2)
    Q, K, V = _qkv_dev(q, k, v, workloads.F32)
    o = bts.bt_ball_attention(Q, K, V, None, 1).cpu().numpy()
    assert np.array_equal(o, v)


def test_ragged_full_size_sampled(orc):
    """The full 8-cloud ragged batch: masked attention on sampled balls, the partly and fully dummy balls at the
    end of every cloud among them, and rows named by no slot left untouched."""
    wl = workloads.ragged()
    L = wl.layers[0]
    n = wl.n_total
    perm_t, pad = bts.bt_build_segmented(_dev(wl.coords), wl.offsets, wl.m)
    perm = perm_t.cpu().numpy()
    sizes = np.diff(pad)
    assert sizes.max() > 32768, "a cloud beyond the one-launch build's 32,768 slots"
    # 64 extra rows that no slot names: the kernel must leave them as they are
    extra = 64
    q, k, v = workloads.random_qkv(n + extra, L.q.shape[1], L.q.shape[2], workloads.BF16, 4242)
    q[:n], k[:n], v[:n] = L.q, L.k, L.v
    Q, K, V = _qkv_dev(q, k, v, workloads.BF16)
    out = torch.full_like(Q, 7.0)
    bts.bt_ball_attention(Q, K, V, perm_t, wl.m, out=out)
    assert bts.bt_last_device_status() == 0
    got = _out_np(out)
    assert np.all(got[n:] == 7.0)
    nb = len(perm) // wl.m
    real = (perm.reshape(nb, wl.m) >= 0).sum(1)
    partial = np.nonzero((real > 0) & (real < wl.m))[0]
    assert (real == 0).any() and partial.size >= 8  # every cloud's padding: some balls wholly dummy
    rng = np.random.Generator(np.random.PCG64(5))
    big = int(np.argmax(sizes))
    big_balls = np.arange(pad[big] // wl.m, pad[big + 1] // wl.m)
    balls = np.unique(np.concatenate([partial, rng.choice(big_balls, 24, replace=False),
                                      rng.choice(np.nonzero(real == wl.m)[0], 40, replace=False)]))
    want = orc.ball_attention(q, k, v, wl.m, perm, balls=balls)
    slots = np.concatenate([np.arange(b * wl.m, (b + 1) * wl.m) for b in balls])
    rows = perm[slots]
    rows = rows[rows >= 0]
    _check(got[rows], want[rows], workloads.BF16)
    # a row is written exactly once: every real row's output is finite
    assert np.isfinite(got[:n]).all()


def test_ellipsoid_full_size(orc):
    """The single 65,536-point ellipsoid cloud: plain ball attention over its tree, every output compared."""
    wl = workloads.ellipsoid()
    L = wl.layers[0]
    perm = bts.bt_build(_dev(wl.coords), wl.m).cpu().numpy()
    _compare(orc, L.q, L.k, L.v, wl.m, perm, workloads.BF16)
