"""GPU parity of the coarser tree levels against the float64 oracle.

Pooling accumulates in float32 and rounds to the tensor's dtype: float32 is
compared at 1e-5 (relative to the value's scale), bf16 at one bf16 rounding
(2^-8 relative).  The coarse slot map and unpooling (a copy) are bit-exact.
Coarse-level attention follows the ball attention tolerances: 1e-4 for
float32, 2e-2 for bf16 (max abs) and, for bf16, a max-abs error of at most 0.08 of the
output RMS.  At stride 1 the coarse path must give the
fine ball attention bit for bit (same rows, same order, same kernel).
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")

REL_BF16 = 0.08  # max-abs error at most this share of the output RMS (the ball attention tests' bound)


def _check_attention(got, want, bf16):
    err, rms = np.abs(got - want).max(), np.sqrt((np.asarray(want, np.float64) ** 2).mean())
    print(f"parity: max_abs {err:.3e} rms {rms:.3e} max_abs/rms {err / rms:.3e}")
    assert err <= (2e-2 if bf16 else 1e-4), f"max abs err {err}"
    if bf16:
        assert err / rms <= REL_BF16, f"max abs err {err} is {err / rms:.3f} of the output rms {rms}"


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf(a):
    return _dev(a.view(np.int16)).view(torch.bfloat16)


def _host(t):
    if t.dtype == torch.bfloat16:
        return workloads.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def _tree(sizes, leaf, seed):
    pts = np.concatenate([workloads.uniform_cloud(s, seed + i) for i, s in enumerate(sizes)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    perm, _ = bts.bt_build_segmented(_dev(pts), offsets, leaf)
    return pts, perm


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("C", [256, 5, 24])
@pytest.mark.parametrize("stride", [1, 2, 8, 64])
def test_pool_mean_matches_oracle(orc, dtype, C, stride):
    pts, perm = _tree([3000, 411, 1200], 1, 10 + C)
    n = len(pts)
    x = np.random.Generator(np.random.PCG64(C + stride)).standard_normal((n, C)).astype(np.float32)
    if dtype == "bf16":
        xb = workloads.f32_to_bf16_bits(x)
        xd, xo = _bf(xb), xb
    else:
        xd, xo = _dev(x), x
    xc, cperm = bts.bt_pool_mean(xd, perm, stride)
    want, wperm = orc.pool_mean(xo, perm.cpu().numpy(), stride)
    assert bts.bt_last_device_status() == 0
    assert np.array_equal(cperm.cpu().numpy(), wperm)
    got = _host(xc)
    tol = 2.0 ** -8 if dtype == "bf16" else 1e-5
    assert np.all(np.abs(got - want) <= tol * np.maximum(np.abs(want), 1e-3) + 1e-6)


@pytest.mark.parametrize("dtype,C", [("f32", 64), ("bf16", 256), ("bf16", 3), ("f32", 7)])
@pytest.mark.parametrize("stride", [1, 4, 32])
def test_unpool_is_the_copy(orc, dtype, C, stride):
    pts, perm = _tree([2000, 900], 1, 20)
    npad, n = perm.numel(), len(pts)
    xc = np.random.Generator(np.random.PCG64(stride)).standard_normal((npad // stride, C)).astype(np.float32)
    if dtype == "bf16":
        xb = workloads.f32_to_bf16_bits(xc)
        xcd = _bf(xb)
        out = torch.full((n, C), 7.0, dtype=torch.bfloat16, device="cuda")
        src = workloads.bf16_bits_to_f32(xb).astype(np.float64)
    else:
        xcd = _dev(xc)
        out = torch.full((n, C), 7.0, dtype=torch.float32, device="cuda")
        src = xc.astype(np.float64)
    bts.bt_unpool(xcd, perm, stride, out)
    want = orc.unpool(src, perm.cpu().numpy(), stride, n)
    assert np.array_equal(_host(out), want)


def _qkv(n, H, d, dtype, seed):
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16 if dtype == "bf16" else workloads.F32, seed)
    dev = (_bf(q), _bf(k), _bf(v)) if dtype == "bf16" else (_dev(q), _dev(k), _dev(v))
    return (q, k, v), dev


@pytest.mark.parametrize("sizes,leaf,m,stride,H,d,dtype", [
    ([8192], 1, 128, 2, 2, 32, "bf16"),      # pair kernel at the coarse level
    ([8192], 1, 128, 4, 3, 32, "bf16"),      # odd H: general tensor-core kernel
    ([5000, 2100], 1, 32, 8, 2, 64, "bf16"),
    ([3000, 700], 2, 16, 2, 2, 32, "f32"),   # CUDA-core path
    ([4096], 4, 64, 16, 1, 32, "f32"),
])
def test_coarse_ball_attention_matches_oracle(orc, sizes, leaf, m, stride, H, d, dtype):
    pts, perm = _tree(sizes, leaf, 30 + stride)
    (q, k, v), (qd, kd, vd) = _qkv(len(pts), H, d, dtype, stride + H)
    got = _host(bts.bt_coarse_ball_attention(qd, kd, vd, perm, m, stride))
    assert bts.bt_last_device_status() == 0
    want = orc.coarse_ball_attention(q, k, v, m, perm.cpu().numpy(), stride)
    _check_attention(got, want, dtype == "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_stride_one_is_the_fine_ball_attention(dtype):
    pts, perm = _tree([4000, 3000], 1, 40)
    _, (qd, kd, vd) = _qkv(len(pts), 2, 32, dtype, 41)
    m = 128 if dtype == "bf16" else 32
    fine = bts.bt_ball_attention(qd, kd, vd, perm, m)
    coarse = bts.bt_coarse_ball_attention(qd, kd, vd, perm, m, 1)
    assert torch.equal(fine, coarse)


def test_gauss_mix_full_size_sampled_coarse_balls(orc):
    # the 4 x 16384 workload, tree of leaf size 1, attention two levels up (stride 4, balls of 128 nodes)
    wl = workloads.gauss_mix()
    L = wl.layers[0]
    perm, _ = bts.bt_build_segmented(_dev(wl.coords), wl.offsets, 1)
    got = _host(bts.bt_coarse_ball_attention(_bf(L.q), _bf(L.k), _bf(L.v), perm, 128, 4))
    p = perm.cpu().numpy()
    pooled = [orc.pool_mean(t, p, 4) for t in (L.q, L.k, L.v)]
    cperm = pooled[0][1]
    balls = np.random.Generator(np.random.PCG64(5)).choice(len(cperm) // 128, 10, replace=False)
    oc = orc.ball_attention(pooled[0][0], pooled[1][0], pooled[2][0], 128, cperm, balls=balls)
    want = orc.unpool(oc, p, 4, len(wl.coords))
    slots = np.concatenate([np.arange(b * 512, (b + 1) * 512) for b in balls])
    rows = p[slots][p[slots] >= 0]
    _check_attention(got[rows], want[rows], True)
