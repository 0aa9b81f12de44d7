"""Pins for the oracle's rotation and attention (CPU only).

Rotation: closed forms (unit vectors, composition to 90 and 360 degrees, the
exact rotation in double) rather than a retyped formula.  Attention: the
reductions the method has (m = 1, m = N, constant logits, one dominant key,
masked dummies) and torch's scaled_dot_product_attention in float64 as an
independent library routine, ball by ball.
"""
import math

import numpy as np
import pytest
import torch

import workloads

C45 = np.array([0x3F3504F3], np.uint32).view(np.float32)[0]


def test_rotate_unit_vectors(orc):
    out = orc.rotate_z(np.array([[1, 0, 0], [0, 1, 0], [0, 0, 5], [-2, 0, 1]], np.float32))
    assert out[0].tolist() == [C45, C45, 0.0]
    assert out[1].tolist() == [-C45, C45, 0.0]
    assert out[2].tolist() == [0.0, 0.0, 5.0]
    assert out[3].tolist() == [np.float32(-2) * C45, np.float32(-2) * C45, 1.0]


def test_rotate_against_exact_and_compositions(orc):
    pts = (workloads.uniform_cloud(5000, 11) - 0.5) * 8
    r1 = orc.rotate_z(pts)
    # against the exact rotation in double: a few float ulps of the radius
    x, y = pts[:, 0].astype(np.float64), pts[:, 1].astype(np.float64)
    ex = np.stack([(x - y) * math.sqrt(0.5), (x + y) * math.sqrt(0.5)], 1)
    rad = np.hypot(x, y)
    assert np.all(np.abs(r1[:, :2] - ex).max(axis=1) <= 4 * np.finfo(np.float32).eps * rad + 1e-30)
    assert np.array_equal(r1[:, 2], pts[:, 2])
    # two steps = 90 degrees: (x, y) -> (-y, x)
    r2 = orc.rotate_z(r1)
    assert np.allclose(r2[:, 0], -pts[:, 1], atol=1e-5 * 8) and np.allclose(r2[:, 1], pts[:, 0], atol=1e-5 * 8)
    # eight steps = identity within a few ulps
    r = pts
    for _ in range(8):
        r = orc.rotate_z(r)
    assert np.allclose(r, pts, rtol=0, atol=16 * np.finfo(np.float32).eps * 8)


def _sdpa(q, k, v):
    """torch SDPA in float64 for one ball: q/k/v [n, H, d] -> [n, H, d]."""
    qt, kt, vt = (torch.from_numpy(np.asarray(t, np.float64)).permute(1, 0, 2) for t in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(1, 0, 2).numpy()


def _widen(a):
    return workloads.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


@pytest.mark.parametrize("dtype", [workloads.F32, workloads.BF16])
def test_ball_attention_matches_sdpa_per_ball(orc, dtype):
    n, m, H, d = 512, 32, 3, 16
    pts = workloads.uniform_cloud(n, 2)
    perm, _ = orc.build(pts, m)
    q, k, v = workloads.random_qkv(n, H, d, dtype, 4)
    o = orc.ball_attention(q, k, v, m, perm)
    Q, K, V = _widen(q), _widen(k), _widen(v)
    for b in range(n // m):
        rows = perm[b * m:(b + 1) * m]
        np.testing.assert_allclose(o[rows], _sdpa(Q[rows], K[rows], V[rows]), rtol=1e-12, atol=1e-12)


def test_m1_is_v(orc):
    n, H, d = 64, 2, 8
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 1)
    perm = np.random.Generator(np.random.PCG64(0)).permutation(n).astype(np.int32)
    o = orc.ball_attention(q, k, v, 1, perm)
    assert np.array_equal(o, _widen(v))


def test_m_equals_n_is_full_attention(orc):
    n, H, d = 256, 2, 32
    q, k, v = workloads.random_qkv(n, H, d, workloads.F32, 2)
    perm, _ = orc.build(workloads.uniform_cloud(n, 5), n)
    o = orc.ball_attention(q, k, v, n, perm)
    np.testing.assert_allclose(o, orc.full_attention(q, k, v), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o, _sdpa(q, k, v), rtol=1e-12, atol=1e-13)


def test_zero_keys_give_ball_mean(orc):
    n, m, H, d = 128, 16, 2, 8
    q, _, v = workloads.random_qkv(n, H, d, workloads.F32, 3)
    k = np.zeros_like(q)
    o = orc.ball_attention(q, k, v, m)
    for b in range(n // m):
        np.testing.assert_allclose(o[b * m:(b + 1) * m], np.broadcast_to(v[b * m:(b + 1) * m].astype(np.float64)
                                                                          .mean(0), (m, H, d)), atol=1e-12)


def test_dominant_key_selects_its_value(orc):
    n, m, H, d = 64, 8, 1, 4
    q = np.zeros((n, H, d), np.float32)
    k = np.zeros((n, H, d), np.float32)
    v = workloads.random_qkv(n, H, d, workloads.F32, 9)[2]
    q[:, 0, 0] = 40.0
    k[3::m, 0, 0] = 40.0  # key 3 of every ball: logit 800 vs 0
    o = orc.ball_attention(q, k, v, m)
    for b in range(n // m):
        np.testing.assert_allclose(o[b * m:(b + 1) * m, 0], np.broadcast_to(v[b * m + 3, 0], (m, d)), atol=1e-12)


def test_dummies_are_masked(orc):
    # a padded cloud: dummy slots are neither queries nor keys
    n, m, H, d = 45, 16, 2, 8
    pts = workloads.uniform_cloud(n, 6)
    perm, _ = orc.build(pts, m)
    assert (perm < 0).sum() == 64 - 45
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, 6)
    o = orc.ball_attention(q, k, v, m, perm)
    Q, K, V = _widen(q), _widen(k), _widen(v)
    for b in range(len(perm) // m):
        rows = perm[b * m:(b + 1) * m]
        rows = rows[rows >= 0]
        if len(rows):
            np.testing.assert_allclose(o[rows], _sdpa(Q[rows], K[rows], V[rows]), rtol=1e-12, atol=1e-12)


def test_shuffle_equivariance(orc):
    n, m, H, d = 1024, 32, 2, 16
    pts = workloads.uniform_cloud(n, 21)
    q, k, v = workloads.random_qkv(n, H, d, workloads.F32, 21)
    o = orc.ball_attention(q, k, v, m, orc.build(pts, m)[0])
    sh = np.random.Generator(np.random.PCG64(3)).permutation(n)
    o2 = orc.ball_attention(q[sh], k[sh], v[sh], m, orc.build(pts[sh], m)[0])
    np.testing.assert_allclose(o2, o[sh], rtol=1e-12, atol=1e-13)
