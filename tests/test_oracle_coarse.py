"""Pins for the oracle's coarser-level ball attention (CPU only).

Coarsening mean-pools each node `stride` consecutive tree slots wide, attention
runs inside balls of m coarse tokens, and refinement copies a node's result
back to its real rows.  Checked against numpy restatements (fancy indexing,
per-node means), the chain rule of nested means, torch SDPA over node means
when one coarse ball covers the cloud, and the stride-1 reduction to plain
ball attention.
"""
import numpy as np
import pytest
import torch

import workloads


def _cloud(sizes, m, seed):
    import oracle
    pts = np.concatenate([workloads.uniform_cloud(s, seed + i) for i, s in enumerate(sizes)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    perm, _ = oracle.build(pts, m, offsets if len(sizes) > 1 else None)
    return pts, perm


def _node_means(x, perm, s):
    """numpy: mean of x over the real slots of each node of s slots; zero and invalid where none"""
    nodes = perm.reshape(-1, s)
    out = np.zeros((len(nodes),) + x.shape[1:])
    valid = np.zeros(len(nodes), bool)
    for j, rows in enumerate(nodes):
        rows = rows[rows >= 0]
        if len(rows):
            out[j] = x[rows].astype(np.float64).mean(0)
            valid[j] = True
    return out, valid


def test_stride_one_is_the_slot_gather(orc):
    pts, perm = _cloud([300, 77], 16, 1)
    x = np.random.Generator(np.random.PCG64(1)).standard_normal((len(pts), 5))
    xc, cperm = orc.pool_mean(x, perm, 1)
    real = perm >= 0
    np.testing.assert_array_equal(xc[real], x[perm[real]])
    np.testing.assert_array_equal(xc[~real], 0.0)
    np.testing.assert_array_equal(cperm, np.where(real, np.arange(len(perm)), -1))


@pytest.mark.parametrize("stride", [2, 4, 16, 64])
def test_pool_is_the_mean_over_real_slots(orc, stride):
    pts, perm = _cloud([1000, 230, 41], 16, 2)
    x = workloads.random_qkv(len(pts), 2, 8, workloads.BF16, 2)[0]
    xc, cperm = orc.pool_mean(x, perm, stride)
    want, valid = _node_means(workloads.bf16_bits_to_f32(x), perm, stride)
    np.testing.assert_allclose(xc, want, rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(cperm, np.where(valid, np.arange(len(valid)), -1))
    if stride <= 16:
        assert (~valid).any()  # the ragged batch has all-dummy nodes at these strides


def test_nested_means_chain_without_dummies(orc):
    pts, perm = _cloud([1024], 16, 3)
    assert (perm >= 0).all()
    x = np.random.Generator(np.random.PCG64(3)).standard_normal((1024, 6))
    x4, _ = orc.pool_mean(x, perm, 4)
    x2, c2 = orc.pool_mean(x, perm, 2)
    x22, _ = orc.pool_mean(x2, c2, 2)
    np.testing.assert_allclose(x22, x4, rtol=1e-13, atol=1e-14)


def test_unpool_copies_the_node_to_its_real_rows(orc):
    pts, perm = _cloud([500, 300], 16, 4)
    rows = len(pts)
    xc = np.random.Generator(np.random.PCG64(4)).standard_normal((len(perm) // 8, 3))
    x = orc.unpool(xc, perm, 8, rows)
    slots = np.nonzero(perm >= 0)[0]
    np.testing.assert_array_equal(x[perm[slots]], xc[slots // 8])
    assert not np.isnan(x).any()  # every row is named by exactly one slot


def test_unpool_after_pool_keeps_node_constant_data(orc):
    pts, perm = _cloud([700, 200], 16, 5)
    xc0 = np.random.Generator(np.random.PCG64(5)).standard_normal((len(perm) // 4, 4))
    x = orc.unpool(xc0, perm, 4, len(pts))
    xc, cperm = orc.pool_mean(x, perm, 4)
    ok = cperm >= 0
    np.testing.assert_allclose(xc[ok], xc0[ok], rtol=1e-15, atol=0)


def test_coarse_attention_stride_one_is_ball_attention(orc):
    pts, perm = _cloud([900, 400], 32, 6)
    q, k, v = workloads.random_qkv(len(pts), 2, 16, workloads.BF16, 6)
    got = orc.coarse_ball_attention(q, k, v, 32, perm, 1)
    want = orc.ball_attention(q, k, v, 32, perm)
    np.testing.assert_array_equal(got, want)


def test_one_coarse_ball_is_sdpa_over_node_means(orc):
    # m * stride == npad: a single ball at the coarse level holds every node
    pts, perm = _cloud([1000], 16, 7)  # npad 1024
    stride, m = 64, 16
    assert m * stride == len(perm)
    q, k, v = workloads.random_qkv(len(pts), 2, 8, workloads.F32, 7)
    got = orc.coarse_ball_attention(q, k, v, m, perm, stride)
    (qm, valid), (km, _), (vm, _) = (_node_means(t, perm, stride) for t in (q, k, v))
    t = [torch.from_numpy(a[valid].transpose(1, 0, 2).copy()) for a in (qm, km, vm)]
    oc = torch.nn.functional.scaled_dot_product_attention(*t).numpy().transpose(1, 0, 2)
    node_of = np.empty(len(pts), np.int64)
    node_of[perm[perm >= 0]] = np.nonzero(perm >= 0)[0] // stride
    idx = np.cumsum(valid) - 1  # node -> position among valid nodes
    np.testing.assert_allclose(got, oc[idx[node_of]], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("m", [4, 16, 128])
def test_leaf_size_one_tree_has_the_same_nodes(orc, m):
    # the split rule above size m does not depend on the leaf size: the nodes of m slots hold the same points,
    # so ball attention on the deeper tree equals ball attention on the leaf-size-m tree
    sizes = [1000, 333, 2048]
    pts = np.concatenate([workloads.uniform_cloud(s, 50 + i) for i, s in enumerate(sizes)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    p1, _ = orc.build(pts, 1, offsets)
    pm, _ = orc.build(pts, m, offsets)
    assert len(p1) == len(pm)
    for b in range(len(pm) // m):
        assert sorted(p1[b * m:(b + 1) * m]) == sorted(pm[b * m:(b + 1) * m])
    q, k, v = workloads.random_qkv(len(pts), 1, 8, workloads.F32, 51)
    np.testing.assert_allclose(orc.ball_attention(q, k, v, m, p1), orc.ball_attention(q, k, v, m, pm),
                               rtol=1e-13, atol=1e-14)


# --- projection of features to Q, K, V (feeds the fused projection + attention path) ---

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_projection_matches_numpy_matmul(orc, dtype):
    rng = np.random.Generator(np.random.PCG64(60))
    x = rng.standard_normal((300, 24)).astype(np.float32)
    w = (rng.standard_normal((24, 3 * 2 * 8)) / np.sqrt(24)).astype(np.float32)
    if dtype == "bf16":
        x, w = workloads.f32_to_bf16_bits(x), workloads.f32_to_bf16_bits(w)
        xd, wd = workloads.bf16_bits_to_f32(x).astype(np.float64), workloads.bf16_bits_to_f32(w).astype(np.float64)
    else:
        xd, wd = x.astype(np.float64), w.astype(np.float64)
    q, k, v = orc.project(x, w, 2, 8)
    y = xd @ wd  # [300, 48]: Q heads, K heads, V heads
    np.testing.assert_allclose(q.reshape(300, 16), y[:, :16], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(k.reshape(300, 16), y[:, 16:32], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(v.reshape(300, 16), y[:, 32:], rtol=1e-12, atol=1e-12)


def test_projection_with_identity_blocks_returns_the_features(orc):
    # W = [I I I]: Q = K = V = X (C = H*d), so attention of the projection is attention of X itself
    rng = np.random.Generator(np.random.PCG64(61))
    x = rng.standard_normal((256, 16)).astype(np.float32)
    w = np.concatenate([np.eye(16, dtype=np.float32)] * 3, axis=1)
    q, k, v = orc.project(x, w, 2, 8)
    np.testing.assert_array_equal(q.reshape(256, 16), x.astype(np.float64))
    pts, perm = _cloud([256], 32, 62)
    xr = x.reshape(256, 2, 8)
    np.testing.assert_array_equal(orc.projected_ball_attention(x, w, 2, 8, 32, perm),
                                  orc.ball_attention(xr, xr, xr, 32, perm))
