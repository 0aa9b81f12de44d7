"""GPU parity of the tree build, rotation and slot maps against the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import workloads
from treecheck import check_tree, padded

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _gpu_build(coords, m, offsets=None):
    n = coords.shape[0]
    c = _dev(coords)
    if offsets is None:
        ws = bts.workspace([0, n], m)
        perm = bts.bt_build(c, m, ws=ws)
    else:
        ws = bts.workspace(offsets, m)
        perm, _ = bts.bt_build_segmented(c, offsets, m, ws=ws)
    assert bts.bt_build_device_status(ws) == 0
    return perm.cpu().numpy()


SINGLE = [
    # (n, m, kind): tail only, several wide levels, many tiles per node, odd m, m = 1
    (1024, 32, "uniform"),
    (32 * 2 ** 9, 32, "uniform"),
    (32 * 2 ** 9, 32, "tied"),
    (128 * 2 ** 10, 128, "uniform"),
    (3 * 2 ** 12, 3, "tied"),
    (2 ** 13, 1, "tied"),
    (7 * 2 ** 11, 7, "uniform"),
    (100 * 2 ** 7, 100, "signed"),
    (128, 128, "uniform"),
    (1, 1, "uniform"),
    (1024 * 8, 1024, "uniform"),
    # one-launch cluster path: 16,384 slots (1,024 per CTA), 32,768 slots (its largest cloud, 2,048 per CTA)
    (16384, 128, "tied"),
    (2 ** 14, 16, "tied"),
    (2 ** 15, 256, "tied"),
    (32768, 64, "uniform"),
    # record path (power-of-two clouds above 32,768 slots) with leaf size 1
    (2 ** 16, 1, "tied"),
    # index-list path (m not a power of two) with several wide levels
    (3 * 2 ** 15, 3, "tied"),
    (100 * 2 ** 10, 100, "uniform"),
]


def _points(n, kind, seed):
    if kind == "uniform":
        return workloads.uniform_cloud(n, seed)
    if kind == "tied":
        return workloads.tied_cloud(n, seed, levels=6)
    sign = np.where(workloads.tied_cloud(n, seed + 1, levels=2) > 0, -1, 1).astype(np.float32)
    return workloads.tied_cloud(n, seed, levels=3) * sign


@pytest.mark.parametrize("n,m,kind", SINGLE)
def test_build_single_bit_exact(orc, n, m, kind):
    pts = _points(n, kind, n + m)
    want, _ = orc.build(pts, m)
    got = _gpu_build(pts, m)
    assert np.array_equal(got, want)
    if n <= 1 << 15:
        check_tree(got, pts, m)


@pytest.mark.parametrize("sizes,m", [([1, 5, 100, 3000, 40000], 128), ([17, 4096, 4097, 300], 16),
                                     ([2000] * 8, 1), ([5, 1, 9], 4),
                                     # one-launch cluster path with few leaves per CTA
                                     ([1200], 4),
                                     # cluster path, clouds of 32,768, 16,384 and 512 slots in one launch
                                     ([20000, 9000, 300], 32), ([12000], 64),
                                     # record path: ragged counts, leaf sizes 1, 2, 16 and 64
                                     ([40000], 1), ([70000], 2), ([33000, 20000], 16), ([200000], 64)])
def test_build_segmented_bit_exact(orc, sizes, m):
    pts = np.concatenate([workloads.tied_cloud(s, 70 + i, levels=9) for i, s in enumerate(sizes)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    want, pad = orc.build(pts, m, offsets)
    got = _gpu_build(pts, m, offsets)
    assert np.array_equal(got, want)
    if sum(sizes) <= 1 << 15:
        check_tree(got, pts, m, offsets)


@pytest.mark.parametrize("sizes,m,flags", [
    # narrow one-launch clusters (2,048 slots per CTA): 16,384-slot clouds, a ragged mix, a lone 8,192
    ([16384] * 4, 128, 1), ([20000, 9000, 300], 32, 1), ([5000], 128, 1), ([600], 16, 1),
    # leaf size 1: every level down to single slots (the most in-CTA levels and node pivots)
    ([32768], 1, 0), ([8192], 1, 1), ([5000, 2100], 1, 0),
    # more clouds than wide clusters fit at once: the library picks narrow ones by itself
    ([16384] * 12, 128, 0),
])
def test_build_flags_bit_exact(orc, sizes, m, flags):
    pts = np.concatenate([workloads.tied_cloud(s, 90 + i, levels=9) for i, s in enumerate(sizes)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    want, pad = orc.build(pts, m, offsets)
    c = torch.from_numpy(pts).to("cuda")
    ws = bts.workspace(offsets, m)
    got, _ = bts.bt_build_segmented_ex(c, offsets, m, flags, ws=ws)
    assert bts.bt_build_device_status(ws) == 0
    assert np.array_equal(got.cpu().numpy(), want)


def test_workload_tiny(orc):
    wl = workloads.tiny()
    assert np.array_equal(_gpu_build(wl.coords, wl.m), orc.build(wl.coords, wl.m)[0])


def test_workload_gauss_mix_both_trees(orc):
    wl = workloads.gauss_mix()
    got = _gpu_build(wl.coords, wl.m, wl.offsets)
    assert np.array_equal(got, orc.build(wl.coords, wl.m, wl.offsets)[0])
    rot = bts.bt_rotate_z(_dev(wl.coords)).cpu().numpy()
    assert np.array_equal(rot.view(np.uint32), orc.rotate_z(wl.coords).view(np.uint32))
    got_b = _gpu_build(rot, wl.m, wl.offsets)
    assert np.array_equal(got_b, orc.build(rot, wl.m, wl.offsets)[0])


def test_workload_ellipsoid(orc):
    wl = workloads.ellipsoid()
    assert np.array_equal(_gpu_build(wl.coords, wl.m), orc.build(wl.coords, wl.m)[0])


def test_workload_box_cluster_full_size(orc):
    wl = workloads.box_cluster(with_qkv=False)
    got = _gpu_build(wl.coords, wl.m)
    assert np.array_equal(got, orc.build(wl.coords, wl.m)[0])
    rot = orc.rotate_z(wl.coords)
    assert np.array_equal(bts.bt_rotate_z(_dev(wl.coords)).cpu().numpy().view(np.uint32), rot.view(np.uint32))
    assert np.array_equal(_gpu_build(rot, wl.m), orc.build(rot, wl.m)[0])


def test_workload_ragged_full_size(orc):
    wl = workloads.ragged(with_qkv=False)
    got = _gpu_build(wl.coords, wl.m, wl.offsets)
    want, pad = orc.build(wl.coords, wl.m, wl.offsets)
    assert np.array_equal(got, want)
    assert np.array_equal(pad, wl.pad_offsets())


def test_repeat_and_reuse_workspace(orc):
    # one workspace reused by a smaller build and by the same build twice in a row
    big = workloads.uniform_cloud(128 * 2 ** 8, 1)
    small = workloads.tied_cloud(128 * 2 ** 5, 2, levels=4)
    ws = bts.workspace([0, len(big)], 128)
    for pts in (big, small, big):
        perm = bts.bt_build(_dev(pts), 128, ws=ws).cpu().numpy()
        assert bts.bt_build_device_status(ws) == 0
        assert np.array_equal(perm, orc.build(pts, 128)[0])


def test_rotate_bit_exact_special_values(orc):
    pts = np.array([[1, 0, 0], [0, 1, 0], [-0.0, -0.0, 3], [1e-40, -1e-40, 0], [3e38, 3e38, -1],
                    [-2.5, 7.25, 1e-3]], np.float32)
    pts = np.concatenate([pts, (workloads.uniform_cloud(5000, 4) - 0.5) * 100])
    got = bts.bt_rotate_z(_dev(pts)).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), orc.rotate_z(pts).view(np.uint32))


def test_invert_compose_bit_exact(orc):
    wl = workloads.ragged(batch=3, n_min=300, n_max=3000)
    pa = _gpu_build(wl.coords, wl.m, wl.offsets)
    rot = orc.rotate_z(wl.coords)
    pb = _gpu_build(rot, wl.m, wl.offsets)
    n = wl.n_total
    inv = bts.bt_invert_perm(_dev(pa), n).cpu().numpy()
    assert np.array_equal(inv, orc.invert(pa, n))
    mp = bts.bt_compose(_dev(inv), _dev(pb)).cpu().numpy()
    assert np.array_equal(mp, orc.compose(inv, pb))


def test_gather_scatter_exact():
    g = np.random.Generator(np.random.PCG64(3))
    n, npad = 1000, 1024
    perm = np.full(npad, -1, np.int32)
    perm[g.permutation(npad)[:n]] = np.arange(n, dtype=np.int32)
    for shape, dt in (((n, 8, 32), torch.bfloat16), ((n, 2, 32), torch.float32), ((n, 3), torch.float32),
                      ((n, 5), torch.uint8)):
        X = (torch.randn(shape, generator=torch.Generator().manual_seed(1)) * 10).to(dt).cuda()
        Y = bts.bt_gather(X, _dev(perm))
        Xc, Yc = X.cpu(), Y.cpu()
        for s in range(npad):
            want = Xc[perm[s]] if perm[s] >= 0 else torch.zeros_like(Xc[0])
            assert torch.equal(Yc[s], want)
        Z = torch.zeros_like(X)
        bts.bt_scatter(Y, _dev(perm), Z)
        assert torch.equal(Z.cpu(), Xc)
