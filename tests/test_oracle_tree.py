"""Pins for the oracle's tree build (CPU only).

The oracle is checked against things other than itself: hand-worked examples
(tests/golden/tree_hand_examples.json), a second brute-force formulation in
pure Python on tiny clouds, and the structural properties that fix the
permutation uniquely.
"""
import json
import os

import numpy as np
import pytest

import workloads
from treecheck import brute_build, check_tree, padded

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tree_hand_examples.json")


def test_hand_examples(orc):
    cases = json.load(open(GOLDEN))["cases"]
    assert len(cases) >= 7
    for c in cases:
        perm, pad = orc.build(np.array(c["points"], np.float32), c["m"])
        assert perm.tolist() == c["perm"], c["name"]
        assert int(pad[-1]) == len(c["perm"])


def _cases():
    rng = np.random.Generator(np.random.PCG64(1234))
    for t in range(60):
        n = int(rng.integers(1, 65))
        m = int(rng.choice([1, 2, 3, 4, 5, 8]))
        kind = t % 4
        if kind == 0:
            pts = workloads.uniform_cloud(n, t)
        elif kind == 1:
            pts = workloads.tied_cloud(n, t, levels=3)
        elif kind == 2:
            pts = (workloads.uniform_cloud(n, t) - 0.5) * 1e-3
        else:
            sign = np.where(workloads.tied_cloud(n, t + 500, levels=2) > 0, -1, 1).astype(np.float32)
            pts = workloads.tied_cloud(n, t, levels=2) * sign  # values -1, -0.0, +0.0, 1
        yield n, m, pts


@pytest.mark.parametrize("n,m,pts", list(_cases()))
def test_brute_force_small(orc, n, m, pts):
    perm, _ = orc.build(pts, m)
    assert perm.tolist() == brute_build(pts, m)


@pytest.mark.parametrize("n,m,seed", [(4096, 32, 0), (3000, 128, 1), (1000, 7, 2), (2048, 1, 3)])
def test_structure(orc, n, m, seed):
    for pts in (workloads.uniform_cloud(n, seed), workloads.tied_cloud(n, seed, levels=5)):
        perm, pad = orc.build(pts, m)
        assert len(perm) == padded(n, m)
        check_tree(perm, pts, m)


def test_batch_equals_separate(orc):
    sizes = [100, 64, 1, 257]
    clouds = [workloads.tied_cloud(s, 40 + i, levels=6) for i, s in enumerate(sizes)]
    offsets = np.concatenate([[0], np.cumsum(sizes)])
    perm, pad = orc.build(np.concatenate(clouds), 16, offsets)
    check_tree(perm, np.concatenate(clouds), 16, offsets)
    for b, c in enumerate(clouds):
        single, _ = orc.build(c, 16)
        got = perm[pad[b]:pad[b + 1]]
        want = np.where(single >= 0, single + offsets[b], -1)
        assert np.array_equal(got, want)


def test_shuffle_equivariance_tie_free(orc):
    # Without coordinate ties the index never decides a split, so the set of rows in every
    # leaf is carried along by a shuffle of the input rows.
    n, m = 2048, 16
    pts = workloads.uniform_cloud(n, 99)
    for a in range(3):
        assert len(np.unique(pts[:, a])) == n
    perm, _ = orc.build(pts, m)
    sh = np.random.Generator(np.random.PCG64(5)).permutation(n)
    perm2, _ = orc.build(pts[sh], m)
    leaves1 = [sorted(perm[i:i + m].tolist()) for i in range(0, n, m)]
    leaves2 = [sorted(sh[perm2[i:i + m]].tolist()) for i in range(0, n, m)]
    assert leaves1 == leaves2


def test_single_leaf_and_identity(orc):
    pts = workloads.uniform_cloud(50, 3)
    perm, _ = orc.build(pts, 64)
    assert perm.tolist() == list(range(50)) + [-1] * 14


def test_rejects_bad_input(orc):
    pts = workloads.uniform_cloud(8, 0)
    bad = pts.copy()
    bad[3, 1] = np.nan
    with pytest.raises(orc.OracleError):
        orc.build(bad, 2)
    bad[3, 1] = np.inf
    with pytest.raises(orc.OracleError):
        orc.build(bad, 2)
    with pytest.raises(orc.OracleError):
        orc.build(pts, 0)


def test_invert_compose(orc):
    pts = workloads.uniform_cloud(300, 8)
    pA, _ = orc.build(pts, 8)
    pB, _ = orc.build(orc.rotate_z(pts), 8)
    inv = orc.invert(pA, 300)
    assert np.array_equal(pA[inv], np.arange(300))
    mp = orc.compose(inv, pB)
    X = np.arange(300) * 10 + 7
    XA = np.where(pA >= 0, X[np.maximum(pA, 0)], -1)    # rows in tree-A order
    XB = np.where(mp >= 0, XA[np.maximum(mp, 0)], -1)   # moved to tree-B order through the map
    assert np.array_equal(XB, np.where(pB >= 0, X[np.maximum(pB, 0)], -1))
