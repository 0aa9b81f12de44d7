"""Independent checks of a ball-tree permutation (pure Python / numpy).

Used to pin the oracle and, on the GPU, to check permutations at sizes where
comparing against the oracle is not enough on its own.  Nothing here calls the
oracle or the CUDA library.
"""
from __future__ import annotations

import numpy as np


def padded(n: int, m: int) -> int:
    leaves = max(1, -(-n // m))
    return m * (1 << (leaves - 1).bit_length())


def brute_build(pts: np.ndarray, m: int) -> list:
    """Second, level-by-level formulation of the split rule for tiny clouds.

    Breadth-first: every level sorts each node's slots with Python's sort on
    (is_dummy, coordinate as a float, index) and cuts it in half; the extent of
    a node is the float32 difference of its largest and smallest real
    coordinate, and the first axis with the largest extent is split.
    """
    pts = np.asarray(pts, dtype=np.float32)
    n = len(pts)
    npad = padded(n, m)
    segs = [list(range(npad))]
    while len(segs[0]) > m:
        nxt = []
        for S in segs:
            real = [i for i in S if i < n]
            ext = [0.0, 0.0, 0.0]
            if real:
                for a in range(3):
                    vals = [float(pts[i, a]) for i in real]
                    ext[a] = float(np.float32(max(vals)) - np.float32(min(vals)))
            axis = 0
            for a in (1, 2):
                if ext[a] > ext[axis]:
                    axis = a
            S2 = sorted(S, key=lambda i: (0, float(pts[i, axis]), i) if i < n else (1, 0.0, i))
            h = len(S2) // 2
            nxt += [S2[:h], S2[h:]]
        segs = nxt
    return [i if i < n else -1 for S in segs for i in sorted(S)]


def check_tree(perm: np.ndarray, coords: np.ndarray, m: int, offsets=None) -> None:
    """Assert every property the split rule fixes, cloud by cloud.

    1. perm is a bijection from the real slots onto the rows; dummies are -1.
    2. every internal node's lower half holds exactly the smaller half of its
       points under (coordinate on the node's widest axis, index), dummies last.
    3. every leaf lists its real rows in ascending order, dummies after them.
    Together these determine perm uniquely.
    """
    perm = np.asarray(perm)
    coords = np.asarray(coords, dtype=np.float32)
    n_all = coords.shape[0]
    offsets = np.array([0, n_all] if offsets is None else offsets, dtype=np.int64)
    real = perm[perm >= 0]
    assert len(real) == n_all, "real slot count != row count"
    assert np.array_equal(np.sort(real), np.arange(n_all)), "not a bijection onto the rows"
    base = 0
    for b in range(len(offsets) - 1):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        n = hi - lo
        s_all = padded(n, m)
        p = perm[base:base + s_all].astype(np.int64)
        assert np.all((p == -1) | ((p >= lo) & (p < hi))), f"cloud {b}: row of another cloud"
        c = coords[lo:hi]
        # local ids with dummies numbered n, n+1, ... in slot order (they sort by index among themselves)
        ids = np.where(p >= 0, p - lo, -1)
        dummy_slots = np.nonzero(ids < 0)[0]
        ids[dummy_slots] = n + np.arange(len(dummy_slots))
        s = s_all
        while s > m:
            for start in range(0, s_all, s):
                node = ids[start:start + s]
                rl = node[node < n]
                ext = np.zeros(3, np.float32)
                if len(rl):
                    ext = (c[rl].max(axis=0) - c[rl].min(axis=0)).astype(np.float32)
                axis = int(np.argmax(ext))  # first maximum: lowest axis on ties
                key = np.where(node < n, c[np.minimum(node, n - 1), axis].astype(np.float64), np.inf)
                key = np.where(key == 0.0, 0.0, key)
                order = np.lexsort((node, key))
                want_left = set(node[order[: s // 2]].tolist())
                assert set(node[: s // 2].tolist()) == want_left, f"cloud {b}: node at {start} size {s} split wrong"
            s //= 2
        for start in range(0, s_all, m):
            leaf = ids[start:start + m]
            assert np.all(np.diff(leaf) > 0), f"cloud {b}: leaf at {start} not in index order"
        base += s_all
    assert base == len(perm), "perm length != sum of padded cloud sizes"
