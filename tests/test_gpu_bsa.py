"""GPU parity of Ball Sparse Attention against the float64 oracle.

The block selection is a discrete decision taken from float scores: the GPU
scores in float32, the oracle in float64.  Selected sets must be equal, except
where the blocks that differ tie with the k-th best block to within 1e-4 in the
oracle's own scores; the outputs are then compared with the oracle recomputed
on the GPU's selection: max-abs 2e-2 and max-abs at most REL_BF16 = 0.08 of the
output RMS (bf16 inputs and outputs; each branch is a ball-attention-like softmax
whose error is bounded that way, see the ball attention tests, and the gates are
below one).  The query-coarsening variant (compression and selection with each
group's pooled query) is compared with the oracle's coarsened BSA the same way.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")

TIE = 1e-4
TOL = 2e-2
REL_BF16 = 0.08


def _check(got, want):
    err, rms = np.abs(got - want).max(), np.sqrt((want.astype(np.float64) ** 2).mean())
    print(f"parity: max_abs {err:.3e} rms {rms:.3e} max_abs/rms {err / rms:.3e}")
    assert err <= TOL, f"max abs err {err}"
    assert err / rms <= REL_BF16, f"max abs err {err} is {err / rms:.3f} of the output rms {rms}"


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf(a):
    return _dev(a.view(np.int16)).view(torch.bfloat16)


def _run_gpu(q, k, v, perm, x, w, b, topk, mask_own=True, coarsen=False):
    nb, H = len(perm) // 128, q.shape[1]
    sel = torch.full((nb, H, max(topk, 1)), -7, dtype=torch.int32, device="cuda")
    o = bts.bsa_forward(_bf(q), _bf(k), _bf(v), _dev(perm), 128, _dev(x), _dev(w),
                        None if b is None else _dev(b), topk=topk, mask_own_ball=mask_own, sel=sel,
                        coarsen_queries=coarsen)
    assert bts.bt_last_device_status() == 0
    return o.float().cpu().numpy().astype(np.float64), sel.cpu().numpy()[:, :, :topk]


def _check_selection(gpu_sel, ref, topk):
    mism = 0
    for g in range(gpu_sel.shape[0]):
        for h in range(gpu_sel.shape[1]):
            a = set(gpu_sel[g, h].tolist()) - {-1}
            b = set(ref["sel"][g, h].tolist()) - {-1}
            if a == b:
                continue
            s = ref["scores"][g, h]
            kth = np.sort(s[np.isfinite(s)])[::-1][topk - 1]
            for blk in a ^ b:
                assert abs(s[blk] - kth) <= TIE, f"group {g} head {h}: block {blk} is not a near-tie"
            mism += 1
    return mism


def _case(sizes, H, C, seed, topk, mask_own=True, bias=True, d=32):
    pts = np.concatenate([workloads.uniform_cloud(s, seed + i) for i, s in enumerate(sizes)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    n = len(pts)
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, seed)
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal((n, C)).astype(np.float32)
    w = (g.standard_normal((C, 3 * H)) / np.sqrt(C)).astype(np.float32)
    b = np.linspace(-0.5, 0.5, 3 * H).astype(np.float32) if bias else None
    perm, _ = bts.bt_build_segmented(_dev(pts), offsets, 128)
    return q, k, v, perm.cpu().numpy(), x, w, b


@pytest.mark.parametrize("coarsen", [False, True])
@pytest.mark.parametrize("sizes,H,topk,mask_own,d", [([2048], 2, 4, True, 32), ([1500, 700, 2100], 3, 3, True, 32),
                                                     ([4096], 1, 8, False, 32), ([1024], 2, 0, True, 32),
                                                     ([300, 40], 2, 5, True, 32), ([1500, 900], 2, 3, True, 64),
                                                     ([2048], 1, 0, False, 64)])
def test_bsa_matches_oracle(orc, sizes, H, topk, mask_own, d, coarsen):
    q, k, v, perm, x, w, b = _case(sizes, H, 24, sum(sizes) + H, topk, mask_own, d=d)
    got, sel = _run_gpu(q, k, v, perm, x, w, b, topk, mask_own, coarsen)
    ref = orc.bsa(q, k, v, 128, perm, x, w, b, topk=topk, mask_own=mask_own, branches=True, coarsen=coarsen)
    if topk:
        _check_selection(sel, ref, topk)
        ref = orc.bsa(q, k, v, 128, perm, x, w, b, topk=topk, mask_own=mask_own, sel_in=sel, branches=True,
                      coarsen=coarsen)
    real = perm[perm >= 0]
    _check(got[real], ref["O"][real])


@pytest.mark.parametrize("C,H", [(13, 10), (40, 2)])
def test_bsa_gate_shapes(orc, C, H):
    # gate input widths that are not a multiple of 4 (scalar loads) or of the 16-column slice, and more than
    # 24 gates per row (H = 10: two passes over the outputs)
    q, k, v, perm, x, w, b = _case([1500, 700], H, C, 31 + C, 3)
    got, sel = _run_gpu(q, k, v, perm, x, w, b, 3)
    _check_selection(sel, orc.bsa(q, k, v, 128, perm, x, w, b, topk=3, mask_own=True, branches=True), 3)
    ref = orc.bsa(q, k, v, 128, perm, x, w, b, topk=3, mask_own=True, sel_in=sel, branches=True)
    real = perm[perm >= 0]
    _check(got[real], ref["O"][real])


def test_bsa_selection_pinned_by_exact_ties(orc):
    # every K row equal: every score ties, so the selection is the lowest balls other than the group's own
    q, k, v, perm, x, w, b = _case([128 * 8], 2, 16, 5, 3)
    k = np.broadcast_to(k[:1], k.shape).copy()
    _, sel = _run_gpu(q, k, v, perm, x, w, b, 3)
    for g in range(8):
        assert sel[g, 0].tolist() == [blk for blk in range(8) if blk != g][:3]


@pytest.mark.parametrize("coarsen", [False, True])
def test_bsa_ellipsoid_full_size_sampled_groups(orc, coarsen):
    wl = workloads.ellipsoid()
    L = wl.layers[0]
    perm = bts.bt_build(_dev(wl.coords), wl.m).cpu().numpy()
    got, sel = _run_gpu(L.q, L.k, L.v, perm, wl.extra["x"], wl.extra["w_g"], None, 8, coarsen=coarsen)
    nb = len(perm) // 128
    groups = np.random.Generator(np.random.PCG64(4)).choice(nb, 12, replace=False)
    ref = orc.bsa(L.q, L.k, L.v, 128, perm, wl.extra["x"], wl.extra["w_g"], topk=8, branches=True, groups=groups,
                  coarsen=coarsen)
    _check_selection(sel, ref, 8)
    ref = orc.bsa(L.q, L.k, L.v, 128, perm, wl.extra["x"], wl.extra["w_g"], topk=8, sel_in=sel, groups=groups,
                  coarsen=coarsen)
    rows = np.concatenate([perm[gi * 128:(gi + 1) * 128] for gi in groups])
    _check(got[rows], ref[rows])
