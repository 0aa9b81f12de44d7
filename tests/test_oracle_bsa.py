"""Pins for the oracle's Ball Sparse Attention (CPU only).

Each branch is checked against an independent restatement: numpy means and
torch scaled_dot_product_attention (float64) for the compression and selection
branches, numpy matmul + sigmoid for the gates, a numpy top-k for the block
selection, the pooled-query identity for the group scores, and the closed
forms the method has (zero gate weights give gates of 1/2; top-k covering
every other block is attention over everything outside the own ball; balls of
one point make the compression branch full attention).
"""
import numpy as np
import pytest
import torch

import workloads


def _widen(a):
    return workloads.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _sdpa_rows(q, keys, vals):
    """q [n, d], keys/vals [k, d] (float64) -> [n, d]"""
    t = [torch.from_numpy(np.ascontiguousarray(a))[None] for a in (q, keys, vals)]
    return torch.nn.functional.scaled_dot_product_attention(*t)[0].numpy()


def _case(n=1024, m=64, H=2, d=32, C=24, seed=0, ragged=False, topk=4):
    rng = np.random.Generator(np.random.PCG64(seed))
    if ragged:
        sizes = [300, 77, 520]
        offsets = np.concatenate([[0], np.cumsum(sizes)])
        pts = np.concatenate([workloads.uniform_cloud(s, seed + i) for i, s in enumerate(sizes)])
        n = len(pts)
    else:
        offsets = None
        pts = workloads.uniform_cloud(n, seed)
    q, k, v = workloads.random_qkv(n, H, d, workloads.BF16, seed + 5)
    x = rng.standard_normal((n, C)).astype(np.float32)
    w = (rng.standard_normal((C, 3 * H)) / np.sqrt(C)).astype(np.float32)
    return dict(n=n, m=m, H=H, d=d, pts=pts, offsets=offsets, q=q, k=k, v=v, x=x, w=w, topk=topk)


def _run(orc, c, **kw):
    perm, _ = orc.build(c["pts"], c["m"], c["offsets"])
    args = dict(topk=c["topk"], branches=True)
    args.update(kw)
    r = orc.bsa(c["q"], c["k"], c["v"], c["m"], perm, c["x"], kw.pop("w", c["w"]), **{k: v for k, v in args.items()
                                                                                       if k != "w"})
    return perm, r


def _means(c, perm):
    """numpy means of Q, K, V per (ball, head) over real rows; valid[b] = ball has a real row"""
    m, H, d = c["m"], c["H"], c["d"]
    nb = len(perm) // m
    Q, K, V = (_widen(t) for t in (c["q"], c["k"], c["v"]))
    qb, kb, vb = (np.zeros((nb, H, d)) for _ in range(3))
    valid = np.zeros(nb, bool)
    for b in range(nb):
        rows = perm[b * m:(b + 1) * m]
        rows = rows[rows >= 0]
        if len(rows):
            valid[b] = True
            qb[b], kb[b], vb[b] = Q[rows].mean(0), K[rows].mean(0), V[rows].mean(0)
    return qb, kb, vb, valid


@pytest.mark.parametrize("ragged", [False, True])
def test_gates_match_numpy(orc, ragged):
    c = _case(ragged=ragged, seed=1)
    b_g = np.linspace(-1, 1, 3 * c["H"]).astype(np.float32)
    perm, r = _run(orc, c, b_g=b_g)
    z = c["x"].astype(np.float64) @ c["w"].astype(np.float64) + b_g
    want = (1 / (1 + np.exp(-z))).reshape(c["n"], c["H"], 3)
    np.testing.assert_allclose(r["gates"], want, rtol=1e-12, atol=1e-14)
    # the gated sum of the three branches
    np.testing.assert_allclose(r["O"], (r["gates"][..., :1] * r["O_ball"] + r["gates"][..., 1:2] * r["O_cmp"] +
                                        r["gates"][..., 2:] * r["O_slc"]), rtol=1e-12, atol=1e-14)


def test_zero_gate_weights_give_half(orc):
    c = _case(seed=2)
    perm, r = _run(orc, c, w=np.zeros_like(c["w"]))
    assert np.all(r["gates"] == 0.5)
    np.testing.assert_allclose(r["O"], 0.5 * (r["O_ball"] + r["O_cmp"] + r["O_slc"]), rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("ragged", [False, True])
def test_compression_branch_vs_sdpa_over_ball_means(orc, ragged):
    c = _case(ragged=ragged, seed=3)
    perm, r = _run(orc, c)
    qb, kb, vb, valid = _means(c, perm)
    Q = _widen(c["q"])
    real = perm[perm >= 0]
    for h in range(c["H"]):
        want = _sdpa_rows(Q[real, h], kb[valid, h], vb[valid, h])
        np.testing.assert_allclose(r["O_cmp"][real, h], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("ragged", [False, True])
def test_group_score_is_group_average_of_logits(orc, ragged):
    # pooled query . coarse key == average over the group of each query's logit against the coarse key
    c = _case(ragged=ragged, seed=4)
    perm, r = _run(orc, c)
    qb, kb, vb, valid = _means(c, perm)
    m, d = c["m"], c["d"]
    Q = _widen(c["q"])
    nb = len(perm) // m
    for g in range(nb):
        rows = perm[g * m:(g + 1) * m]
        rows = rows[rows >= 0]
        for h in range(c["H"]):
            avg = (Q[rows, h] @ kb[:, h].T).mean(0) / np.sqrt(d) if len(rows) else np.full(nb, -np.inf)
            got = r["scores"][g, h]
            ok = np.isfinite(got)
            expect_ok = valid & (np.arange(nb) != g) & (len(rows) > 0)
            assert np.array_equal(ok, expect_ok)
            np.testing.assert_allclose(got[ok], avg[ok], rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("ragged", [False, True])
def test_selection_is_topk_with_own_ball_masked(orc, ragged):
    c = _case(ragged=ragged, seed=5, topk=3)
    perm, r = _run(orc, c)
    nb = len(perm) // c["m"]
    for g in range(nb):
        for h in range(c["H"]):
            s = r["scores"][g, h]
            order = sorted((b for b in range(nb) if np.isfinite(s[b])), key=lambda b: (-s[b], b))
            want = (order + [-1] * c["topk"])[:c["topk"]]
            assert r["sel"][g, h].tolist() == want
            assert g not in r["sel"][g, h].tolist()


def test_selection_branch_vs_sdpa_over_selected_balls(orc):
    c = _case(seed=6, topk=3)
    perm, r = _run(orc, c)
    m = c["m"]
    Q, K, V = (_widen(t) for t in (c["q"], c["k"], c["v"]))
    for g in range(len(perm) // m):
        qrows = perm[g * m:(g + 1) * m]
        for h in range(c["H"]):
            krows = np.concatenate([perm[b * m:(b + 1) * m] for b in r["sel"][g, h] if b >= 0])
            krows = krows[krows >= 0]
            np.testing.assert_allclose(r["O_slc"][qrows, h], _sdpa_rows(Q[qrows, h], K[krows, h], V[krows, h]),
                                       rtol=1e-11, atol=1e-12)


def test_topk_covering_all_blocks_is_attention_outside_own_ball(orc):
    c = _case(n=512, m=64, seed=7)
    nb = 512 // 64
    perm, r = _run(orc, c, topk=nb - 1)
    Q, K, V = (_widen(t) for t in (c["q"], c["k"], c["v"]))
    for g in range(nb):
        own = perm[g * 64:(g + 1) * 64]
        others = np.setdiff1d(np.arange(512), own)
        for h in range(c["H"]):
            np.testing.assert_allclose(r["O_slc"][own, h], _sdpa_rows(Q[own, h], K[others, h], V[others, h]),
                                       rtol=1e-11, atol=1e-12)


def test_single_point_balls_make_compression_full_attention(orc):
    c = _case(n=256, m=1, seed=8, topk=2)
    perm, r = _run(orc, c)
    np.testing.assert_allclose(r["O_cmp"], orc.full_attention(c["q"], c["k"], c["v"]), rtol=1e-11, atol=1e-12)


def test_ball_branch_is_ball_attention(orc):
    c = _case(ragged=True, seed=9)
    perm, r = _run(orc, c)
    want = orc.ball_attention(c["q"], c["k"], c["v"], c["m"], perm)
    np.testing.assert_allclose(r["O_ball"], want, rtol=1e-14, atol=1e-15)


def test_given_selection_is_used(orc):
    c = _case(seed=10, topk=2)
    perm, r = _run(orc, c)
    sel = np.roll(r["sel"], 1, axis=2)
    _, r2 = _run(orc, c, sel_in=sel)
    assert np.array_equal(r2["sel"], sel)
    np.testing.assert_allclose(r2["O_slc"], r["O_slc"], rtol=1e-12, atol=1e-13)  # same set, other order


def test_exact_score_ties_pick_the_lower_ball(orc):
    # every K row the same: all coarse keys are equal, so every score ties and the lowest balls win
    c = _case(n=512, m=64, seed=11, topk=3)
    c["k"] = np.broadcast_to(c["k"][:1], c["k"].shape).copy()
    perm, r = _run(orc, c)
    for g in range(512 // 64):
        want = [b for b in range(8) if b != g][:3]
        for h in range(c["H"]):
            assert r["sel"][g, h].tolist() == want


# --- query coarsening (BSA with group compression): compression and selection take the group's pooled query ---

@pytest.mark.parametrize("ragged", [False, True])
def test_coarsened_branches_vs_sdpa_of_pooled_query(orc, ragged):
    c = _case(ragged=ragged, seed=12, topk=3)
    perm, r = _run(orc, c, coarsen=True)
    _, r0 = _run(orc, c)
    assert np.array_equal(r["sel"], r0["sel"])  # the selection already uses the pooled query
    qb, kb, vb, valid = _means(c, perm)
    m = c["m"]
    K, V = _widen(c["k"]), _widen(c["v"])
    for g in range(len(perm) // m):
        qrows = perm[g * m:(g + 1) * m]
        qrows = qrows[qrows >= 0]
        if not len(qrows):
            continue
        for h in range(c["H"]):
            cmp = _sdpa_rows(qb[g, h][None], kb[valid, h], vb[valid, h])[0]
            krows = np.concatenate([perm[b * m:(b + 1) * m] for b in r["sel"][g, h] if b >= 0])
            krows = krows[krows >= 0]
            slc = _sdpa_rows(qb[g, h][None], K[krows, h], V[krows, h])[0]
            np.testing.assert_allclose(r["O_cmp"][qrows, h], np.broadcast_to(cmp, (len(qrows), c["d"])),
                                       rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(r["O_slc"][qrows, h], np.broadcast_to(slc, (len(qrows), c["d"])),
                                       rtol=1e-11, atol=1e-12)
    # the ball branch and the gates are per query and do not change
    np.testing.assert_array_equal(r["O_ball"], r0["O_ball"])
    np.testing.assert_array_equal(r["gates"], r0["gates"])
    np.testing.assert_allclose(r["O"], (r["gates"][..., :1] * r["O_ball"] + r["gates"][..., 1:2] * r["O_cmp"]
                                        + r["gates"][..., 2:] * r["O_slc"]), rtol=1e-13, atol=1e-14)


def test_coarsening_single_point_balls_changes_nothing(orc):
    # with one point per ball the pooled query is the query itself
    c = _case(n=256, m=1, seed=13, topk=4)
    _, r = _run(orc, c, coarsen=True)
    _, r0 = _run(orc, c)
    for key in ("O", "O_cmp", "O_slc"):
        np.testing.assert_allclose(r[key], r0[key], rtol=1e-14, atol=1e-15)


def test_coarsening_with_identical_group_queries_changes_nothing(orc):
    # every query of a ball equal: the pooled query equals each of them
    c = _case(n=1024, m=64, seed=14, topk=3)
    perm, _ = orc.build(c["pts"], c["m"], None)
    q = c["q"].copy()
    for b in range(len(perm) // 64):
        rows = perm[b * 64:(b + 1) * 64]
        q[rows] = q[rows[0]]
    c["q"] = q
    _, r = _run(orc, c, coarsen=True)
    _, r0 = _run(orc, c)
    assert np.array_equal(r["sel"], r0["sel"])
    for key in ("O", "O_cmp", "O_slc"):
        np.testing.assert_allclose(r[key], r0[key], rtol=1e-12, atol=1e-13)
