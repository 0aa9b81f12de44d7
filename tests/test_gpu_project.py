"""GPU parity of the Q/K/V projection into tree order and of the attention layer built on it.

bt_qkv_project against the oracle's float64 projection (X[perm[slot]] times W): bf16 outputs are the exact
value rounded to bf16, so each element is within 2^-8 of its magnitude (2^-9 for the rounding plus float
accumulation error far below it) plus 2^-14 absolute for values near zero; float outputs within 1e-5
relative.  bt_ball_attention_tree on slot-ordered Q/K/V gives exactly what bt_ball_attention gives on the
same values in the original order (the kernel sees the same tiles).  bt_projected_ball_attention against
the oracle's projected ball attention (float64 projections, no rounding) with the ball-attention
tolerances: 2e-2 absolute and 0.08 of the output RMS for bf16, 1e-4 for float.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

bts = pytest.importorskip("ball_tree_sparse_b200")

REL_BF16 = 0.08


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf(bits):
    return _dev(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _inputs(rows, C, H, d, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    x = workloads.f32_to_bf16_bits(g.standard_normal((rows, C), dtype=np.float32))
    w = workloads.f32_to_bf16_bits((g.standard_normal((C, 3 * H * d)) / np.sqrt(C)).astype(np.float32))
    return x, w


def _check_proj(got, want, bf16=True):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    if bf16:
        bound = 2.0 ** -8 * np.abs(want) + 2.0 ** -14
    else:
        bound = 1e-5 * np.abs(want) + 1e-6
    bad = np.abs(got - want) > bound
    assert not bad.any(), f"{bad.sum()} elements off, worst {np.abs(got - want).max()}"


@pytest.mark.parametrize("n,C,H,d,m", [(8192, 256, 8, 32, 128), (3000, 64, 4, 32, 16), (5000, 512, 2, 64, 64),
                                       (700, 128, 8, 32, 32), (100, 128, 8, 32, 32)])
def test_project_tree_order_matches_oracle(orc, n, C, H, d, m):
    # padded cloud (dummy slots at the end of the tree), tensor-core shapes (a ragged last row tile, the
    # 3*H*d % 256 != 0 tail) and fewer than 128 rows (the CUDA-core kernel)
    pts = workloads.uniform_cloud(n, n + C)
    perm_t, _ = bts.bt_build_segmented(_dev(pts), [0, n], m)
    perm = perm_t.cpu().numpy()
    x, w = _inputs(n, C, H, d, n + H)
    Q, K, V = (torch.full((len(perm), H, d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    bts.bt_qkv_project(_bf(x), _bf(w.T.copy()), H, d, perm=perm_t, out=(Q, K, V))
    assert bts.bt_last_device_status() == 0
    q, k, v = orc.project(x, w, H, d)
    real = perm >= 0
    for got, want in zip((Q, K, V), (q, k, v)):
        g = _np(got)
        _check_proj(g[real], want[perm[real]])
        assert np.all(g[~real] == 0.0)  # dummy slots hold zero rows


def test_project_original_order(orc):
    n, C, H, d = 4000, 256, 8, 32
    x, w = _inputs(n, C, H, d, 9)
    out = bts.bt_qkv_project(_bf(x), _bf(w.T.copy()), H, d)
    q, k, v = orc.project(x, w, H, d)
    for got, want in zip(out, (q, k, v)):
        _check_proj(_np(got), want)


def test_project_bad_slot_is_recorded_not_written(orc):
    n, C, H, d, m = 1024, 128, 8, 32, 128
    perm_t = bts.bt_build(_dev(workloads.uniform_cloud(n, 5)), m)
    inv = bts.bt_invert_perm(perm_t, n)
    inv[17] = n + 3  # not a slot
    x, w = _inputs(n, C, H, d, 13)
    out = tuple(torch.full((n, H, d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    bts.bt_qkv_project(_bf(x), _bf(w.T.copy()), H, d, perm=perm_t, inv=inv, out=out)
    assert bts.bt_last_device_status() == 8  # BT_ERR_INTERNAL
    perm = perm_t.cpu().numpy()
    q, _, _ = orc.project(x, w, H, d)
    g = _np(out[0])
    slot17 = int(np.nonzero(perm == 17)[0][0])
    assert np.all(g[slot17] == 7.0)  # row 17 was not stored anywhere
    keep = perm != 17
    _check_proj(g[keep], q[perm[keep]])


def test_project_float_cuda_cores(orc):
    wl = workloads.tiny()
    perm_t = bts.bt_build(_dev(wl.coords), wl.m)
    perm = perm_t.cpu().numpy()
    x, w = wl.extra["x"], wl.extra["w_qkv"]
    Q, K, V = bts.bt_qkv_project(_dev(x), _dev(w.T.copy()), wl.H, wl.d, perm=perm_t)
    q, k, v = orc.project(x, w, wl.H, wl.d)
    for got, want in zip((Q, K, V), (q, k, v)):
        _check_proj(got.cpu().numpy(), want[perm], bf16=False)


@pytest.mark.parametrize("m", [128, 32])
def test_tree_order_attention_equals_gathered(m):
    wl = workloads.gauss_mix()
    L = wl.layers[1]
    perm, _ = bts.bt_build_segmented(bts.bt_rotate_z(_dev(wl.coords)), wl.offsets, m)
    Q, K, V = _bf(L.q), _bf(L.k), _bf(L.v)
    want = bts.bt_ball_attention(Q, K, V, perm, m)
    Qt, Kt, Vt = (bts.bt_gather(t, perm) for t in (Q, K, V))
    got = bts.bt_ball_attention_tree(Qt, Kt, Vt, perm, m, rows=wl.n_total)
    assert bts.bt_last_device_status() == 0
    assert torch.equal(got, want)


def test_tree_order_attention_ragged_padding(orc):
    wl = workloads.ragged(batch=3, n_min=300, n_max=3000)
    L = wl.layers[0]
    perm_t, _ = bts.bt_build_segmented(_dev(wl.coords), wl.offsets, wl.m)
    perm = perm_t.cpu().numpy()
    Q, K, V = _bf(L.q), _bf(L.k), _bf(L.v)
    Qt, Kt, Vt = (bts.bt_gather(t, perm_t) for t in (Q, K, V))
    got = _np(bts.bt_ball_attention_tree(Qt, Kt, Vt, perm_t, wl.m, rows=wl.n_total))
    want = orc.ball_attention(L.q, L.k, L.v, wl.m, perm)
    err, rms = np.abs(got - want).max(), np.sqrt((want ** 2).mean())
    print(f"parity: max_abs {err:.3e} rms {rms:.3e} max_abs/rms {err / rms:.3e}")
    assert err <= 2e-2 and err / rms <= REL_BF16


def test_projected_layer_ellipsoid_full_size_sampled(orc):
    wl = workloads.ellipsoid()
    x, w = wl.extra["x_bf16"], wl.extra["w_qkv_bf16"]
    perm_t = bts.bt_build(_dev(wl.coords), wl.m)
    perm = perm_t.cpu().numpy()
    o = bts.bt_projected_ball_attention(_bf(x), perm_t, _bf(w.T.copy()), wl.m, wl.H, wl.d)
    assert bts.bt_last_device_status() == 0
    got = _np(o)
    balls = np.random.Generator(np.random.PCG64(11)).choice(len(perm) // wl.m, 40, replace=False)
    rows = np.concatenate([perm[b * wl.m:(b + 1) * wl.m] for b in balls])
    rows = rows[rows >= 0]
    # the oracle projects only the sampled balls' rows
    q, k, v = orc.project(x[rows], w, wl.H, wl.d)
    local = np.arange(len(rows), dtype=np.int32)
    want = orc.ball_attention(q, k, v, wl.m, local)
    err, rms = np.abs(got[rows] - want).max(), np.sqrt((want ** 2).mean())
    print(f"parity: max_abs {err:.3e} rms {rms:.3e} max_abs/rms {err / rms:.3e}")
    assert err <= 2e-2 and err / rms <= REL_BF16


def test_projected_layer_float_tiny(orc):
    wl = workloads.tiny()
    x, w = wl.extra["x"], wl.extra["w_qkv"]
    perm_t = bts.bt_build(_dev(wl.coords), wl.m)
    got = bts.bt_projected_ball_attention(_dev(x), perm_t, _dev(w.T.copy()), wl.m, wl.H, wl.d).cpu().numpy()
    want = orc.projected_ball_attention(x, w, wl.H, wl.d, wl.m, perm_t.cpu().numpy())
    assert np.abs(got - want).max() <= 1e-4


def test_projected_layer_ragged_bf16(orc):
    wl = workloads.ragged(batch=3, n_min=500, n_max=4000, with_qkv=False)
    n = wl.n_total
    x, w = _inputs(n, 128, 8, 32, 31)
    perm_t, _ = bts.bt_build_segmented(_dev(wl.coords), wl.offsets, wl.m)
    got = _np(bts.bt_projected_ball_attention(_bf(x), perm_t, _bf(w.T.copy()), wl.m, 8, 32))
    want = orc.projected_ball_attention(x, w, 8, 32, wl.m, perm_t.cpu().numpy())
    err, rms = np.abs(got - want).max(), np.sqrt((want ** 2).mean())
    print(f"parity: max_abs {err:.3e} rms {rms:.3e} max_abs/rms {err / rms:.3e}")
    assert err <= 2e-2 and err / rms <= REL_BF16
