"""The seeded input generators: the recipes stated for the synthetic workloads (sizes, layouts, value
distributions, seeds) and the bf16 rounding that both the CUDA path and the oracle read their inputs through.
CPU only; the large workloads are drawn at reduced sizes where the generator takes them as arguments."""
import numpy as np
import torch

import workloads


def test_bf16_rounding_is_nearest_even():
    g = np.random.Generator(np.random.PCG64(3))
    x = np.concatenate([g.standard_normal(10000).astype(np.float32) * 10.0 ** g.integers(-30, 30, 10000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1.0e-40], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(workloads.f32_to_bf16_bits(x), want)
    # ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 and rounds to the even one (1.0)
    assert workloads.f32_to_bf16_bits(np.array([1.00390625], np.float32))[0] == 0x3F80


def test_bf16_widening_is_exact():
    bits = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    f = workloads.bf16_bits_to_f32(bits)
    finite = np.isfinite(f)
    assert np.array_equal(workloads.f32_to_bf16_bits(f[finite]), bits[finite])


def test_padded_size():
    assert [workloads.padded_size(n, 128) for n in (1, 128, 129, 256, 257, 16384, 16385)] == \
        [128, 128, 256, 256, 512, 16384, 32768]
    assert workloads.padded_size(5000, 1) == 8192 and workloads.padded_size(3, 4) == 4


def test_seeded_and_repeatable():
    a, b = workloads.gauss_mix(n_per_cloud=512, batch=2), workloads.gauss_mix(n_per_cloud=512, batch=2)
    assert np.array_equal(a.coords, b.coords) and np.array_equal(a.layers[1].v, b.layers[1].v)
    c = workloads.ragged(batch=3, n_min=300, n_max=900)
    assert not np.array_equal(a.coords[:300], c.coords[:300])


def test_gauss_mix_layout():
    wl = workloads.gauss_mix(n_per_cloud=2048, batch=4)
    assert wl.coords.shape == (8192, 3) and wl.coords.dtype == np.float32
    assert wl.offsets.tolist() == [0, 2048, 4096, 6144, 8192] and wl.m == 128
    assert [L.rotated for L in wl.layers] == [False, True]
    for L in wl.layers:
        for t in (L.q, L.k, L.v):
            assert t.shape == (8192, 8, 32) and t.dtype == np.uint16
    v = workloads.bf16_bits_to_f32(wl.layers[0].q)
    assert abs(float(v.mean())) < 0.02 and abs(float(v.std()) - 1.0) < 0.02  # N(0, 1)
    # each cloud: 8 tight Gaussian blobs (sigma 0.05) around centres in the unit cube
    p = wl.coords[:2048]
    assert p.min() > -0.5 and p.max() < 1.5


def test_box_cluster_mixture():
    wl = workloads.box_cluster(n=20000, with_qkv=False)
    p = wl.coords.astype(np.float64)
    assert p.shape == (20000, 3)
    # 10% of the points sit in one blob of sigma 0.02; the rest spread over [0,4] x [0,1] x [0,1] (about 4.5
    # points per 0.1-wide cell): the densest cell holds part of the blob, and 0.1 (5 sigma) around the blob's
    # mean holds all 2,000 of its points plus a few background ones
    cell = np.floor(p / 0.1).astype(np.int64)
    keys, counts = np.unique(cell, axis=0, return_counts=True)
    assert counts.max() > 200
    centre = p[(cell == keys[np.argmax(counts)]).all(axis=1)].mean(axis=0)
    near = np.linalg.norm(p - centre, axis=1) < 0.1
    centre = p[near].mean(axis=0)
    inside = int((np.linalg.norm(p - centre, axis=1) < 0.1).sum())
    assert 1990 <= inside <= 2100
    assert p[:, 0].max() > 3.9 and p[:, 1].max() < 1.1 and p[:, 2].min() > -0.1


def test_ragged_sizes_and_padding():
    wl = workloads.ragged(with_qkv=False)
    sizes = np.diff(wl.offsets)
    assert len(sizes) == 8 and sizes.min() >= 10_000 and sizes.max() < 200_000
    pad = np.diff(wl.pad_offsets())
    for n, s in zip(sizes, pad):
        assert s >= n and s % 128 == 0 and ((s // 128) & (s // 128 - 1)) == 0 and s < 2 * max(n, 128)


def test_ellipsoid_surface_and_gate_inputs():
    wl = workloads.ellipsoid(n=4096, C=64, H=2)
    p = wl.coords.astype(np.float64)
    r = (p[:, 0] / 2.0) ** 2 + p[:, 1] ** 2 + (p[:, 2] / 0.7) ** 2
    assert np.abs(r - 1.0).max() < 0.02  # on the surface up to the 1e-3 jitter
    assert wl.extra["x"].shape == (4096, 64) and wl.extra["w_g"].shape == (64, 6)
    assert abs(float(wl.extra["w_g"].std()) * 8.0 - 1.0) < 0.1  # N(0, 1/C), C = 64


def test_tiny_projection():
    wl = workloads.tiny()
    assert wl.dtype == workloads.F32 and wl.coords.shape == (1024, 3)
    q = wl.layers[0].q
    assert q.shape == (1024, 2, 32) and q.dtype == np.float32
    assert 0.8 < float(q.std()) < 1.2  # X ~ N(0,1) through W ~ N(0, 1/64): unit variance
