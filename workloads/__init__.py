"""Seeded synthetic inputs for the ball-tree build and ball attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no tree build, no rotation, no attention).  Both the CUDA
path (tests, bench, smoke) and the CPU oracle consume the arrays it returns, so
the two sides always see bit-identical inputs.

The five workloads stand in for the datasets the pages measure on
(ShapeNet-Car, Elasticity, cosmology, molecular dynamics, EAGLE), which are not
available here.  Each generator takes its sizes as arguments; the defaults are
the full-size workloads, smaller values give the same distribution at test
size.

Seeds: base 0xB75EED + 1000 * workload_id, plus a per-stream offset
(+1 coordinates, +2 features X, +3..5 projection weights, +6 gate weights,
+10+3l .. +12+3l the Q/K/V of layer l, +20 ragged cloud sizes).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 0xB75EED

F32 = "f32"
BF16 = "bf16"


def _rng(workload_id: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(SEED_BASE + 1000 * workload_id + stream))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the raw uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen raw bfloat16 bits to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def padded_size(n: int, m: int) -> int:
    """Smallest m * 2^k that holds n points (k >= 0)."""
    leaves = max(1, -(-n // m))
    return m * (1 << (leaves - 1).bit_length())


@dataclass
class Layer:
    """One ball-attention layer: Q/K/V rows in the original point order."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    rotated: bool  # True: the tree of this layer is built on coordinates rotated 45 deg about z


@dataclass
class Workload:
    name: str
    coords: np.ndarray          # float32 [N_total, 3], clouds concatenated
    offsets: np.ndarray         # int64 [B+1], cloud b is rows offsets[b]..offsets[b+1]
    m: int
    H: int
    d: int
    dtype: str                  # F32 or BF16 (bf16 arrays hold raw uint16 bits)
    layers: list = field(default_factory=list)
    extra: dict = field(default_factory=dict)

    @property
    def n_total(self) -> int:
        return int(self.offsets[-1])

    @property
    def batch(self) -> int:
        return len(self.offsets) - 1

    def pad_offsets(self) -> np.ndarray:
        sizes = [padded_size(int(self.offsets[b + 1] - self.offsets[b]), self.m) for b in range(self.batch)]
        return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


def _qkv(workload_id: int, layer: int, n: int, H: int, d: int, dtype: str):
    out = []
    for j in range(3):
        g = _rng(workload_id, 10 + 3 * layer + j)
        a = g.standard_normal((n, H, d), dtype=np.float32)
        out.append(f32_to_bf16_bits(a) if dtype == BF16 else a)
    return out


def _gauss_mix_cloud(g: np.ndarray, n: int, centres: int = 8, sigma: float = 0.05) -> np.ndarray:
    c = g.random((centres, 3))
    pick = g.integers(0, centres, size=n)
    p = c[pick] + sigma * g.standard_normal((n, 3))
    return p.astype(np.float32)


def tiny(n: int = 1024, m: int = 32, C: int = 64, H: int = 2, d: int = 32) -> Workload:
    """Uniform points in [0,1)^3, fp32 features projected to H heads by N(0, 1/C) weights."""
    wid = 1
    coords = _rng(wid, 1).random((n, 3)).astype(np.float32)
    x = _rng(wid, 2).standard_normal((n, C))
    proj, ws = [], []
    for j in range(3):
        w = _rng(wid, 3 + j).standard_normal((C, H * d)) / math.sqrt(C)
        ws.append(w)
        proj.append((x @ w).astype(np.float32).reshape(n, H, d))
    wl = Workload("tiny", coords, np.array([0, n], np.int64), m, H, d, F32)
    wl.layers.append(Layer(proj[0], proj[1], proj[2], rotated=False))
    # the same features and weights rounded to float, for a layer that projects on the device:
    # X [n, C] and W [C, 3 H d] (Q, K, V column blocks)
    wl.extra["x"] = x.astype(np.float32)
    wl.extra["w_qkv"] = np.concatenate(ws, axis=1).astype(np.float32)
    return wl


def gauss_mix(n_per_cloud: int = 16384, batch: int = 4, m: int = 128, H: int = 8, d: int = 32) -> Workload:
    """Batch of clouds, each a mixture of 8 isotropic Gaussians (sigma 0.05, centres in the unit cube).
    Two layers: A on the original tree, B on the tree of the coordinates rotated 45 deg about z."""
    wid = 2
    g = _rng(wid, 1)
    coords = np.concatenate([_gauss_mix_cloud(g, n_per_cloud) for _ in range(batch)])
    n = n_per_cloud * batch
    wl = Workload("gauss_mix", coords, np.arange(batch + 1, dtype=np.int64) * n_per_cloud, m, H, d, BF16)
    for layer, rot in ((0, False), (1, True)):
        q, k, v = _qkv(wid, layer, n, H, d, BF16)
        wl.layers.append(Layer(q, k, v, rotated=rot))
    return wl


def ellipsoid(n: int = 65536, m: int = 128, C: int = 256, H: int = 8, d: int = 32,
              semi_axes=(2.0, 1.0, 0.7), jitter: float = 1e-3) -> Workload:
    """Points uniform on an ellipsoid surface (area-element rejection), plus Gaussian jitter.
    Carries the gate features X [n, C] and gate weights W_g [C, 3H] ~ N(0, 1/C); for a layer that projects its
    own Q/K/V, X rounded to bf16 and projection weights W_qkv [C, 3 H d] ~ N(0, 1/C) in bf16 (raw bits)."""
    wid = 3
    a, b, c = semi_axes
    g = _rng(wid, 1)
    pts = []
    have = 0
    gmax = max(b * c, a * c, a * b)
    while have < n:
        u = g.standard_normal((2 * n, 3))
        u /= np.linalg.norm(u, axis=1, keepdims=True)
        area = np.sqrt((b * c * u[:, 0]) ** 2 + (a * c * u[:, 1]) ** 2 + (a * b * u[:, 2]) ** 2)
        keep = g.random(2 * n) * gmax < area
        p = u[keep] * np.array([a, b, c])
        pts.append(p)
        have += len(p)
    p = np.concatenate(pts)[:n]
    p = p + jitter * g.standard_normal((n, 3))
    coords = p.astype(np.float32)
    wl = Workload("ellipsoid", coords, np.array([0, n], np.int64), m, H, d, BF16)
    q, k, v = _qkv(wid, 0, n, H, d, BF16)
    wl.layers.append(Layer(q, k, v, rotated=False))
    wl.extra["x"] = _rng(wid, 2).standard_normal((n, C), dtype=np.float32)
    wl.extra["w_g"] = (_rng(wid, 6).standard_normal((C, 3 * H)) / math.sqrt(C)).astype(np.float32)
    wl.extra["x_bf16"] = f32_to_bf16_bits(wl.extra["x"])
    wl.extra["w_qkv_bf16"] = f32_to_bf16_bits(
        (_rng(wid, 7).standard_normal((C, 3 * H * d), dtype=np.float32) / np.float32(math.sqrt(C))).astype(np.float32))
    return wl


def box_cluster(n: int = 1 << 20, m: int = 128, H: int = 4, d: int = 32, with_qkv: bool = True) -> Workload:
    """90% of points uniform in [0,4]x[0,1]x[0,1], 10% in one Gaussian sub-cluster (sigma 0.02)
    whose centre is uniform in the box; rows shuffled by a seeded permutation.
    Two layers: A on the original tree, B on the rotated tree."""
    wid = 4
    g = _rng(wid, 1)
    n_clu = n // 10
    box = g.random((n - n_clu, 3)) * np.array([4.0, 1.0, 1.0])
    mu = g.random(3) * np.array([4.0, 1.0, 1.0])
    clu = mu + 0.02 * g.standard_normal((n_clu, 3))
    p = np.concatenate([box, clu])[g.permutation(n)]
    coords = p.astype(np.float32)
    wl = Workload("box_cluster", coords, np.array([0, n], np.int64), m, H, d, BF16)
    if with_qkv:
        for layer, rot in ((0, False), (1, True)):
            q, k, v = _qkv(wid, layer, n, H, d, BF16)
            wl.layers.append(Layer(q, k, v, rotated=rot))
    return wl


def ragged(batch: int = 8, n_min: int = 10_000, n_max: int = 200_000, m: int = 128, H: int = 8,
           d: int = 32, with_qkv: bool = True) -> Workload:
    """Batch of clouds with log-uniform sizes, Gaussian-mixture coordinates as in gauss_mix.
    Each cloud is padded to m * 2^k slots by dummy points (masked in attention)."""
    wid = 5
    gs = _rng(wid, 20)
    sizes = np.floor(np.exp(gs.uniform(math.log(n_min), math.log(n_max), size=batch))).astype(np.int64)
    g = _rng(wid, 1)
    coords = np.concatenate([_gauss_mix_cloud(g, int(s)) for s in sizes])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    n = int(offsets[-1])
    wl = Workload("ragged", coords, offsets, m, H, d, BF16)
    if with_qkv:
        q, k, v = _qkv(wid, 0, n, H, d, BF16)
        wl.layers.append(Layer(q, k, v, rotated=False))
    return wl


def uniform_cloud(n: int, seed: int, scale=(1.0, 1.0, 1.0)) -> np.ndarray:
    """Plain uniform points for small tests (float32 [n, 3])."""
    g = np.random.Generator(np.random.PCG64(SEED_BASE + 7_000_000 + seed))
    return (g.random((n, 3)) * np.asarray(scale)).astype(np.float32)


def tied_cloud(n: int, seed: int, levels: int = 4) -> np.ndarray:
    """Points on a coarse integer grid, so that coordinate ties are frequent (float32 [n, 3])."""
    g = np.random.Generator(np.random.PCG64(SEED_BASE + 8_000_000 + seed))
    return g.integers(0, levels, size=(n, 3)).astype(np.float32)


def random_qkv(n: int, H: int, d: int, dtype: str, seed: int):
    """N(0,1) Q, K, V [n, H, d] for small tests (bf16 as raw uint16 bits)."""
    out = []
    for j in range(3):
        g = np.random.Generator(np.random.PCG64(SEED_BASE + 9_000_000 + 10 * seed + j))
        a = g.standard_normal((n, H, d), dtype=np.float32)
        out.append(f32_to_bf16_bits(a) if dtype == BF16 else a)
    return out
