"""Pins for the rounding of the oracle's rotation (CPU only).

The rotated layers of Erwin (author's thread, the post on cross-partition exchange: trees are rotated
where Swin would shift windows) rebuild the tree on rotated floats, and the build is bit-exact, so the
rotation's rounding is part of the result.  The reading: every product and every sum rounded to float on
its own, x' = rn(rn(c x) - rn(s y)), y' = rn(rn(s x) + rn(c y)), c = s = float bits 0x3F3504F3.

Two pins that do not go through the oracle's code:
  - numpy float32 array arithmetic (each ufunc rounds its own result; no contraction across ufuncs) on
    200,000 points of the workloads' kinds plus exponent extremes, compared bit for bit;
  - tests/golden/rotation_fma_cases.json: inputs where a fused multiply-add gives a different float,
    with the expected bits derived in exact rational arithmetic.
A version of the oracle whose rotation contracts a product into a sum fails both.
"""
import importlib.util
import json
import os
import struct
from fractions import Fraction

import numpy as np

import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
C45 = np.array([0x3F3504F3], np.uint32).view(np.float32)[0]


def _golden_module():
    spec = importlib.util.spec_from_file_location("make_rotation_cases",
                                                  os.path.join(GOLDEN, "make_rotation_cases.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def _numpy_rotation(p):
    x, y = p[:, 0], p[:, 1]
    c = np.float32(C45)
    with np.errstate(over="ignore", under="ignore"):
        cx, sy, sx, cy = c * x, c * y, c * x, c * y  # four float32 products, each rounded
    out = np.empty_like(p)
    with np.errstate(over="ignore"):  # the 3e38 rows overflow to infinity on both sides
        out[:, 0] = cx - sy
        out[:, 1] = sx + cy
    out[:, 2] = p[:, 2]
    return out


def _points():
    rng = np.random.default_rng(0xB75EED)
    parts = [
        workloads.uniform_cloud(60_000, 3),
        (workloads.uniform_cloud(50_000, 4) - 0.5) * 8.0,
        rng.normal(0.5, 0.05, size=(40_000, 3)).astype(np.float32),
        # exponents from 2^-140 (subnormal products) to 2^100
        (rng.uniform(-1, 1, size=(50_000, 3)) * 2.0 ** rng.integers(-140, 100, size=(50_000, 1))).astype(np.float32),
        np.array([[0.0, -0.0, 1.0], [-0.0, 0.0, -1.0], [1e-45, -1e-45, 0.0], [3e38, -3e38, 2.0],
                  [1.0, 1.0, 0.0], [-1.0, 1.0, 0.0]] * 10, np.float32),
    ]
    return np.ascontiguousarray(np.concatenate(parts), np.float32)


def test_rotation_bits_equal_numpy_float32(orc):
    p = _points()
    assert p.shape[0] >= 200_000
    got = orc.rotate_z(p)
    want = _numpy_rotation(p)
    bad = np.nonzero(_bits(got) != _bits(want))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {p[bad[0] // 3]}"


def test_rotation_fma_sensitive_golden_cases(orc):
    doc = json.load(open(os.path.join(GOLDEN, "rotation_fma_cases.json")))
    cases = doc["cases"]
    kinds = set()
    for c in cases:
        kinds.update(c["fused_differs"])
    # every contraction a compiler may form is caught by at least one case
    assert kinds == {"x_fma_first", "x_fma_second", "y_fma_first", "y_fma_second"}
    inp = np.array([[int(v, 16) for v in c["in"]] for c in cases], np.uint32).view(np.float32)
    want = np.array([[int(v, 16) for v in c["out"]] for c in cases], np.uint32)
    got = _bits(orc.rotate_z(inp)).reshape(-1, 3)
    assert np.array_equal(got, want)
    # the stored bits are what exact arithmetic with per-operation rounding gives, and numpy agrees
    gm = _golden_module()
    for c, row in zip(cases, inp):
        xs, ys = gm.rotate_separate(Fraction(float(row[0])), Fraction(float(row[1])))
        assert [gm.bits_of(xs), gm.bits_of(ys)] == [int(c["out"][0], 16), int(c["out"][1], 16)]
        for k, v in c["fused_differs"].items():
            assert int(v, 16) != int(c["out"][0 if k.startswith("x") else 1], 16)
    assert np.array_equal(_bits(_numpy_rotation(inp)).reshape(-1, 3), want)


def test_exact_rounding_helper_matches_float32_products():
    """The golden cases' rn() agrees with IEEE float32 multiplication on random operands."""
    gm = _golden_module()
    rng = np.random.default_rng(7)
    a = (rng.uniform(-4, 4, 2000) * 2.0 ** rng.integers(-60, 60, 2000)).astype(np.float32)
    b = (rng.uniform(-4, 4, 2000) * 2.0 ** rng.integers(-60, 60, 2000)).astype(np.float32)
    prod = a * b
    for x, y, p in zip(a.tolist(), b.tolist(), prod.tolist()):
        assert gm.bits_of(gm.rn(Fraction(x) * Fraction(y))) == struct.unpack("<I", struct.pack("<f", p))[0]
