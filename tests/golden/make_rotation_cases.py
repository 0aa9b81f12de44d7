"""Writes rotation_fma_cases.json: inputs where the rotation's per-operation rounding and a fused
multiply-add give different floats, with the expected outputs derived in exact rational arithmetic.

The rotated layers of Erwin (author's thread, the post on cross-partition exchange: the tree is rotated
where Swin would shift its windows) rebuild the tree on rotated coordinates, so the rotated floats are
inputs of a bit-exact build and their rounding has to be fixed.  The reading taken: 45 degrees about +z,
c = s = float(sqrt(1/2)) (bits 0x3F3504F3), every product and every sum rounded to float on its own:
    x' = rn(rn(c x) - rn(s y)),   y' = rn(rn(s x) + rn(c y)).
A fused form rounds once where two roundings are expected, e.g. x' = rn(c x - rn(s y)).

This script imports neither the oracle nor the library: products and sums are exact Fractions, and
rn() is round-to-nearest-even onto the float32 grid written out below.  Run it from the repository
root: python tests/golden/make_rotation_cases.py
"""
from __future__ import annotations

import json
import os
import random
import struct
from fractions import Fraction

C_BITS = 0x3F3504F3


def f32_from_bits(b: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", b))[0])


def bits_of(v: Fraction) -> int:
    return struct.unpack("<I", struct.pack("<f", float(v)))[0]


def rn(v: Fraction) -> Fraction:
    """Round an exact rational to the nearest float32, ties to even (no overflow handling needed here)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()  # 2^e <= a < 2^(e+1) after the fix below
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)                     # below the normal range the grid spacing stays 2^-149
    ulp = Fraction(2) ** (e - 23)
    q = a / ulp
    n = q.numerator // q.denominator
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def rotate_separate(x: Fraction, y: Fraction):
    c = f32_from_bits(C_BITS)
    return rn(rn(c * x) - rn(c * y)), rn(rn(c * x) + rn(c * y))


def rotate_fused_variants(x: Fraction, y: Fraction):
    """The contractions a compiler may form: one product kept exact inside each sum."""
    c = f32_from_bits(C_BITS)
    return {
        "x_fma_first": rn(c * x - rn(c * y)),
        "x_fma_second": rn(rn(c * x) - c * y),
        "y_fma_first": rn(c * x + rn(c * y)),
        "y_fma_second": rn(rn(c * x) + c * y),
    }


def main():
    rng = random.Random(20240521)
    cases = []
    want = {"x_fma_first": 2, "x_fma_second": 2, "y_fma_first": 2, "y_fma_second": 2}
    while any(v > 0 for v in want.values()):
        # coordinates of the workloads' scale: a few units, both signs, plus some of large exponent spread
        xf = struct.unpack("<f", struct.pack("<f", rng.uniform(-4, 4)))[0]
        yf = struct.unpack("<f", struct.pack("<f", rng.uniform(-4, 4) * (2.0 ** rng.randint(-12, 12))))[0]
        x, y = Fraction(xf), Fraction(yf)
        xs, ys = rotate_separate(x, y)
        fused = rotate_fused_variants(x, y)
        differs = [k for k, v in fused.items() if v != (xs if k.startswith("x") else ys)]
        hit = [k for k in differs if want[k] > 0]
        if not hit:
            continue
        for k in hit:
            want[k] -= 1
        cases.append({
            "in": [f"0x{bits_of(x):08X}", f"0x{bits_of(y):08X}", "0x40400000"],
            "out": [f"0x{bits_of(xs):08X}", f"0x{bits_of(ys):08X}", "0x40400000"],
            "fused_differs": {k: f"0x{bits_of(fused[k]):08X}" for k in differs},
        })
    doc = {
        "source": "Erwin author's thread, the post on cross-partition exchange (rotated trees in place of "
                  "shifted windows); angle, axis and per-operation rounding are the library's stated reading",
        "rule": "x' = rn(rn(c*x) - rn(s*y)), y' = rn(rn(s*x) + rn(c*y)), z' = z, c = s = float bits 0x3F3504F3",
        "derivation": "exact rational products and sums rounded to float32 (nearest, ties to even) by "
                      "tests/golden/make_rotation_cases.py; each case is one where a fused multiply-add "
                      "(listed under fused_differs) gives a different float",
        "cases": cases,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rotation_fma_cases.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    print(f"wrote {len(cases)} cases to {path}")


if __name__ == "__main__":
    main()
