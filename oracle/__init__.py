"""CPU oracle: plain, slow, obviously correct restatement of the hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library; the only thing the two sides share is the seeded input
generator in ``workloads``.

The arithmetic lives in ``oracle.c`` (single-threaded C, compiled with
``-O2 -ffp-contract=off``, no fast-math); this file only marshals numpy arrays.

Pinned functions (each checked by ``tests/test_oracle_*.py`` against worked
examples, brute force, closed forms or a library routine): ``build``,
``rotate_z``, ``ball_attention``, ``full_attention``, ``invert``,
``compose``, ``bsa``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def compile_oracle(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                               "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(compile_oracle())
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.orc_build.argtypes = [P, P, i32, i32, P, P]
        lib.orc_build.restype = ctypes.c_int
        lib.orc_rotate_z.argtypes = [P, i64, P]
        lib.orc_rotate_z.restype = None
        lib.orc_ball_attention.argtypes = [P, P, P, ctypes.c_int, P, i64, i32, i32, i32, P, i64, P]
        lib.orc_ball_attention.restype = ctypes.c_int
        lib.orc_full_attention.argtypes = [P, P, P, ctypes.c_int, i64, i32, i32, P, i64, P]
        lib.orc_full_attention.restype = ctypes.c_int
        lib.orc_invert.argtypes = [P, i64, P, i64]
        lib.orc_invert.restype = None
        lib.orc_compose.argtypes = [P, P, i64, P]
        lib.orc_compose.restype = None
        lib.orc_bsa.argtypes = [P, P, P, ctypes.c_int, P, i64, i64, i32, i32, i32, P, i32, P, P, i32, i32, i32, P,
                                P, i64, P, P, P, P, P, P, P]
        lib.orc_bsa.restype = ctypes.c_int
        lib.orc_pool_mean.argtypes = [P, ctypes.c_int, P, i64, i64, i32, i32, P, P]
        lib.orc_pool_mean.restype = ctypes.c_int
        lib.orc_unpool.argtypes = [P, P, i64, i64, i32, i32, P]
        lib.orc_unpool.restype = ctypes.c_int
        lib.orc_project.argtypes = [P, ctypes.c_int, P, ctypes.c_int, i64, i32, i32, i32, P, P, P]
        lib.orc_project.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    pass


def padded_size(n: int, m: int) -> int:
    leaves = max(1, -(-n // m))
    return m * (1 << (leaves - 1).bit_length())


def build(coords: np.ndarray, m: int, offsets=None):
    """Ball tree of every cloud.  Returns (perm int32 [Npad_total], pad_offsets int64 [B+1]).
    perm[slot] = global row of the point in that slot, -1 for a dummy slot."""
    coords = np.ascontiguousarray(coords, dtype=np.float32)
    n = coords.shape[0]
    offsets = np.array([0, n] if offsets is None else offsets, dtype=np.int64)
    B = len(offsets) - 1
    npad = sum(padded_size(int(offsets[b + 1] - offsets[b]), m) for b in range(B)) if m >= 1 else 0
    perm = np.empty(max(npad, 1), np.int32)
    pad = np.empty(B + 1, np.int64)
    rc = _load().orc_build(_ptr(coords), _ptr(offsets), B, m, _ptr(perm), _ptr(pad))
    if rc != 0:
        raise OracleError(f"orc_build failed with status {rc}")
    return perm[:npad], pad


def rotate_z(coords: np.ndarray) -> np.ndarray:
    coords = np.ascontiguousarray(coords, dtype=np.float32)
    out = np.empty_like(coords)
    _load().orc_rotate_z(_ptr(coords), coords.shape[0], _ptr(out))
    return out


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    if a.dtype == np.float64:
        return 2
    raise TypeError("Q/K/V must be float32, float64 or raw bfloat16 bits (uint16)")


def ball_attention(q, k, v, m: int, perm=None, balls=None, out=None):
    """Ball attention in float64.  q/k/v [rows, H, d] float32 or bf16 bits, original row order.
    perm: slot -> row (or None: identity).  Returns O float64 [rows, H, d] (rows outside the listed
    balls are left as in ``out`` / NaN)."""
    q, k, v = (np.ascontiguousarray(t) for t in (q, k, v))
    rows, H, d = q.shape
    dt = _dtype_code(q)
    npad = rows if perm is None else len(perm)
    perm_a = None if perm is None else np.ascontiguousarray(perm, dtype=np.int32)
    balls_a = None if balls is None else np.ascontiguousarray(balls, dtype=np.int64)
    o = np.full((rows, H, d), np.nan) if out is None else out
    rc = _load().orc_ball_attention(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(perm_a), npad, m, H, d, _ptr(balls_a),
                                    0 if balls_a is None else len(balls_a), _ptr(o))
    if rc != 0:
        raise OracleError(f"orc_ball_attention failed with status {rc}")
    return o


def full_attention(q, k, v, rows=None):
    q, k, v = (np.ascontiguousarray(t) for t in (q, k, v))
    n, H, d = q.shape
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.full((n, H, d), np.nan)
    rc = _load().orc_full_attention(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), n, H, d, _ptr(rows_a),
                                    0 if rows_a is None else len(rows_a), _ptr(o))
    if rc != 0:
        raise OracleError(f"orc_full_attention failed with status {rc}")
    return o


def invert(perm: np.ndarray, n_rows: int) -> np.ndarray:
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    inv = np.empty(n_rows, np.int32)
    _load().orc_invert(_ptr(perm), len(perm), _ptr(inv), n_rows)
    return inv


def compose(invA: np.ndarray, permB: np.ndarray) -> np.ndarray:
    invA = np.ascontiguousarray(invA, dtype=np.int32)
    permB = np.ascontiguousarray(permB, dtype=np.int32)
    out = np.empty(len(permB), np.int32)
    _load().orc_compose(_ptr(invA), _ptr(permB), len(permB), _ptr(out))
    return out


def bsa(q, k, v, m: int, perm, x, w_g, b_g=None, topk: int = 8, mask_own: bool = True, sel_in=None,
        branches: bool = False, groups=None, coarsen: bool = False):
    """Ball Sparse Attention in float64 (see oracle.c, orc_bsa).  Returns O [rows, H, d]; with branches=True
    a dict with O, O_ball, O_cmp, O_slc, gates [rows, H, 3], sel [nb, H, topk] and scores [nb, H, nb].
    coarsen=True is the query-coarsening variant: compression and selection use the group's pooled query."""
    q, k, v = (np.ascontiguousarray(t) for t in (q, k, v))
    rows, H, d = q.shape
    npad = rows if perm is None else len(perm)
    nb = npad // m
    perm_a = None if perm is None else np.ascontiguousarray(perm, dtype=np.int32)
    x = np.ascontiguousarray(x, dtype=np.float32)
    w_g = np.ascontiguousarray(w_g, dtype=np.float32)
    b_a = None if b_g is None else np.ascontiguousarray(b_g, dtype=np.float32)
    sel_a = None if sel_in is None else np.ascontiguousarray(sel_in, dtype=np.int32)
    grp = None if groups is None else np.ascontiguousarray(groups, dtype=np.int64)
    out = {name: np.full((rows, H, d), np.nan) for name in ("O", "O_ball", "O_cmp", "O_slc")}
    out["gates"] = np.full((rows, H, 3), np.nan)
    out["sel"] = np.full((nb, H, topk), -2, np.int32)
    out["scores"] = np.full((nb, H, nb), np.nan)
    rc = _load().orc_bsa(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(perm_a), npad, rows, m, H, d, _ptr(x),
                         x.shape[1], _ptr(w_g), _ptr(b_a), topk, int(mask_own), int(coarsen), _ptr(sel_a), _ptr(grp),
                         0 if grp is None else len(grp), _ptr(out["O"]),
                         _ptr(out["O_ball"]), _ptr(out["O_cmp"]), _ptr(out["O_slc"]), _ptr(out["gates"]),
                         _ptr(out["sel"]), _ptr(out["scores"]))
    if rc != 0:
        raise OracleError(f"orc_bsa failed with status {rc}")
    return out if branches else out["O"]


def pool_mean(x, perm, stride: int, npad: int | None = None):
    """Mean over the real slots of each node `stride` slots wide (see oracle.c, orc_pool_mean).
    x [rows, ...] float32 / float64 / bf16 bits in original row order.  Returns (xc float64
    [npad/stride, ...] in coarse slot order, cperm int32 [npad/stride])."""
    x = np.ascontiguousarray(x)
    rows = x.shape[0]
    C = int(np.prod(x.shape[1:]))
    npad = (rows if perm is None else len(perm)) if npad is None else npad
    perm_a = None if perm is None else np.ascontiguousarray(perm, dtype=np.int32)
    xc = np.full((npad // stride,) + x.shape[1:], np.nan)
    cperm = np.full(npad // stride, -2, np.int32)
    rc = _load().orc_pool_mean(_ptr(x), _dtype_code(x), _ptr(perm_a), npad, rows, C, stride, _ptr(xc), _ptr(cperm))
    if rc != 0:
        raise OracleError(f"orc_pool_mean failed with status {rc}")
    return xc, cperm


def unpool(xc, perm, stride: int, rows: int, out=None):
    """Copy each node's value back to its real slots' rows (see oracle.c, orc_unpool).  Returns
    float64 [rows, ...]; rows no slot names stay NaN (or as in ``out``)."""
    xc = np.ascontiguousarray(xc, dtype=np.float64)
    C = int(np.prod(xc.shape[1:]))
    npad = xc.shape[0] * stride if perm is None else len(perm)
    perm_a = None if perm is None else np.ascontiguousarray(perm, dtype=np.int32)
    o = np.full((rows,) + xc.shape[1:], np.nan) if out is None else out
    rc = _load().orc_unpool(_ptr(xc), _ptr(perm_a), npad, rows, C, stride, _ptr(o))
    if rc != 0:
        raise OracleError(f"orc_unpool failed with status {rc}")
    return o


def coarse_ball_attention(q, k, v, m: int, perm, stride: int):
    """Ball attention `log2(stride)` levels up the tree: Q/K/V mean-pooled over nodes of `stride` slots,
    attention inside balls of m coarse tokens (m*stride slots), and the result copied back to every real
    row of the node.  Returns float64 [rows, H, d]."""
    rows = q.shape[0]
    qc, cperm = pool_mean(q, perm, stride)
    kc, _ = pool_mean(k, perm, stride)
    vc, _ = pool_mean(v, perm, stride)
    oc = ball_attention(qc, kc, vc, m, cperm)
    return unpool(oc, perm, stride, rows)


def project(x, w, H: int, d: int):
    """Q, K, V = X W in float64 (see oracle.c, orc_project).  x [rows, C], w [C, 3*H*d] (float32, float64 or bf16
    bits); returns three float64 arrays [rows, H, d]."""
    x = np.ascontiguousarray(x)
    w = np.ascontiguousarray(w)
    rows, C = x.shape
    q, k, v = (np.full((rows, H, d), np.nan) for _ in range(3))
    rc = _load().orc_project(_ptr(x), _dtype_code(x), _ptr(w), _dtype_code(w), rows, C, H, d, _ptr(q), _ptr(k), _ptr(v))
    if rc != 0:
        raise OracleError(f"orc_project failed with status {rc}")
    return q, k, v


def projected_ball_attention(x, w, H: int, d: int, m: int, perm, balls=None):
    """Ball attention of the projected features: Q, K, V = X W (float64), then attention inside the balls."""
    q, k, v = project(x, w, H, d)
    return ball_attention(q, k, v, m, perm, balls=balls)
