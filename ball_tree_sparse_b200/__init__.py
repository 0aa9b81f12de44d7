"""Python binding of libbts.so (ball-tree build + ball attention on B200).

Argument marshalling only: every step runs in the library's CUDA kernels.
The functions carry the names of the C entry points in ``include/bts.h``,
take torch CUDA tensors (torch supplies device memory and the current
stream) and raise :class:`BtsError` on a non-OK status.  There is no CPU
fallback: importing fails loudly when the compiled library is missing.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbts.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libbts.so not found at {LIB_PATH}; build it with "
                      "`python -m ball_tree_sparse_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

STATUS = {0: "BT_OK", 1: "BT_ERR_ARG", 2: "BT_ERR_SHAPE", 3: "BT_ERR_NONFINITE", 4: "BT_ERR_WORKSPACE",
          5: "BT_ERR_CUDA", 6: "BT_ERR_TIMEOUT", 7: "BT_ERR_UNSUPPORTED",
          8: "BT_ERR_INTERNAL"}
BT_F32, BT_BF16 = 0, 1
MAX_CLOUDS = 64

_P, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
_SIGS = {
    "bt_version": ([], ctypes.c_int32),
    "bt_build_workspace_size": ([_P, _i32, _i32], _sz),
    "bt_build": ([_P, _i64, _i32, _P, _P, _sz, _P], ctypes.c_int),
    "bt_build_segmented": ([_P, _P, _i32, _i32, _P, _P, _P, _sz, _P], ctypes.c_int),
    "bt_build_segmented_ex": ([_P, _P, _i32, _i32, _P, _P, _P, _sz, ctypes.c_uint32, _P], ctypes.c_int),
    "bt_build_device_status": ([_P, _P], ctypes.c_int),
    "bt_build_noalloc": ([_P, _i64, _i32, _P, _P, _P], ctypes.c_int),
    "bt_rotate_z": ([_P, _i64, _P, _P], ctypes.c_int),
    "bt_invert_perm": ([_P, _i64, _i64, _P, _P], ctypes.c_int),
    "bt_compose": ([_P, _P, _i64, _P, _P], ctypes.c_int),
    "bt_gather": ([_P, _P, _i64, _i32, _P, _P], ctypes.c_int),
    "bt_scatter": ([_P, _P, _i64, _i32, _P, _P], ctypes.c_int),
    "bt_ball_attention": ([_P, _P, _P, _P, _i64, _i64, _i32, _i32, _i32, ctypes.c_int, _P, _P], ctypes.c_int),
    "bt_qkv_project": ([_P, _i64, _i32, _P, _i32, _i32, ctypes.c_int, _P, _P, _i64, _P, _P, _P, _P], ctypes.c_int),
    "bt_ball_attention_tree": ([_P, _P, _P, _P, _i64, _i64, _i32, _i32, _i32, ctypes.c_int, _P, _P], ctypes.c_int),
    "bt_projected_workspace_size": ([_i64, _i64, _i32, _i32, ctypes.c_int], _sz),
    "bt_projected_ball_attention": ([_P, _P, _i64, _i64, _i32, _P, _i32, _i32, _i32, ctypes.c_int, _P, _P, _sz, _P],
                                    ctypes.c_int),
    "bt_attention_device_status": ([_P], ctypes.c_int),
    "bt_last_device_status": ([_P], ctypes.c_int),
    "bsa_workspace_size": ([_i64, _i64, _i32, _i32, _i32, _i32], _sz),
    "bsa_forward": ([_P, _P, _P, _P, _i64, _i64, _i32, _i32, _i32, ctypes.c_int, _P, _i32, _P, _P, None, _P, _P,
                     _P, _sz, _P], ctypes.c_int),
    "bt_pool_mean": ([_P, _P, _i64, _i64, _i32, _i32, ctypes.c_int, _P, _P, _P], ctypes.c_int),
    "bt_unpool": ([_P, _P, _i64, _i64, _i32, _i32, ctypes.c_int, _P, _P], ctypes.c_int),
    "bt_coarse_workspace_size": ([_i64, _i32, _i32, _i32, ctypes.c_int], _sz),
    "bt_coarse_ball_attention": ([_P, _P, _P, _P, _i64, _i64, _i32, _i32, _i32, ctypes.c_int, _i32, _P, _P, _sz,
                                  _P], ctypes.c_int),
}


class bsa_params(ctypes.Structure):
    _fields_ = [("topk", ctypes.c_int32), ("mask_own_ball", ctypes.c_int32), ("coarsen_queries", ctypes.c_int32)]


_SIGS["bsa_forward"][0][14] = bsa_params
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTED = tuple(_SIGS)


class BtsError(RuntimeError):
    def __init__(self, call: str, code: int):
        super().__init__(f"{call} returned {STATUS.get(code, code)}")
        self.code = code
        self.status = STATUS.get(code, str(code))


def _check(call: str, code: int) -> None:
    if code != 0:
        raise BtsError(call, code)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _offsets_array(offsets) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))


def bt_version() -> int:
    return int(_lib.bt_version())


version = bt_version


def bt_build_workspace_size(offsets, m: int) -> int:
    off = _offsets_array(offsets)
    return int(_lib.bt_build_workspace_size(off.ctypes.data_as(_P), len(off) - 1, m))


def workspace(offsets, m: int, device=None) -> torch.Tensor:
    """A workspace tensor of the size bt_build_workspace_size() asks for (torch allocates it)."""
    n = bt_build_workspace_size(offsets, m)
    if n == 0:
        raise BtsError("bt_build_workspace_size", 1)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def bt_build(coords: torch.Tensor, m: int, perm: torch.Tensor | None = None, ws: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """Ball tree of one cloud of N = m * 2^L points: returns perm int32 [N] (slot -> row)."""
    N = coords.shape[0]
    if perm is None:
        perm = torch.empty(N, dtype=torch.int32, device=coords.device)
    if ws is None:
        ws = workspace([0, N], m, coords.device)
    _check("bt_build", _lib.bt_build(_dptr(coords), N, m, _dptr(perm), _dptr(ws), ws.numel(), _stream(stream)))
    return perm


def bt_build_segmented(coords: torch.Tensor, offsets, m: int, perm: torch.Tensor | None = None,
                       ws: torch.Tensor | None = None, stream=None):
    """Ball trees of a batch of clouds (padded with dummies).  Returns (perm int32 [sum Npad], pad_offsets)."""
    return _segmented("bt_build_segmented", coords, offsets, m, perm, ws, stream)


BT_BUILD_NARROW = 1


def bt_build_segmented_ex(coords: torch.Tensor, offsets, m: int, flags: int = 0, perm: torch.Tensor | None = None,
                          ws: torch.Tensor | None = None, stream=None):
    """bt_build_segmented with flags (BT_BUILD_NARROW: half the SMs per cloud, for a build beside other
    kernels); the result does not depend on the flags."""
    return _segmented("bt_build_segmented_ex", coords, offsets, m, perm, ws, stream, flags)


def _segmented(name, coords, offsets, m, perm, ws, stream, *flags):
    off = _offsets_array(offsets)
    B = len(off) - 1
    pad = np.zeros(B + 1, np.int64)
    if perm is None:
        sizes = [_padded(int(off[b + 1] - off[b]), m) for b in range(B)]
        perm = torch.empty(sum(sizes), dtype=torch.int32, device=coords.device)
    if ws is None:
        ws = workspace(off, m, coords.device)
    _check(name, getattr(_lib, name)(_dptr(coords), off.ctypes.data_as(_P), B, m, _dptr(perm),
                                     pad.ctypes.data_as(_P), _dptr(ws), ws.numel(), *flags, _stream(stream)))
    return perm, pad


def _padded(n: int, m: int) -> int:
    leaves = max(1, -(-n // m))
    return m * (1 << (leaves - 1).bit_length())


def bt_build_noalloc(coords: torch.Tensor, m: int, perm: torch.Tensor, status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """bt_build with the library's own static scratch (N <= 65,536); allocates nothing."""
    _check("bt_build_noalloc", _lib.bt_build_noalloc(_dptr(coords), coords.shape[0], m, _dptr(perm),
                                                     _dptr(status), _stream(stream)))
    return perm


def bt_build_device_status(ws: torch.Tensor, stream=None) -> int:
    return int(_lib.bt_build_device_status(_dptr(ws), _stream(stream)))


def bt_rotate_z(coords: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty_like(coords)
    _check("bt_rotate_z", _lib.bt_rotate_z(_dptr(coords), coords.shape[0], _dptr(out), _stream(stream)))
    return out


def bt_invert_perm(perm: torch.Tensor, n_rows: int, inv: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if inv is None:
        inv = torch.empty(n_rows, dtype=torch.int32, device=perm.device)
    _check("bt_invert_perm", _lib.bt_invert_perm(_dptr(perm), perm.numel(), n_rows, _dptr(inv), _stream(stream)))
    return inv


def bt_compose(invA: torch.Tensor, permB: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    if out is None:
        out = torch.empty_like(permB)
    _check("bt_compose", _lib.bt_compose(_dptr(invA), _dptr(permB), permB.numel(), _dptr(out), _stream(stream)))
    return out


def bt_gather(X: torch.Tensor, idx: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y[s] = X[idx[s]] (zero row where idx[s] < 0); rows are X's trailing dimensions."""
    npad = idx.numel()
    if out is None:
        out = torch.empty((npad, *X.shape[1:]), dtype=X.dtype, device=X.device)
    row_bytes = X[0].numel() * X.element_size() if X.shape[0] else out[0].numel() * out.element_size()
    _check("bt_gather", _lib.bt_gather(_dptr(X), _dptr(idx), npad, row_bytes, _dptr(out), _stream(stream)))
    return out


def bt_scatter(Y: torch.Tensor, idx: torch.Tensor, X: torch.Tensor, stream=None) -> torch.Tensor:
    """X[idx[s]] = Y[s] for idx[s] >= 0."""
    npad = idx.numel()
    row_bytes = Y[0].numel() * Y.element_size()
    _check("bt_scatter", _lib.bt_scatter(_dptr(Y), _dptr(idx), npad, row_bytes, _dptr(X), _stream(stream)))
    return X


def bt_ball_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, perm: torch.Tensor | None, m: int,
                      out: torch.Tensor | None = None, npad: int | None = None, stream=None) -> torch.Tensor:
    """Attention inside every ball of m slots.  Q/K/V/O [rows, H, d] fp32 or bf16 in original row order;
    perm int32 [npad] slot -> row (-1 dummy) or None (row s in slot s)."""
    rows, H, d = Q.shape
    if Q.dtype == torch.float32:
        dt = BT_F32
    elif Q.dtype == torch.bfloat16:
        dt = BT_BF16
    else:
        raise TypeError("Q/K/V must be float32 or bfloat16")
    if not (K.dtype == V.dtype == Q.dtype):
        raise TypeError("Q, K and V must share one dtype")
    if npad is None:
        npad = perm.numel() if perm is not None else rows
    if out is None:
        out = torch.empty_like(Q)
    _check("bt_ball_attention",
           _lib.bt_ball_attention(_dptr(Q), _dptr(K), _dptr(V), _dptr(perm), npad, rows, m, H, d, dt,
                                  _dptr(out), _stream(stream)))
    return out


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BT_F32
    if t.dtype == torch.bfloat16:
        return BT_BF16
    raise TypeError("tensors must be float32 or bfloat16")


def bt_pool_mean(X: torch.Tensor, perm: torch.Tensor | None, stride: int, out: torch.Tensor | None = None,
                 cperm: torch.Tensor | None = None, npad: int | None = None, stream=None):
    """Mean over the real slots of every node `stride` slots wide.  X [rows, ...] in original row order; returns
    (Xc [npad/stride, ...] in coarse slot order, cperm int32 [npad/stride]: j, or -1 for a node of dummies)."""
    rows = X.shape[0]
    C = X[0].numel() if rows else 1
    if npad is None:
        npad = perm.numel() if perm is not None else rows
    nc = npad // stride
    if out is None:
        out = torch.empty((nc, *X.shape[1:]), dtype=X.dtype, device=X.device)
    if cperm is None:
        cperm = torch.empty(nc, dtype=torch.int32, device=X.device)
    _check("bt_pool_mean", _lib.bt_pool_mean(_dptr(X), _dptr(perm), npad, rows, C, stride, _dt(X), _dptr(out),
                                             _dptr(cperm), _stream(stream)))
    return out, cperm


def bt_unpool(Xc: torch.Tensor, perm: torch.Tensor | None, stride: int, X: torch.Tensor, npad: int | None = None,
              stream=None) -> torch.Tensor:
    """X[perm[s]] = Xc[s // stride] for every real slot s; X [rows, ...] original row order (written in place)."""
    rows = X.shape[0]
    C = X[0].numel() if rows else 1
    if npad is None:
        npad = perm.numel() if perm is not None else Xc.shape[0] * stride
    _check("bt_unpool", _lib.bt_unpool(_dptr(Xc), _dptr(perm), npad, rows, C, stride, _dt(X), _dptr(X),
                                       _stream(stream)))
    return X


def bt_coarse_workspace_size(npad: int, H: int, d: int, stride: int, dtype: torch.dtype) -> int:
    return int(_lib.bt_coarse_workspace_size(npad, H, d, stride, BT_F32 if dtype == torch.float32 else BT_BF16))


def bt_coarse_ball_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, perm: torch.Tensor | None, m: int,
                             stride: int, out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                             npad: int | None = None, stream=None) -> torch.Tensor:
    """Ball attention log2(stride) levels up the tree: Q/K/V pooled to nodes of `stride` slots, attention in balls
    of m coarse tokens, each node's output copied back to its real rows.  Q/K/V/O [rows, H, d]."""
    rows, H, d = Q.shape
    if not (K.dtype == V.dtype == Q.dtype):
        raise TypeError("Q, K and V must share one dtype")
    if npad is None:
        npad = perm.numel() if perm is not None else rows
    if out is None:
        out = torch.empty_like(Q)
    if ws is None:
        n = bt_coarse_workspace_size(npad, H, d, stride, Q.dtype)
        if n == 0:
            raise BtsError("bt_coarse_workspace_size", 1)
        ws = torch.empty(n, dtype=torch.uint8, device=Q.device)
    _check("bt_coarse_ball_attention",
           _lib.bt_coarse_ball_attention(_dptr(Q), _dptr(K), _dptr(V), _dptr(perm), npad, rows, m, H, d, _dt(Q),
                                         stride, _dptr(out), _dptr(ws), ws.numel(), _stream(stream)))
    return out


def bt_qkv_project(X: torch.Tensor, Wt: torch.Tensor, H: int, d: int, perm: torch.Tensor | None = None,
                   inv: torch.Tensor | None = None, out=None, stream=None):
    """Q, K, V = X Wt^T.  X [rows, C] original order; Wt [3*H*d, C].  With perm (slot -> row) the outputs are
    [npad, H, d] in slot order (row r at slot inv[r]; zeros for dummy slots) and inv is computed when not given;
    without, [rows, H, d] in the original order."""
    rows, C = X.shape
    npad = perm.numel() if perm is not None else rows
    if perm is not None and inv is None:
        inv = bt_invert_perm(perm, rows, stream=stream)
    if out is None:
        out = tuple(torch.empty((npad, H, d), dtype=X.dtype, device=X.device) for _ in range(3))
    Q, K, V = out
    _check("bt_qkv_project", _lib.bt_qkv_project(_dptr(X), rows, C, _dptr(Wt), H, d, _dt(X), _dptr(perm), _dptr(inv),
                                                 npad, _dptr(Q), _dptr(K), _dptr(V), _stream(stream)))
    return Q, K, V


def bt_ball_attention_tree(Qt: torch.Tensor, Kt: torch.Tensor, Vt: torch.Tensor, perm: torch.Tensor, m: int,
                           rows: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Ball attention of slot-ordered Q/K/V [npad, H, d]; O [rows, H, d] in the original order."""
    npad, H, d = Qt.shape
    if out is None:
        out = torch.empty((rows, H, d), dtype=Qt.dtype, device=Qt.device)
    _check("bt_ball_attention_tree",
           _lib.bt_ball_attention_tree(_dptr(Qt), _dptr(Kt), _dptr(Vt), _dptr(perm), npad, rows, m, H, d, _dt(Qt),
                                       _dptr(out), _stream(stream)))
    return out


def bt_projected_workspace_size(npad: int, rows: int, H: int, d: int, dtype: torch.dtype) -> int:
    return int(_lib.bt_projected_workspace_size(npad, rows, H, d, BT_F32 if dtype == torch.float32 else BT_BF16))


def bt_projected_ball_attention(X: torch.Tensor, perm: torch.Tensor | None, Wt: torch.Tensor, m: int, H: int, d: int,
                                out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                                npad: int | None = None, stream=None) -> torch.Tensor:
    """One attention layer from the features: Q/K/V = X Wt^T (in slot order where the tile kernel takes the shape),
    then ball attention.  X [rows, C]; Wt [3*H*d, C]; returns O [rows, H, d] in the original order."""
    rows, C = X.shape
    if npad is None:
        npad = perm.numel() if perm is not None else rows
    if out is None:
        out = torch.empty((rows, H, d), dtype=X.dtype, device=X.device)
    if ws is None:
        n = bt_projected_workspace_size(npad, rows, H, d, X.dtype)
        if n == 0:
            raise BtsError("bt_projected_workspace_size", 1)
        ws = torch.empty(n, dtype=torch.uint8, device=X.device)
    _check("bt_projected_ball_attention",
           _lib.bt_projected_ball_attention(_dptr(X), _dptr(perm), npad, rows, C, _dptr(Wt), m, H, d, _dt(X),
                                            _dptr(out), _dptr(ws), ws.numel(), _stream(stream)))
    return out


def bt_last_device_status(stream=None) -> int:
    """First device-side error of the library's work on `stream` since the last call (synchronises it)."""
    return int(_lib.bt_last_device_status(_stream(stream)))


def bt_attention_device_status(stream=None) -> int:
    return int(_lib.bt_attention_device_status(_stream(stream)))


def bsa_workspace_size(npad: int, rows: int, m: int, H: int, d: int, topk: int) -> int:
    return int(_lib.bsa_workspace_size(npad, rows, m, H, d, topk))


def bsa_forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, perm: torch.Tensor | None, m: int,
                X: torch.Tensor, Wg: torch.Tensor, bg: torch.Tensor | None = None, topk: int = 8,
                mask_own_ball: bool = True, out: torch.Tensor | None = None, sel: torch.Tensor | None = None,
                ws: torch.Tensor | None = None, npad: int | None = None, stream=None,
                coarsen_queries: bool = False) -> torch.Tensor:
    """Ball Sparse Attention: ball + compression + top-k selection branches mixed by sigmoid gates.
    Q/K/V/O bf16 [rows, H, d] in original row order; X float [rows, C]; Wg float [C, 3H].
    coarsen_queries=True: compression and selection attend with each group's pooled query."""
    rows, H, d = Q.shape
    if Q.dtype != torch.bfloat16:
        raise TypeError("bsa_forward takes bfloat16 Q/K/V")
    if npad is None:
        npad = perm.numel() if perm is not None else rows
    if out is None:
        out = torch.empty_like(Q)
    if ws is None:
        n = bsa_workspace_size(npad, rows, m, H, d, topk)
        if n == 0:
            raise BtsError("bsa_workspace_size", 2)
        ws = torch.empty(n, dtype=torch.uint8, device=Q.device)
    _check("bsa_forward",
           _lib.bsa_forward(_dptr(Q), _dptr(K), _dptr(V), _dptr(perm), npad, rows, m, H, d, BT_BF16, _dptr(X),
                            X.shape[1], _dptr(Wg), _dptr(bg), bsa_params(topk, int(mask_own_ball), int(coarsen_queries)),
                            _dptr(out),
                            _dptr(sel), _dptr(ws), ws.numel(), _stream(stream)))
    return out
