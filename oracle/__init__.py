"""fp64 CPU oracle for the DBF layer forward (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` and ``--impl reference`` legs) may import this package.  The
product path in ``binary_factorized_weight_b200`` never imports it, and this
package never imports the product: the two share no code.  The arithmetic lives
in ``dbf_oracle.c`` (plain C loops, fp64); this module only marshals numpy
arrays into it.

Each function cites the passage of "Addition is almost all you need:
Compressing large language models with double binary factorization" it
follows (gist.science technical summary, section 2.1, and sciencestack.ai
Figure 1).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None


def _setup(lib):
    """Declare the C signatures on a loaded oracle library."""
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    lib.oracle_words_per_row.argtypes = [i64]
    lib.oracle_words_per_row.restype = i64
    lib.oracle_unpack_signs.argtypes = [vp, i64, i64, vp]
    lib.oracle_unpack_signs.restype = i64
    lib.oracle_pack_signs.argtypes = [vp, i64, i64, vp]
    lib.oracle_pack_signs.restype = None
    lib.oracle_forward_staged.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, vp]
    lib.oracle_forward_staged.restype = None
    lib.oracle_forward_transposed.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
    lib.oracle_forward_transposed.restype = None
    lib.oracle_dense_weight.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    lib.oracle_dense_weight.restype = None
    lib.oracle_bqq_dense_weight.argtypes = [vp, vp, vp, vp, vp, dbl, i64, i64, i64, i64, vp]
    lib.oracle_bqq_dense_weight.restype = None
    lib.oracle_forward_dense.argtypes = [vp, vp, i64, i64, i64, vp]
    lib.oracle_forward_dense.restype = None
    lib.oracle_bits_per_weight.argtypes = [i64, i64, i64]
    lib.oracle_bits_per_weight.restype = dbl
    lib.oracle_scale_bits_per_weight.argtypes = [i64, i64, i64]
    lib.oracle_scale_bits_per_weight.restype = dbl
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _setup(ctypes.CDLL(_build.build()))
    return _lib


def use_library(path):
    """Point this module at another build of dbf_oracle.c (used by the tests that
    plant mistakes in a copy of the oracle); returns the previous library."""
    global _lib
    prev = _lib
    _lib = _setup(ctypes.CDLL(path)) if path is not None else None
    return prev


def restore_library(prev):
    global _lib
    _lib = prev


def _f64(a) -> np.ndarray:
    # fp16 -> fp64 widening is exact.
    return np.ascontiguousarray(np.asarray(a), dtype=np.float64)


def _i8(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=np.int8)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads the oracle's loops use (timing only; the results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))


def words_per_row(cols: int) -> int:
    """32-bit words per packed row (rows are padded to whole 256-column blocks of 8 words)."""
    return int(_load().oracle_words_per_row(cols))


def unpack_signs(packed, rows: int, cols: int):
    """Decode the documented packed layout into int8 +-1 (rows x cols).

    Returns (signs, n_set_padding_bits)."""
    lib = _load()
    packed = np.ascontiguousarray(np.asarray(packed), dtype=np.uint32).reshape(-1)
    if packed.size < rows * words_per_row(cols):
        raise ValueError("packed buffer too small")
    out = np.empty((rows, cols), dtype=np.int8)
    bad = lib.oracle_unpack_signs(_ptr(packed), rows, cols, _ptr(out))
    return out, int(bad)


def pack_signs(signs) -> np.ndarray:
    """Encode int8 signs (< 0 -> set bit) into the documented packed layout."""
    lib = _load()
    s = _i8(signs)
    rows, cols = s.shape
    out = np.empty(rows * words_per_row(cols), dtype=np.uint32)
    lib.oracle_pack_signs(_ptr(s), rows, cols, _ptr(out))
    return out


def forward_staged(x, A, B, a, mid, b, return_v: bool = False):
    """((((x (.) b) B^T) (.) mid) A^T) (.) a in fp64 (section 2.1, computation process).

    x: batch x m_in; A: n x k signs; B: k x m_in signs; a: n; mid: k; b: m_in.
    Returns y (batch x n), and v = mid (.) (B (x (.) b)) (batch x k) if asked."""
    lib = _load()
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    A, B = _i8(A), _i8(B)
    a, mid, b = _f64(a), _f64(mid), _f64(b)
    n, k = A.shape
    k2, m_in = B.shape
    batch = x.shape[0]
    if k2 != k or x.shape[1] != m_in or a.size != n or mid.size != k or b.size != m_in:
        raise ValueError("shape mismatch")
    y = np.empty((batch, n), dtype=np.float64)
    v = np.empty((batch, k), dtype=np.float64) if return_v else None
    lib.oracle_forward_staged(_ptr(x), _ptr(A), _ptr(B), _ptr(a), _ptr(mid), _ptr(b), n, k, m_in,
                              batch, _ptr(y), _ptr(v) if v is not None else None)
    return (y, v) if return_v else y


def forward_transposed(dy, A, B, a, mid, b):
    """dx = dy W for W = (a (.) A (.) mid^T)(B (.) b^T), fp64, right to left without forming W
    (the transpose of the forward of section 2.1).  dy: batch x n; returns batch x m_in."""
    lib = _load()
    dy = _f64(dy)
    if dy.ndim == 1:
        dy = dy[None, :]
    A, B = _i8(A), _i8(B)
    a, mid, b = _f64(a), _f64(mid), _f64(b)
    n, k = A.shape
    k2, m_in = B.shape
    batch = dy.shape[0]
    if k2 != k or dy.shape[1] != n or a.size != n or mid.size != k or b.size != m_in:
        raise ValueError("shape mismatch")
    dx = np.empty((batch, m_in), dtype=np.float64)
    lib.oracle_forward_transposed(_ptr(dy), _ptr(A), _ptr(B), _ptr(a), _ptr(mid), _ptr(b), n, k, m_in, batch,
                                  _ptr(dx))
    return dx


def dense_weight(A, B, a, mid, b) -> np.ndarray:
    """W = (a (.) A (.) mid^T)(B (.) b^T), n x m_in, fp64 (section 2.1, factorisation)."""
    lib = _load()
    A, B = _i8(A), _i8(B)
    a, mid, b = _f64(a), _f64(mid), _f64(b)
    n, k = A.shape
    m_in = B.shape[1]
    if B.shape[0] != k or a.size != n or mid.size != k or b.size != m_in:
        raise ValueError("shape mismatch")
    W = np.empty((n, m_in), dtype=np.float64)
    lib.oracle_dense_weight(_ptr(A), _ptr(B), _ptr(a), _ptr(mid), _ptr(b), n, k, m_in, _ptr(W))
    return W


def forward_dense(x, W) -> np.ndarray:
    """y = x W^T with a dense fp64 W."""
    lib = _load()
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    W = _f64(W)
    n, m_in = W.shape
    y = np.empty((x.shape[0], n), dtype=np.float64)
    lib.oracle_forward_dense(_ptr(x), _ptr(W), n, m_in, x.shape[0], _ptr(y))
    return y


def bits_per_weight(n: int, k: int, m_in: int) -> float:
    """Sign bits per dense weight, k(n + m_in)/(n m_in) (section 2.1: k sets the rate)."""
    return float(_load().oracle_bits_per_weight(n, k, m_in))


def scale_bits_per_weight(n: int, k: int, m_in: int) -> float:
    """fp16 scale-vector bits per dense weight, 16(n + k + m_in)/(n m_in)."""
    return float(_load().oracle_scale_bits_per_weight(n, k, m_in))


def bqq_dense_weight(Y, Z, r, s, t, u) -> np.ndarray:
    """W = sum_i (r_i Y_i Z_i + s_i Y_i 1_Z + t_i 1_Y Z_i) + u 1 (sciencestack.ai page of "Binary Quadratic
    Quantization", TL;DR formula), fp64.  Y: p x n x k and Z: p x k x m binary {0, 1}; r, s, t: p; u scalar."""
    lib = _load()
    Y, Z = _i8(Y), _i8(Z)
    if Y.ndim == 2:
        Y, Z = Y[None], Z[None]
    p, n, k = Y.shape
    p2, k2, m = Z.shape
    r, s, t = _f64(r).reshape(-1), _f64(s).reshape(-1), _f64(t).reshape(-1)
    if p2 != p or k2 != k or r.size != p or s.size != p or t.size != p:
        raise ValueError("shape mismatch")
    if Y.size and (Y.min() < 0 or Y.max() > 1) or Z.size and (Z.min() < 0 or Z.max() > 1):
        raise ValueError("Y and Z must hold 0 or 1")
    W = np.empty((n, m), dtype=np.float64)
    lib.oracle_bqq_dense_weight(_ptr(Y), _ptr(Z), _ptr(r), _ptr(s), _ptr(t), float(u), n, k, m, p, _ptr(W))
    return W


def bqq_forward(x, Y, Z, r, s, t, u) -> np.ndarray:
    """y = x W^T for the BQQ weight W of bqq_dense_weight (x: batch x m)."""
    return forward_dense(x, bqq_dense_weight(Y, Z, r, s, t, u))
