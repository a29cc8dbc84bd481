"""DBF (Double Binary Factorization) layer forward on B200: Python binding.

A thin ctypes binding of ``libdbf.so`` (C ABI in ``include/dbf.h``).  Every
function here only marshals torch tensors into pointers, sizes and the current
CUDA stream; all computation runs in the library's sm_100a kernels.  There is
no CPU or library fallback: if ``libdbf.so`` is missing the import of the
binding's functions raises, and a call on a machine without a B200 returns the
library's error as :class:`DBFError`.

    y = W x with W = (a (.) A (.) m^T)(B (.) b^T)  ("Addition is almost all you
    need", gist.science technical summary section 2.1), evaluated as
    ((((x (.) b) B^T) (.) m) A^T) (.) a without forming W.

Build the library with ``python -m binary_factorized_weight_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "DBFError",
    "DBF_I8", "DBF_F16", "DBF_F32",
    "DBF_FWD_WEIGHTS_STATIC", "DBF_FWD_FORCE_DECODE", "DBF_FWD_FORCE_PREFILL", "DBF_FWD_DECODE_SHIFT_EXPAND",
    "DBF_FWD_DECODE_TWO_STAGE", "DBF_FWD_DECODE_SINGLE", "DBF_FWD_DECODE_TABLE", "DBF_FWD_TEST_LOSE_ARRIVAL",
    "EXPORTED_SYMBOLS",
    "library_path", "load_library",
    "dbf_packed_words_per_row", "dbf_packed_words", "dbf_pack_signs",
    "dbf_forward_workspace_bytes", "dbf_new_workspace", "dbf_forward",
    "dbf_reconstruct_dense", "dbf_workspace_status", "dbf_status_string", "dbf_forward_noalloc",
    "dbf_noalloc_status",
    "DBF_MAX_GROUP", "dbf_forward_grouped_workspace_bytes", "dbf_new_grouped_workspace", "dbf_forward_grouped",
    "dbf_transpose_signs", "dbf_forward_transposed",
    "dbf_bqq_prepared_bytes", "dbf_bqq_prepare", "dbf_bqq_workspace_bytes", "dbf_bqq_forward",
    "dbf_factorize_workspace_bytes", "dbf_factorize_start", "dbf_factorize_pass", "dbf_factorize_finish", "dbf_svid",
    "dbf_factorize",
]

DBF_I8, DBF_F16, DBF_F32 = 0, 1, 2
DBF_FWD_WEIGHTS_STATIC = 1 << 0
DBF_FWD_FORCE_DECODE = 1 << 1
DBF_FWD_FORCE_PREFILL = 1 << 2
DBF_FWD_DECODE_SHIFT_EXPAND = 1 << 3
DBF_FWD_DECODE_TWO_STAGE = 1 << 4
DBF_FWD_DECODE_SINGLE = 1 << 5
DBF_FWD_DECODE_TABLE = 1 << 6
DBF_FWD_TEST_LOSE_ARRIVAL = 1 << 30  # test only: makes a bounded device wait run out

STATUS_NAMES = {
    0: "DBF_OK", 1: "DBF_ERR_INVALID_ARG", 2: "DBF_ERR_UNSUPPORTED_SHAPE", 3: "DBF_ERR_MISALIGNED",
    4: "DBF_ERR_WORKSPACE", 5: "DBF_ERR_CUDA", 6: "DBF_ERR_TIMEOUT", 7: "DBF_ERR_DEVICE",
}

EXPORTED_SYMBOLS = (
    "dbf_packed_words_per_row",
    "dbf_packed_words",
    "dbf_pack_signs",
    "dbf_forward_workspace_bytes",
    "dbf_forward",
    "dbf_reconstruct_dense",
    "dbf_workspace_status",
    "dbf_forward_noalloc",
    "dbf_noalloc_status",
    "dbf_forward_grouped_workspace_bytes",
    "dbf_forward_grouped",
    "dbf_transpose_signs",
    "dbf_forward_transposed",
    "dbf_bqq_prepared_bytes",
    "dbf_bqq_prepare",
    "dbf_bqq_workspace_bytes",
    "dbf_bqq_forward",
    "dbf_factorize_workspace_bytes",
    "dbf_factorize_start",
    "dbf_factorize_pass",
    "dbf_factorize_finish",
    "dbf_svid_workspace_bytes",
    "dbf_svid",
    "dbf_status_string",
)

DBF_MAX_GROUP = 8


class _LayerDesc(ctypes.Structure):
    """struct dbf_layer_desc of include/dbf.h."""
    _fields_ = [
        ("packedA", ctypes.c_void_p), ("packedB", ctypes.c_void_p),
        ("a", ctypes.c_void_p), ("m", ctypes.c_void_p), ("b", ctypes.c_void_p),
        ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("y", ctypes.c_void_p),
    ]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


class DBFError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        super().__init__(f"{func} failed: {dbf_status_string(status)}")


def library_path() -> str:
    return os.path.join(_HERE, "libdbf.so")


def load_library():
    """Load libdbf.so (built in-tree) and declare its signatures."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m binary_factorized_weight_b200.build`")
    lib = ctypes.CDLL(path)
    i64, u32, i32, vp, sz = ctypes.c_int64, ctypes.c_uint32, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    lib.dbf_packed_words_per_row.argtypes = [i64]
    lib.dbf_packed_words_per_row.restype = i64
    lib.dbf_packed_words.argtypes = [i64, i64]
    lib.dbf_packed_words.restype = i64
    lib.dbf_pack_signs.argtypes = [vp, i32, i64, i64, vp, vp]
    lib.dbf_pack_signs.restype = i32
    lib.dbf_forward_workspace_bytes.argtypes = [i64, i64, i64, i64]
    lib.dbf_forward_workspace_bytes.restype = sz
    lib.dbf_forward.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, vp, sz, u32, vp]
    lib.dbf_forward.restype = i32
    lib.dbf_reconstruct_dense.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, i32, vp]
    lib.dbf_reconstruct_dense.restype = i32
    lib.dbf_workspace_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
    lib.dbf_workspace_status.restype = i32
    lib.dbf_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, u32, vp]
    lib.dbf_forward_noalloc.restype = i32
    lib.dbf_noalloc_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.dbf_noalloc_status.restype = i32
    lib.dbf_forward_grouped_workspace_bytes.argtypes = [ctypes.POINTER(_LayerDesc), i32, i64, i64]
    lib.dbf_forward_grouped_workspace_bytes.restype = sz
    lib.dbf_forward_grouped.argtypes = [vp, i64, i64, ctypes.POINTER(_LayerDesc), i32, i32, vp, sz, u32, vp]
    lib.dbf_forward_grouped.restype = i32
    lib.dbf_transpose_signs.argtypes = [vp, i64, i64, vp, vp]
    lib.dbf_transpose_signs.restype = i32
    lib.dbf_forward_transposed.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i32, vp, sz, u32, vp]
    lib.dbf_forward_transposed.restype = i32
    lib.dbf_bqq_prepared_bytes.argtypes = [i64, i64, i64, i64]
    lib.dbf_bqq_prepared_bytes.restype = sz
    lib.dbf_bqq_prepare.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, sz, vp]
    lib.dbf_bqq_prepare.restype = i32
    lib.dbf_bqq_workspace_bytes.argtypes = [i64, i64, i64, i64, i64]
    lib.dbf_bqq_workspace_bytes.restype = sz
    lib.dbf_bqq_forward.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, vp, i32, vp, sz, u32, vp]
    lib.dbf_bqq_forward.restype = i32
    lib.dbf_factorize_workspace_bytes.argtypes = [i64, i64, i64]
    lib.dbf_factorize_workspace_bytes.restype = sz
    lib.dbf_factorize_start.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp, sz, vp]
    lib.dbf_factorize_start.restype = i32
    lib.dbf_factorize_pass.argtypes = [vp, i64, i64, i64, vp, vp, i32, vp, vp, sz, vp]
    lib.dbf_factorize_pass.restype = i32
    lib.dbf_factorize_finish.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dbf_factorize_finish.restype = i32
    lib.dbf_svid_workspace_bytes.argtypes = [i64, i64]
    lib.dbf_svid_workspace_bytes.restype = sz
    lib.dbf_svid.argtypes = [vp, i64, i64, vp, vp, vp, vp, sz, vp]
    lib.dbf_svid.restype = i32
    lib.dbf_status_string.argtypes = [i32]
    lib.dbf_status_string.restype = ctypes.c_char_p
    _LIB = lib
    return lib


def _check(func: str, status: int):
    if status != 0:
        raise DBFError(func, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.int8:
        return DBF_I8
    if dtype == torch.float16:
        return DBF_F16
    if dtype == torch.float32:
        return DBF_F32
    raise TypeError(f"unsupported dtype {dtype}")


def dbf_status_string(status: int) -> str:
    try:
        return load_library().dbf_status_string(int(status)).decode()
    except ImportError:
        return STATUS_NAMES.get(int(status), "unknown dbf_status")


def dbf_packed_words_per_row(cols: int) -> int:
    return int(load_library().dbf_packed_words_per_row(int(cols)))


def dbf_packed_words(rows: int, cols: int) -> int:
    return int(load_library().dbf_packed_words(int(rows), int(cols)))


def dbf_pack_signs(src: torch.Tensor, packed: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pack a rows x cols sign matrix (int8/fp16/fp32 CUDA tensor; < 0 -> -1).

    Returns an int32 CUDA tensor holding the packed 32-bit words."""
    if src.dim() != 2 or not src.is_contiguous():
        raise ValueError("src must be a contiguous 2-D tensor")
    rows, cols = src.shape
    n_words = dbf_packed_words(rows, cols)
    if packed is None:
        packed = torch.empty(n_words, dtype=torch.int32, device=src.device)
    elif packed.numel() < n_words or packed.dtype != torch.int32:
        raise ValueError("packed must be an int32 tensor of dbf_packed_words(rows, cols) words")
    _check("dbf_pack_signs", load_library().dbf_pack_signs(
        _ptr(src), _dtype_code(src.dtype), rows, cols, _ptr(packed), _stream(stream)))
    return packed


def dbf_forward_workspace_bytes(n: int, k: int, m_in: int, batch: int) -> int:
    return int(load_library().dbf_forward_workspace_bytes(int(n), int(k), int(m_in), int(batch)))


def dbf_new_workspace(n: int, k: int, m_in: int, batch: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size dbf_forward needs (uint8 CUDA tensor)."""
    return torch.zeros(dbf_forward_workspace_bytes(n, k, m_in, batch), dtype=torch.uint8, device=device)


def dbf_forward(x: torch.Tensor, packedA: torch.Tensor, packedB: torch.Tensor, a: torch.Tensor, m: torch.Tensor,
                b: torch.Tensor, n: int, k: int, m_in: int, y: Optional[torch.Tensor] = None,
                y_dtype: torch.dtype = torch.float16, workspace: Optional[torch.Tensor] = None, flags: int = 0,
                stream=None) -> torch.Tensor:
    """y = ((((x (.) b) B^T) (.) m) A^T) (.) a for fp16 x (batch x m_in); returns y (batch x n)."""
    if x.dtype != torch.float16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp16 batch x m_in tensor")
    batch = x.shape[0]
    if x.shape[1] != m_in:
        raise ValueError("x.shape[1] != m_in")
    if y is None:
        y = torch.empty((batch, n), dtype=y_dtype, device=x.device)
    if workspace is None:
        workspace = dbf_new_workspace(n, k, m_in, batch, device=x.device)
    y_code = _dtype_code(y.dtype)
    _check("dbf_forward", load_library().dbf_forward(
        _ptr(x), _ptr(packedA), _ptr(packedB), _ptr(a), _ptr(m), _ptr(b), int(n), int(k), int(m_in), int(batch),
        _ptr(y), y_code, _ptr(workspace), workspace.numel() * workspace.element_size(), int(flags), _stream(stream)))
    return y


def dbf_forward_noalloc(x: torch.Tensor, packedA: torch.Tensor, packedB: torch.Tensor, a: torch.Tensor,
                        m: torch.Tensor, b: torch.Tensor, n: int, k: int, m_in: int, y: Optional[torch.Tensor] = None,
                        y_dtype: torch.dtype = torch.float16, flags: int = 0, stream=None) -> torch.Tensor:
    """dbf_forward without a workspace, for callers that cannot allocate device memory.

    The library's own 2 MiB buffer stands in for the workspace (limit: 256 + batch*k*2
    bytes); every call shares it, so calls that overlap on the GPU race.  The first call
    on a device looks the buffer up; make it before any stream capture."""
    if x.dtype != torch.float16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp16 batch x m_in tensor")
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, n), dtype=y_dtype, device=x.device)
    _check("dbf_forward_noalloc", load_library().dbf_forward_noalloc(
        _ptr(x), _ptr(packedA), _ptr(packedB), _ptr(a), _ptr(m), _ptr(b), int(n), int(k), int(m_in), int(batch),
        _ptr(y), _dtype_code(y.dtype), int(flags), _stream(stream)))
    return y


def dbf_noalloc_status(stream=None) -> int:
    """Status word of dbf_forward_noalloc's library buffer on the current device (synchronises the stream)."""
    out = ctypes.c_int32(0)
    _check("dbf_noalloc_status", load_library().dbf_noalloc_status(_stream(stream), ctypes.byref(out)))
    return int(out.value)


def dbf_reconstruct_dense(packedA: torch.Tensor, packedB: torch.Tensor, a: torch.Tensor, m: torch.Tensor,
                          b: torch.Tensor, n: int, k: int, m_in: int, W: Optional[torch.Tensor] = None,
                          W_dtype: torch.dtype = torch.float32, stream=None) -> torch.Tensor:
    """Dense W = (a (.) A (.) m^T)(B (.) b^T), n x m_in."""
    if W is None:
        W = torch.empty((n, m_in), dtype=W_dtype, device=a.device)
    _check("dbf_reconstruct_dense", load_library().dbf_reconstruct_dense(
        _ptr(packedA), _ptr(packedB), _ptr(a), _ptr(m), _ptr(b), int(n), int(k), int(m_in), _ptr(W),
        _dtype_code(W.dtype), _stream(stream)))
    return W


def dbf_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """The workspace's device status word (0, or the dbf_status of the first device-side failure)."""
    out = ctypes.c_int32(0)
    _check("dbf_workspace_status", load_library().dbf_workspace_status(
        _ptr(workspace), _stream(stream), ctypes.byref(out)))
    return int(out.value)


def _layer_array(layers, ys=None):
    arr = (_LayerDesc * len(layers))()
    for i, L in enumerate(layers):
        y = None if ys is None else ys[i]
        arr[i] = _LayerDesc(L["packedA"].data_ptr(), L["packedB"].data_ptr(), L["a"].data_ptr(), L["m"].data_ptr(),
                            L["b"].data_ptr(), int(L["n"]), int(L["k"]), None if y is None else y.data_ptr())
    return arr


def dbf_forward_grouped_workspace_bytes(layers, m_in: int, batch: int) -> int:
    """Workspace bytes for dbf_forward_grouped over `layers` (dicts with at least n and k)."""
    arr = (_LayerDesc * len(layers))()
    for i, L in enumerate(layers):
        arr[i].n, arr[i].k = int(L["n"]), int(L["k"])
    return int(load_library().dbf_forward_grouped_workspace_bytes(arr, len(layers), int(m_in), int(batch)))


def dbf_new_grouped_workspace(layers, m_in: int, batch: int, device="cuda") -> torch.Tensor:
    return torch.zeros(dbf_forward_grouped_workspace_bytes(layers, m_in, batch), dtype=torch.uint8, device=device)


def dbf_forward_grouped(x: torch.Tensor, layers, m_in: int, ys=None, y_dtype: torch.dtype = torch.float16,
                        workspace: Optional[torch.Tensor] = None, flags: int = 0, stream=None):
    """Layers that share the input x: layers is a list of dicts with packedA, packedB, a, m, b (CUDA tensors)
    and n, k; returns the list of outputs (batch x n_g each)."""
    if x.dtype != torch.float16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp16 batch x m_in tensor")
    batch = x.shape[0]
    if x.shape[1] != m_in:
        raise ValueError("x.shape[1] != m_in")
    if ys is None:
        ys = [torch.empty((batch, int(L["n"])), dtype=y_dtype, device=x.device) for L in layers]
    if workspace is None:
        workspace = dbf_new_grouped_workspace(layers, m_in, batch, device=x.device)
    arr = _layer_array(layers, ys)
    _check("dbf_forward_grouped", load_library().dbf_forward_grouped(
        _ptr(x), int(m_in), int(batch), arr, len(layers), _dtype_code(ys[0].dtype), _ptr(workspace),
        workspace.numel() * workspace.element_size(), int(flags), _stream(stream)))
    return ys


def dbf_transpose_signs(packed: torch.Tensor, rows: int, cols: int, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """Packed S (rows x cols) -> packed S^T (cols x rows), int32 CUDA tensor."""
    n_words = dbf_packed_words(cols, rows)
    if out is None:
        out = torch.empty(n_words, dtype=torch.int32, device=packed.device)
    elif out.numel() < n_words or out.dtype != torch.int32:
        raise ValueError("out must be an int32 tensor of dbf_packed_words(cols, rows) words")
    _check("dbf_transpose_signs", load_library().dbf_transpose_signs(
        _ptr(packed), int(rows), int(cols), _ptr(out), _stream(stream)))
    return out


def dbf_forward_transposed(dy: torch.Tensor, packedAT: torch.Tensor, packedBT: torch.Tensor, a: torch.Tensor,
                           m: torch.Tensor, b: torch.Tensor, n: int, k: int, m_in: int, dx: Optional[torch.Tensor] = None,
                           dx_dtype: torch.dtype = torch.float16, workspace: Optional[torch.Tensor] = None,
                           flags: int = 0, stream=None) -> torch.Tensor:
    """dx = b (.) (B^T (m (.) (A^T (a (.) dy)))) for fp16 dy (batch x n); returns dx (batch x m_in)."""
    if dy.dtype != torch.float16 or dy.dim() != 2 or not dy.is_contiguous():
        raise ValueError("dy must be a contiguous fp16 batch x n tensor")
    batch = dy.shape[0]
    if dy.shape[1] != n:
        raise ValueError("dy.shape[1] != n")
    if dx is None:
        dx = torch.empty((batch, m_in), dtype=dx_dtype, device=dy.device)
    if workspace is None:
        workspace = dbf_new_workspace(m_in, k, n, batch, device=dy.device)
    _check("dbf_forward_transposed", load_library().dbf_forward_transposed(
        _ptr(dy), _ptr(packedAT), _ptr(packedBT), _ptr(a), _ptr(m), _ptr(b), int(n), int(k), int(m_in), int(batch),
        _ptr(dx), _dtype_code(dx.dtype), _ptr(workspace), workspace.numel() * workspace.element_size(), int(flags),
        _stream(stream)))
    return dx


def dbf_bqq_prepare(packedY: torch.Tensor, packedZ: torch.Tensor, r: torch.Tensor, s: torch.Tensor, t: torch.Tensor,
                    u: torch.Tensor, n: int, k: int, p: int, m_in: int, stream=None) -> torch.Tensor:
    """The weight-only part of the BQQ forward (mid, c, d); returns the prepared buffer (uint8 CUDA tensor)."""
    nbytes = int(load_library().dbf_bqq_prepared_bytes(int(n), int(k), int(p), int(m_in)))
    if nbytes == 0:
        raise ValueError("shape outside the BQQ contract")
    prep = torch.empty(nbytes, dtype=torch.uint8, device=packedY.device)
    _check("dbf_bqq_prepare", load_library().dbf_bqq_prepare(
        _ptr(packedY), _ptr(packedZ), _ptr(r), _ptr(s), _ptr(t), _ptr(u), int(n), int(k), int(p), int(m_in),
        _ptr(prep), nbytes, _stream(stream)))
    return prep


def dbf_bqq_forward(x: torch.Tensor, packedY: torch.Tensor, packedZ: torch.Tensor, prepared: torch.Tensor, n: int,
                    k: int, p: int, m_in: int, y: Optional[torch.Tensor] = None, y_dtype: torch.dtype = torch.float16,
                    workspace: Optional[torch.Tensor] = None, flags: int = 0, stream=None) -> torch.Tensor:
    """y = x W^T for the BQQ weight W = sum_i (r_i Y_i Z_i + s_i Y_i 1 + t_i 1 Z_i) + u 1; x fp16 batch x m_in."""
    if x.dtype != torch.float16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp16 batch x m_in tensor")
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, n), dtype=y_dtype, device=x.device)
    if workspace is None:
        workspace = torch.zeros(int(load_library().dbf_bqq_workspace_bytes(int(n), int(k), int(p), int(m_in),
                                                                           int(batch))),
                                dtype=torch.uint8, device=x.device)
    _check("dbf_bqq_forward", load_library().dbf_bqq_forward(
        _ptr(x), _ptr(packedY), _ptr(packedZ), _ptr(prepared), int(n), int(k), int(p), int(m_in), int(batch),
        _ptr(y), _dtype_code(y.dtype), _ptr(workspace), workspace.numel(), int(flags), _stream(stream)))
    return y


def _factorize_ws(n, m, k, device):
    nbytes = int(load_library().dbf_factorize_workspace_bytes(int(n), int(m), int(k)))
    if nbytes == 0:
        raise ValueError("shape outside the factorisation contract")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def dbf_factorize_start(W: torch.Tensor, Omega: torch.Tensor, workspace=None, stream=None):
    """L = SVID(W Omega), R = SVID(Omega^T); returns (L, R, err) with err a 1-element fp32 CUDA tensor."""
    n, m = W.shape
    k = Omega.shape[1]
    ws = _factorize_ws(n, m, k, W.device) if workspace is None else workspace
    L = torch.empty((n, k), dtype=torch.float32, device=W.device)
    R = torch.empty((k, m), dtype=torch.float32, device=W.device)
    err = torch.empty(4, dtype=torch.float32, device=W.device)
    _check("dbf_factorize_start", load_library().dbf_factorize_start(
        _ptr(W), _ptr(Omega), n, m, k, _ptr(L), _ptr(R), _ptr(err), _ptr(ws), ws.numel(), _stream(stream)))
    return L, R, err[:1]


def dbf_factorize_pass(W: torch.Tensor, L: torch.Tensor, R: torch.Tensor, admm_steps: int = 20, workspace=None,
                       stream=None) -> torch.Tensor:
    """One alternating pass in place on L (n x k) and R (k x m); returns the error (1-element fp32 CUDA tensor)."""
    n, m = W.shape
    k = L.shape[1]
    ws = _factorize_ws(n, m, k, W.device) if workspace is None else workspace
    err = torch.empty(4, dtype=torch.float32, device=W.device)
    _check("dbf_factorize_pass", load_library().dbf_factorize_pass(
        _ptr(W), n, m, k, _ptr(L), _ptr(R), int(admm_steps), _ptr(err), _ptr(ws), ws.numel(), _stream(stream)))
    return err[:1]


def dbf_factorize_finish(L: torch.Tensor, R: torch.Tensor, workspace=None, stream=None):
    """The DBF form of an SVID-form pair: (packedA, packedB, a, mid, b)."""
    n, k = L.shape
    m = R.shape[1]
    ws = _factorize_ws(n, m, k, L.device) if workspace is None else workspace
    pA = torch.empty(dbf_packed_words(n, k), dtype=torch.int32, device=L.device)
    pB = torch.empty(dbf_packed_words(k, m), dtype=torch.int32, device=L.device)
    a = torch.empty(n, dtype=torch.float16, device=L.device)
    mid = torch.empty(k, dtype=torch.float16, device=L.device)
    b = torch.empty(m, dtype=torch.float16, device=L.device)
    _check("dbf_factorize_finish", load_library().dbf_factorize_finish(
        _ptr(L), _ptr(R), n, m, k, _ptr(pA), _ptr(pB), _ptr(a), _ptr(mid), _ptr(b), _ptr(ws), ws.numel(),
        _stream(stream)))
    return pA, pB, a, mid, b


def dbf_svid(M: torch.Tensor, stream=None):
    """Leading singular pair of |M|: (u, v, sigma) with sign(M) (.) sigma u v^T the SVID projection of M."""
    rows, cols = M.shape
    u = torch.empty(rows, dtype=torch.float32, device=M.device)
    v = torch.empty(cols, dtype=torch.float32, device=M.device)
    sigma = torch.empty(4, dtype=torch.float32, device=M.device)
    ws = torch.empty(int(load_library().dbf_svid_workspace_bytes(rows, cols)), dtype=torch.uint8, device=M.device)
    _check("dbf_svid", load_library().dbf_svid(_ptr(M), rows, cols, _ptr(u), _ptr(v), _ptr(sigma), _ptr(ws),
                                               ws.numel(), _stream(stream)))
    return u, v, sigma[:1]


def dbf_factorize(W: torch.Tensor, Omega: torch.Tensor, passes: int = 10, admm_steps: int = 20, stream=None):
    """Factorise a dense fp32 weight (n x m CUDA tensor) with middle dimension k = Omega.shape[1]: the start,
    `passes` alternating passes keeping the best pair, and the DBF form.  Returns
    (packedA, packedB, a, mid, b, errors) with errors the relative error of the start and after each pass
    (non-increasing)."""
    n, m = W.shape
    k = Omega.shape[1]
    ws = _factorize_ws(n, m, k, W.device)
    L, R, err = dbf_factorize_start(W, Omega, workspace=ws, stream=stream)
    best = float(err.item())
    errors = [best]
    for _ in range(passes):
        Lc, Rc = L.clone(), R.clone()
        e = float(dbf_factorize_pass(W, Lc, Rc, admm_steps, workspace=ws, stream=stream).item())
        if e < best:
            L, R, best = Lc, Rc, e
        errors.append(best)
    return (*dbf_factorize_finish(L, R, workspace=ws, stream=stream), errors)
