"""Host-only checks of the C ABI: the library loads, exports every symbol that
include/dbf.h declares, and rejects bad arguments before touching a device.

No test here launches a kernel or needs a GPU.  Pointers passed to calls that
must fail validation are never dereferenced (validation returns first).
"""
import ctypes
import os
import re

import pytest

import binary_factorized_weight_b200 as dbf
from binary_factorized_weight_b200 import build as dbf_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dbf.h")

OK, INVALID, SHAPE, MISALIGNED, WORKSPACE, CUDA_ERR = 0, 1, 2, 3, 4, 5


@pytest.fixture(scope="module")
def lib():
    dbf_build.build()
    return dbf.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*DBF_API\s+(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(dbf_[a-z_]+)\s*\(", text,
                       flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_api():
    names = declared_functions()
    assert set(names) == set(dbf.EXPORTED_SYMBOLS), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_packed_words(lib):
    assert dbf.dbf_packed_words_per_row(1) == 8
    assert dbf.dbf_packed_words_per_row(256) == 8
    assert dbf.dbf_packed_words_per_row(257) == 16
    assert dbf.dbf_packed_words_per_row(832) == 32
    assert dbf.dbf_packed_words_per_row(4096) == 128
    assert dbf.dbf_packed_words(4096, 2048) == 4096 * 64
    assert dbf.dbf_packed_words(0, 64) == 0
    assert dbf.dbf_packed_words(3, -1) == 0


def test_workspace_bytes(lib):
    # status block + V (batch x k fp16, padded to 256 bytes) + for batch <= 16 the
    # single-launch decode's tagged partials: batch x n x 8 words of 8 bytes
    assert dbf.dbf_forward_workspace_bytes(4096, 2048, 4096, 1) == 256 + 4096 + 8 * 4096 * 8
    assert dbf.dbf_forward_workspace_bytes(256, 128, 256, 4) == 256 + 1024 + 8 * 4 * 256 * 8
    assert dbf.dbf_forward_workspace_bytes(256, 64, 256, 1) == 256 + 256 + 8 * 256 * 8
    assert dbf.dbf_forward_workspace_bytes(256, 128, 256, 17) == 256 + 17 * 256  # no partials past 16 tokens
    assert dbf.dbf_forward_workspace_bytes(256, 128, 256, 128) == 256 + 128 * 256
    # past 128 tokens: the stream-K area (1 KiB of flags, 160 partial tiles of 128 x 256 fp32) after V
    assert dbf.dbf_forward_workspace_bytes(256, 128, 256, 129) == 256 + 129 * 256 + 1024 + 160 * 128 * 256 * 4
    assert dbf.dbf_forward_workspace_bytes(0, 128, 256, 4) == 0


def test_status_strings(lib):
    for code, name in dbf.STATUS_NAMES.items():
        assert dbf.dbf_status_string(code).startswith(name)
    assert "unknown" in dbf.dbf_status_string(99)


# fake, never-dereferenced device addresses
P = 1 << 20  # 16-byte aligned
MIS = P + 2


def fwd(lib, x=P, A=P, B=P, a=P, m=P, b=P, n=256, k=128, m_in=256, batch=4, y=P, y_t=1, ws=P, ws_bytes=1 << 20,
        flags=0):
    return lib.dbf_forward(x, A, B, a, m, b, n, k, m_in, batch, y, y_t, ws, ws_bytes, flags, None)


@pytest.mark.parametrize(
    "kwargs,expect",
    [
        (dict(x=None), INVALID), (dict(A=None), INVALID), (dict(B=None), INVALID), (dict(a=None), INVALID),
        (dict(m=None), INVALID), (dict(b=None), INVALID), (dict(y=None), INVALID),
        (dict(n=0), INVALID), (dict(batch=0), INVALID), (dict(batch=-3), INVALID), (dict(k=0), INVALID),
        (dict(k=96), SHAPE), (dict(m_in=100), SHAPE), (dict(k=1 << 21), SHAPE), (dict(n=(1 << 24) + 1), SHAPE),
        (dict(batch=(1 << 24) + 1), SHAPE),
        (dict(y_t=0), INVALID), (dict(y_t=7), INVALID),
        (dict(flags=1 << 9), INVALID), (dict(flags=2 | 4), INVALID), (dict(flags=32 | 16), INVALID),
        (dict(flags=32 | 8), INVALID), (dict(flags=32 | 64), INVALID), (dict(flags=64 | 8), INVALID),
        (dict(flags=1 << 7), INVALID),
        (dict(x=MIS), MISALIGNED), (dict(A=MIS), MISALIGNED), (dict(B=MIS), MISALIGNED),
        (dict(a=MIS), MISALIGNED), (dict(y=MIS), MISALIGNED),
        (dict(ws=None), WORKSPACE), (dict(ws=MIS), WORKSPACE), (dict(ws_bytes=256 + 1023), WORKSPACE),
    ],
)
def test_forward_validation(lib, kwargs, expect):
    assert fwd(lib, **kwargs) == expect


def test_forward_valid_args_without_device(lib):
    """Valid arguments on a machine with no usable B200 must fail cleanly, not crash."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    assert fwd(lib) in (CUDA_ERR, 7)


def test_pack_validation(lib):
    assert lib.dbf_pack_signs(None, 0, 4, 64, P, None) == INVALID
    assert lib.dbf_pack_signs(P, 0, 4, 64, None, None) == INVALID
    assert lib.dbf_pack_signs(P, 5, 4, 64, P, None) == INVALID
    assert lib.dbf_pack_signs(P, 0, 0, 64, P, None) == INVALID
    assert lib.dbf_pack_signs(P, 0, 4, 64, MIS, None) == MISALIGNED
    assert lib.dbf_pack_signs(P + 1, 2, 4, 64, P, None) == MISALIGNED  # fp32 source not 4-byte aligned


def test_reconstruct_validation(lib):
    assert lib.dbf_reconstruct_dense(P, P, P, P, P, 256, 128, 256, None, 2, None) == INVALID
    assert lib.dbf_reconstruct_dense(P, P, P, P, P, 256, 100, 256, P, 2, None) == SHAPE
    assert lib.dbf_reconstruct_dense(P, P, P, P, P, 256, 128, 256, P, 0, None) == INVALID
    assert lib.dbf_reconstruct_dense(P, P, P, P, P, 256, 128, 256, MIS, 2, None) == MISALIGNED


def test_noalloc_validation(lib):
    # same argument checks as dbf_forward, then the 2 MiB limit of its own buffer
    def call(x=P, n=256, k=128, m_in=256, batch=4, y_t=1, flags=0):
        return lib.dbf_forward_noalloc(x, P, P, P, P, P, n, k, m_in, batch, P, y_t, flags, None)

    assert call(x=None) == INVALID
    assert call(k=96) == SHAPE
    assert call(x=MIS) == MISALIGNED
    assert call(flags=1 << 9) == INVALID
    assert call(k=16384, batch=64) == WORKSPACE  # 256 + 64*16384*2 bytes > 2 MiB


def test_workspace_status_validation(lib):
    out = ctypes.c_int32()
    assert lib.dbf_workspace_status(None, None, ctypes.byref(out)) == INVALID
    assert lib.dbf_workspace_status(P, None, None) == INVALID


def grouped(lib, descs=None, x=P, m_in=256, batch=4, y_t=1, ws=P, ws_bytes=1 << 20, flags=0, num=None):
    if descs is None:
        descs = [dict(n=256, k=128), dict(n=64, k=64)]
    arr = (dbf._LayerDesc * max(1, len(descs)))()
    for i, d in enumerate(descs):
        arr[i] = dbf._LayerDesc(d.get("A", P), d.get("B", P), d.get("a", P), d.get("m", P), d.get("b", P),
                                d.get("n", 256), d.get("k", 128), d.get("y", P))
    return lib.dbf_forward_grouped(x, m_in, batch, arr, len(descs) if num is None else num, y_t, ws, ws_bytes,
                                   flags, None)


def test_grouped_workspace_bytes(lib):
    # 256 + sum of round_up(batch * k_g * 2, 256)
    assert dbf.dbf_forward_grouped_workspace_bytes([dict(n=256, k=128), dict(n=64, k=64)], 256, 4) == \
        256 + 1024 + 512
    assert dbf.dbf_forward_grouped_workspace_bytes([dict(n=8, k=832)], 4096, 3) == 256 + 5120
    # past 128 tokens the stream-K area follows the V blocks
    assert dbf.dbf_forward_grouped_workspace_bytes([dict(n=8, k=64)], 64, 200) == \
        256 + 200 * 128 + 1024 + 160 * 128 * 256 * 4
    assert dbf.dbf_forward_grouped_workspace_bytes([dict(n=0, k=64)], 64, 1) == 0
    assert dbf.dbf_forward_grouped_workspace_bytes([dict(n=1, k=64)] * 9, 64, 1) == 0


@pytest.mark.parametrize(
    "kwargs,expect",
    [
        (dict(x=None), INVALID), (dict(num=0), INVALID), (dict(num=9), INVALID),
        (dict(descs=[dict(y=None)]), INVALID), (dict(descs=[dict(A=None)]), INVALID),
        (dict(descs=[dict(n=0)]), INVALID), (dict(descs=[dict(k=96)]), SHAPE), (dict(m_in=100), SHAPE),
        (dict(descs=[dict(), dict(k=1 << 21)]), SHAPE),
        (dict(batch=0), INVALID), (dict(y_t=2 + 5), INVALID), (dict(flags=2 | 4), INVALID),
        (dict(x=MIS), MISALIGNED), (dict(descs=[dict(), dict(y=MIS)]), MISALIGNED),
        (dict(descs=[dict(B=MIS)]), MISALIGNED),
        (dict(ws=None), WORKSPACE), (dict(ws_bytes=256 + 1024 + 511), WORKSPACE),
    ],
)
def test_grouped_validation(lib, kwargs, expect):
    assert grouped(lib, **kwargs) == expect


def test_grouped_valid_args_without_device(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    assert grouped(lib) in (CUDA_ERR, 7)


def test_transpose_validation(lib):
    assert lib.dbf_transpose_signs(None, 4, 64, P, None) == INVALID
    assert lib.dbf_transpose_signs(P, 4, 64, None, None) == INVALID
    assert lib.dbf_transpose_signs(P, 0, 64, P, None) == INVALID
    assert lib.dbf_transpose_signs(P, 4, (1 << 24) + 1, P, None) == SHAPE
    assert lib.dbf_transpose_signs(MIS, 4, 64, P, None) == MISALIGNED
    assert lib.dbf_transpose_signs(P, 4, 64, MIS, None) == MISALIGNED


def test_forward_transposed_validation(lib):
    # dy (batch x n), dx (batch x m_in); n takes the place of the forward's m_in
    def call(dy=P, n=256, k=128, m_in=200, batch=4, dx=P, ws_bytes=1 << 20):
        return lib.dbf_forward_transposed(dy, P, P, P, P, P, n, k, m_in, batch, dx, 1, P, ws_bytes, 0, None)

    assert call(dy=None) == INVALID
    assert call(n=100) == SHAPE       # n must be a multiple of 64 here
    assert call(k=96) == SHAPE
    assert call(dx=MIS) == MISALIGNED
    assert call(ws_bytes=255) == WORKSPACE


def no_device():
    import torch

    return not torch.cuda.is_available()


def test_factorize_workspace_bytes(lib):
    f = lib.dbf_factorize_workspace_bytes
    assert f(0, 4, 4) == 0 and f(4, 0, 4) == 0 and f(4, 4, 0) == 0
    assert f(65537, 4, 4) == 0 and f(4, 65537, 4) == 0 and f(4, 4, 16385) == 0
    assert f(65536, 65536, 1) == 0          # n * m above 2^31
    assert f(65536, 64, 16384) > 0          # the largest factor: 2^30 elements
    n, m, k = 4096, 4096, 2048
    # at least: W - L R (n x m), six factor-sized buffers, the Gram matrix and its inverse with the
    # solver's two k x k slots, all fp32
    assert f(n, m, k) >= 4 * (n * m + 6 * max(n, m) * k + 4 * k * k)
    assert f(n, m, k) % 256 == 0
    assert f(n, m, 2 * k) > f(n, m, k)


def test_svid_workspace_bytes(lib):
    assert lib.dbf_svid_workspace_bytes(4096, 2048) == 32 * 2048 * 4  # 32 row chunks of fp32 column sums
    assert lib.dbf_svid_workspace_bytes(1, 1) == 32 * 4
    assert lib.dbf_svid_workspace_bytes(0, 5) == 0 and lib.dbf_svid_workspace_bytes(5, 0) == 0


def test_svid_validation(lib):
    def call(M=P, rows=64, cols=32, u=P, v=P, sigma=P, ws=P, ws_bytes=1 << 20):
        return lib.dbf_svid(M, rows, cols, u, v, sigma, ws, ws_bytes, None)

    for bad in ("M", "u", "v", "sigma", "ws"):
        assert call(**{bad: None}) == INVALID, bad
    assert call(rows=0) == INVALID and call(cols=-1) == INVALID
    assert call(rows=1 << 16, cols=(1 << 15) + 1) == SHAPE
    for bad in ("M", "u", "v", "sigma", "ws"):
        assert call(**{bad: MIS}) == MISALIGNED, bad
    assert call(ws_bytes=32 * 32 * 4 - 1) == WORKSPACE
    if no_device():
        assert call(ws_bytes=32 * 32 * 4) in (CUDA_ERR, 7)


def test_factorize_validation(lib):
    ws_ok = lib.dbf_factorize_workspace_bytes(200, 256, 64)

    def pass_(W=P, n=200, m=256, k=64, L=P, R=P, steps=20, err=P, ws=P, ws_bytes=ws_ok):
        return lib.dbf_factorize_pass(W, n, m, k, L, R, steps, err, ws, ws_bytes, None)

    def start(W=P, Om=P, n=200, m=256, k=64, L=P, R=P, err=P, ws=P, ws_bytes=ws_ok):
        return lib.dbf_factorize_start(W, Om, n, m, k, L, R, err, ws, ws_bytes, None)

    def finish(L=P, R=P, n=200, m=256, k=64, pA=P, pB=P, a=P, mid=P, b=P, ws=P, ws_bytes=ws_ok):
        return lib.dbf_factorize_finish(L, R, n, m, k, pA, pB, a, mid, b, ws, ws_bytes, None)

    for call, ptrs in ((pass_, ("W", "L", "R", "err", "ws")), (start, ("W", "Om", "L", "R", "err", "ws")),
                       (finish, ("L", "R", "pA", "pB", "a", "mid", "b", "ws"))):
        for name in ptrs:
            assert call(**{name: None}) == INVALID, (call.__name__, name)
            assert call(**{name: MIS}) == MISALIGNED, (call.__name__, name)
        assert call(n=0) == INVALID and call(k=0) == INVALID
        assert call(n=65537) == SHAPE and call(k=16385) == SHAPE and call(n=65536, m=65536, k=1) == SHAPE
        assert call(ws_bytes=ws_ok - 1) == WORKSPACE
        if no_device():
            assert call() in (CUDA_ERR, 7), call.__name__
    assert pass_(steps=0) == INVALID and pass_(steps=1001) == INVALID


def test_bqq_sizes(lib):
    # (n, k, p, m_in): p terms of k middle rows each, p * k and m_in multiples of 64
    assert lib.dbf_bqq_prepared_bytes(256, 32, 2, 256) > 0
    assert lib.dbf_bqq_prepared_bytes(256, 32, 1, 256) == 0      # p * k = 32 is not a multiple of 64
    assert lib.dbf_bqq_prepared_bytes(256, 64, 1, 100) == 0      # m_in not a multiple of 64
    assert lib.dbf_bqq_prepared_bytes(256, 64, 4097, 256) == 0   # more than 4096 terms
    assert lib.dbf_bqq_prepared_bytes(0, 64, 1, 256) == 0
    # the DBF forward's workspace for the k p middle rows, then the fp32 sign-product term (batch x n)
    for n, k, p, m_in, batch in ((256, 32, 2, 256, 4), (4096, 256, 8, 4096, 2048), (100, 64, 3, 64, 1)):
        assert lib.dbf_bqq_workspace_bytes(n, k, p, m_in, batch) == \
            lib.dbf_forward_workspace_bytes(n, k * p, m_in, batch) + (batch * n * 4 + 255) // 256 * 256
    assert lib.dbf_bqq_workspace_bytes(256, 32, 2, 256, 0) == 0


def test_bqq_validation(lib):
    prep_ok = lib.dbf_bqq_prepared_bytes(256, 32, 2, 256)
    ws_ok = lib.dbf_bqq_workspace_bytes(256, 32, 2, 256, 4)

    def prepare(Y=P, Z=P, r=P, s=P, t=P, u=P, n=256, k=32, p=2, m_in=256, prep=P, prep_bytes=prep_ok):
        return lib.dbf_bqq_prepare(Y, Z, r, s, t, u, n, k, p, m_in, prep, prep_bytes, None)

    def forward(x=P, Y=P, Z=P, prep=P, n=256, k=32, p=2, m_in=256, batch=4, y=P, y_t=1, ws=P, ws_bytes=ws_ok,
                flags=0):
        return lib.dbf_bqq_forward(x, Y, Z, prep, n, k, p, m_in, batch, y, y_t, ws, ws_bytes, flags, None)

    for name in ("Y", "Z", "r", "s", "t", "u", "prep"):
        assert prepare(**{name: None}) == INVALID, name
    assert prepare(k=48) == SHAPE and prepare(m_in=100) == SHAPE and prepare(n=0) == INVALID
    for name in ("Y", "Z", "prep"):
        assert prepare(**{name: MIS}) == MISALIGNED, name
    assert prepare(prep_bytes=prep_ok - 1) == WORKSPACE
    for name in ("x", "Y", "Z", "prep", "y"):
        assert forward(**{name: None}) == INVALID, name
    assert forward(k=48) == SHAPE and forward(batch=0) == INVALID and forward(y_t=7) == INVALID
    assert forward(flags=1 << 9) == INVALID
    for name in ("x", "Y", "Z", "prep", "y"):
        assert forward(**{name: MIS}) == MISALIGNED, name
    assert forward(ws=None) == WORKSPACE and forward(ws=MIS) == WORKSPACE and forward(ws_bytes=ws_ok - 1) == WORKSPACE
    if no_device():
        assert prepare() in (CUDA_ERR, 7)
        assert forward() in (CUDA_ERR, 7)
