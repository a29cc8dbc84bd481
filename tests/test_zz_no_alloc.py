"""dbf_forward_noalloc, the workspace-free forward, checked through the C ABI.

Some callers cannot allocate device memory (a plugin inside a host application
that owns every allocation, or a thread that must never call cudaMalloc because
it can block and synchronise the device).  dbf_forward_noalloc serves them
with a fixed 2 MiB buffer inside the library instead of a caller workspace.
Here it must give the same output as dbf_forward with a workspace, on two
calls in a row (the buffer keeps the previous call's contents), on both paths.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import dbf_inputs as gen

pytestmark = pytest.mark.gpu

REL_FRO = 2e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from binary_factorized_weight_b200 import build

    build.build()
    import binary_factorized_weight_b200 as dbf

    return dbf, dbf.load_library()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("config,batch,y_dtype", [("tiny", 4, torch.float16), ("tiny", 256, torch.float16),
                                                  ("tiny_int", 16, torch.float32), ("attn_1b", 1, torch.float16)])
def test_noalloc_matches_workspace_forward_twice(lib, config, batch, y_dtype):
    dbf, c = lib
    shape = gen.CONFIGS[config]
    L = gen.make_layer(shape, batch)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pA, pB = dbf.dbf_pack_signs(dev(L["A"])), dbf.dbf_pack_signs(dev(L["B"]))
    a, mid, b, x = dev(L["a"]), dev(L["mid"]), dev(L["b"]), dev(L["x"])
    n, k, m_in = shape.n, shape.k, shape.m_in
    ref = dbf.dbf_forward(x, pA, pB, a, mid, b, n, k, m_in, y_dtype=y_dtype, flags=dbf.DBF_FWD_WEIGHTS_STATIC)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    y_code = 2 if y_dtype == torch.float32 else 1
    for _ in range(2):
        y = torch.full((batch, n), float("nan"), dtype=y_dtype, device="cuda")
        st = c.dbf_forward_noalloc(_ptr(x), _ptr(pA), _ptr(pB), _ptr(a), _ptr(mid), _ptr(b), n, k, m_in, batch,
                                   _ptr(y), y_code, dbf.DBF_FWD_WEIGHTS_STATIC, stream)
        assert st == 0, dbf.dbf_status_string(st)
        torch.cuda.synchronize()
        yn, rn = y.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(yn))
        if config == "tiny_int":
            assert np.array_equal(yn, rn)
        else:
            assert np.linalg.norm(yn - rn) / np.linalg.norm(rn) <= REL_FRO
        status = ctypes.c_int32(-1)
        assert c.dbf_noalloc_status(stream, ctypes.byref(status)) == 0
        assert status.value == 0  # no device-side wait gave up


def test_noalloc_rejects_sizes_beyond_its_buffer(lib):
    dbf, c = lib
    big = 1 << 20  # 256 + 64 * 16384 * 2 bytes > 2 MiB
    fake = ctypes.c_void_p(1 << 20)
    st = c.dbf_forward_noalloc(fake, fake, fake, fake, fake, fake, 256, 16384, 256, 64, fake, 1, 0, None)
    assert st == 4  # DBF_ERR_WORKSPACE, before anything is enqueued
    del big
