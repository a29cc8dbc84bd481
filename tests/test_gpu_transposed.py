"""GPU parity of the transpose product dx = dy W (the input gradient of the
layer of "Addition is almost all you need", gist.science technical summary,
section 2.1): dbf_transpose_signs against the oracle's encoder of S^T (bit-exact),
and dbf_forward_transposed against the oracle's forward_transposed with the bars
of test_gpu_parity.py."""
import numpy as np
import pytest
import torch

import dbf_inputs as gen
import oracle
from test_gpu_parity import PATHS, assert_fp16_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from binary_factorized_weight_b200 import build

    build.build()
    import binary_factorized_weight_b200 as mod

    mod.load_library()
    return mod


@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 64), (64, 832), (300, 257), (832, 1024), (4096, 2048)])
def test_transpose_signs_bit_exact(dbf, rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    S = gen.sign_matrix(rng, rows, cols)
    packed = dev(oracle.pack_signs(S).view(np.int32))
    out = dbf.dbf_transpose_signs(packed, rows, cols)
    torch.cuda.synchronize()
    want = oracle.pack_signs(np.ascontiguousarray(S.T))
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want)


def transposed_layer(dbf, n, k, m_in, batch, seed, integer=False):
    rng = np.random.default_rng(seed)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    if integer:
        a, mid, b = gen.unit_scales(n), gen.unit_scales(k), gen.unit_scales(m_in)
        lim = max(1, min(8, 2048 // n))
        dy = rng.integers(-lim, lim + 1, size=(batch, n)).astype(np.float16)
    else:
        a, mid, b = gen.lognormal_scales(rng, n), gen.lognormal_scales(rng, k), gen.lognormal_scales(rng, m_in)
        dy = gen.normal_activations(rng, batch, n)
    pA = dbf.dbf_pack_signs(dev(A))
    pB = dbf.dbf_pack_signs(dev(B))
    pAT = dbf.dbf_transpose_signs(pA, n, k)
    pBT = dbf.dbf_transpose_signs(pB, k, m_in)
    return dict(A=A, B=B, a=a, mid=mid, b=b, dy=dy, pAT=pAT, pBT=pBT)


@pytest.mark.parametrize("path", ["default", "decode_fused", "decode_class", "decode_shift", "prefill"])
@pytest.mark.parametrize("n,k,m_in,batch", [(256, 128, 256, 1), (128, 64, 200, 5), (64, 192, 65, 17),
                                            (192, 128, 320, 130)])
def test_forward_transposed_integer_bit_exact(dbf, path, n, k, m_in, batch):
    L = transposed_layer(dbf, n, k, m_in, batch, seed=n + k + batch, integer=True)
    flags = 0 if path == "default" else PATHS[path]
    dx = dbf.dbf_forward_transposed(dev(L["dy"]), L["pAT"], L["pBT"], dev(L["a"]), dev(L["mid"]), dev(L["b"]),
                                    n, k, m_in, dx_dtype=torch.float32, flags=flags)
    torch.cuda.synchronize()
    ref = oracle.forward_transposed(L["dy"], L["A"], L["B"], L["a"], L["mid"], L["b"])
    assert np.array_equal(dx.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("path", ["default", "decode_fused", "decode_class", "prefill"])
@pytest.mark.parametrize("batch", [1, 16, 128])
def test_forward_transposed_fp16(dbf, path, batch):
    n, k, m_in = 256, 128, 320
    L = transposed_layer(dbf, n, k, m_in, batch, seed=batch)
    flags = 0 if path == "default" else PATHS[path]
    dx = dbf.dbf_forward_transposed(dev(L["dy"]), L["pAT"], L["pBT"], dev(L["a"]), dev(L["mid"]), dev(L["b"]),
                                    n, k, m_in, flags=flags)
    torch.cuda.synchronize()
    ref = oracle.forward_transposed(L["dy"], L["A"], L["B"], L["a"], L["mid"], L["b"])
    assert_fp16_close(dx.float().cpu().numpy(), ref, "dx")


@pytest.mark.parametrize("batch", [1, 2048])
def test_forward_transposed_full_size(dbf, batch):
    """4096 x 4096 at k = 2048 (1 bit/weight); every token at batch 2048."""
    n = m_in = 4096
    k = 2048
    L = transposed_layer(dbf, n, k, m_in, batch, seed=99)
    dx = dbf.dbf_forward_transposed(dev(L["dy"]), L["pAT"], L["pBT"], dev(L["a"]), dev(L["mid"]), dev(L["b"]),
                                    n, k, m_in, flags=dbf.DBF_FWD_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    ref = oracle.forward_transposed(L["dy"], L["A"], L["B"], L["a"], L["mid"], L["b"])
    assert_fp16_close(dx.float().cpu().numpy(), ref, "dx")  # every token
