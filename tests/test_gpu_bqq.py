"""GPU parity of the Binary Quadratic Quantization (BQQ) forward through the C ABI.

W = sum_i (r_i Y_i Z_i + s_i Y_i 1_Z + t_i 1_Y Z_i) + u 1 (sciencestack.ai page
of "Binary Quadratic Quantization", TL;DR formula; binary entries read as
{0, 1}), y = x W^T, against the fp64 oracle's BQQ weight:
  * integer mode (r multiple of 4, integer s, t, u and x, fp32 output): exact;
  * fp16 data: the bars of the DBF forward (relative Frobenius <= 2e-3, max
    error <= 1e-2 * rms(y));
on both the single-launch decode path and the tensor-core path.
"""
import numpy as np
import pytest
import torch

import oracle
from test_gpu_parity import assert_fp16_close, dev

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


def _bqq(dbf, rng, p, n, k, m_in, integer):
    Y = rng.integers(0, 2, size=(p, n, k)).astype(np.int8)
    Z = rng.integers(0, 2, size=(p, k, m_in)).astype(np.int8)
    if integer:
        r = (4 * rng.integers(-2, 3, size=p)).astype(np.float16)
        s, t = rng.integers(-3, 4, size=p).astype(np.float16), rng.integers(-3, 4, size=p).astype(np.float16)
        u = np.array([rng.integers(-5, 6)], np.float16)
    else:
        r = (rng.standard_normal(p) * 0.05).astype(np.float16)
        s = (rng.standard_normal(p) * 0.01).astype(np.float16)
        t = (rng.standard_normal(p) * 0.01).astype(np.float16)
        u = np.array([0.003], np.float16)
    SY = np.concatenate([1 - 2 * Y[i] for i in range(p)], axis=1).astype(np.int8)  # set bit = binary 1
    SZ = np.concatenate([1 - 2 * Z[i] for i in range(p)], axis=0).astype(np.int8)
    pY, pZ = dbf.dbf_pack_signs(dev(SY)), dbf.dbf_pack_signs(dev(SZ))
    prep = dbf.dbf_bqq_prepare(pY, pZ, dev(r), dev(s), dev(t), dev(u), n, k, p, m_in)
    W = oracle.bqq_dense_weight(Y, Z, r.astype(np.float64), s.astype(np.float64), t.astype(np.float64),
                                float(u[0]))
    return pY, pZ, prep, W


@pytest.mark.parametrize("p,n,k,m_in", [(1, 256, 128, 256), (2, 192, 96, 320), (3, 1000, 256, 512)])
@pytest.mark.parametrize("batch,flags", [(1, 0), (5, 0), (5, 16), (40, 0)])
def test_bqq_forward_integer_exact(dbf, p, n, k, m_in, batch, flags):
    rng = np.random.default_rng(p * 1000 + n + batch)
    pY, pZ, prep, W = _bqq(dbf, rng, p, n, k, m_in, integer=True)
    x = rng.integers(-2, 3, size=(batch, m_in)).astype(np.float16)
    y = dbf.dbf_bqq_forward(dev(x), pY, pZ, prep, n, k, p, m_in, y_dtype=torch.float32, flags=flags)
    torch.cuda.synchronize()
    ref = oracle.forward_dense(x, W)
    assert np.abs(ref).max() < 2 ** 24
    assert np.array_equal(y.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("batch", [1, 16, 300])
def test_bqq_forward_fp16(dbf, batch):
    p, n, k, m_in = 2, 1024, 512, 2048
    rng = np.random.default_rng(batch)
    pY, pZ, prep, W = _bqq(dbf, rng, p, n, k, m_in, integer=False)
    x = rng.standard_normal((batch, m_in)).astype(np.float16)
    y = dbf.dbf_bqq_forward(dev(x), pY, pZ, prep, n, k, p, m_in)
    torch.cuda.synchronize()
    assert_fp16_close(y.float().cpu().numpy(), oracle.forward_dense(x, W), f"bqq b{batch}")
