"""GPU factorisation (dbf_factorize_start / _pass / _finish, dbf_svid) against the fp64 reference.

The factorisation of "Addition is almost all you need" (gist.science technical
summary, section 2.2: alternating minimisation, ADMM, SVID projection) makes
discrete sign decisions, so the GPU (fp32) and the reference (fp64) agree on
what is unique and are checked for validity elsewhere:
  * SVID's rank-one magnitude (the leading singular pair of |M|) and the start
    L = SVID(W Omega), R = SVID(Omega^T): equal to the reference's within fp32
    rounding;
  * one alternating pass from the same start: the same relative error within
    a fraction of a percent, the same signs on all but a few entries;
  * a whole run: non-increasing errors, the final error close to the
    reference's, and k = 1 recovering a DBF layer exactly;
  * the DBF form: signs bit-exact against the reference's decoder, the
    reconstruction through dbf_reconstruct_dense within the fp16 bar.
"""
import numpy as np
import pytest
import torch

import dbf_inputs as gen
import oracle
from oracle import factorize as F

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


def dev32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _problem(n, m, k, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((n, m)) * np.linspace(2.0, 0.2, m)[None, :]).astype(np.float32)
    Om = gen.projection_signs(rng, m, k)
    return W, Om


@pytest.mark.parametrize("rows,cols", [(300, 200), (64, 1000), (1, 17)])
def test_svid_pair_matches_reference(dbf, rows, cols):
    rng = np.random.default_rng(rows + cols)
    M = rng.standard_normal((rows, cols)).astype(np.float32)
    u, v, sigma = dbf.dbf_svid(dev32(M))
    torch.cuda.synchronize()
    got = float(sigma.item()) * np.outer(u.cpu().numpy(), v.cpu().numpy())
    uu, S, vv = F.svid(M.astype(np.float64))
    ref = np.outer(uu, vv)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-5


def test_start_matches_reference(dbf):
    W, Om = _problem(256, 192, 64, seed=1)
    L, R, err = dbf.dbf_factorize_start(dev32(W), dev32(Om))
    torch.cuda.synchronize()
    L0, R0 = F.start_factors(W.astype(np.float64), Om.astype(np.float64))
    assert np.linalg.norm(L.cpu().numpy() - L0) / np.linalg.norm(L0) < 1e-5
    assert np.linalg.norm(R.cpu().numpy() - R0) / np.linalg.norm(R0) < 1e-5
    assert float(err.item()) == pytest.approx(F.relative_error(W, L0, R0), rel=1e-5)


def test_one_pass_matches_reference(dbf):
    W, Om = _problem(256, 192, 64, seed=2)
    L0, R0 = F.start_factors(W.astype(np.float64), Om.astype(np.float64))
    L, R = dev32(L0), dev32(R0)
    err = float(dbf.dbf_factorize_pass(dev32(W), L, R, admm_steps=20).item())
    Lr, Rr = F.alternating_pass(W.astype(np.float64), L0, R0, admm_steps=20)
    err_ref = F.relative_error(W, Lr, Rr)
    assert err == pytest.approx(err_ref, rel=5e-3)
    assert err == pytest.approx(F.relative_error(W, L.cpu().numpy().astype(np.float64),
                                                 R.cpu().numpy().astype(np.float64)), rel=1e-4)
    agree_L = np.mean(np.sign(L.cpu().numpy()) == np.sign(Lr))
    agree_R = np.mean(np.sign(R.cpu().numpy()) == np.sign(Rr))
    assert agree_L > 0.99 and agree_R > 0.99, (agree_L, agree_R)


def test_run_is_monotone_and_close_to_reference(dbf):
    W, Om = _problem(192, 160, 96, seed=3)
    *_, errors = dbf.dbf_factorize(dev32(W), dev32(Om), passes=5)
    assert all(errors[i + 1] <= errors[i] for i in range(len(errors) - 1))
    ref = F.factorize(W.astype(np.float64), Om.astype(np.float64), passes=5)["errors"]
    assert errors[-1] < errors[0]
    assert errors[-1] == pytest.approx(ref[-1], rel=0.02)


def test_k1_recovers_a_dbf_layer(dbf):
    n, m = 96, 128
    rng = np.random.default_rng(4)
    a, b = np.abs(rng.standard_normal(n)) + 0.1, np.abs(rng.standard_normal(m)) + 0.1
    A = np.where(rng.random((n, 1)) < 0.5, -1, 1)
    B = np.where(rng.random((1, m)) < 0.5, -1, 1)
    W = ((a[:, None] * A * 0.7) @ (B * b[None, :])).astype(np.float32)
    Om = gen.projection_signs(rng, m, 1)
    *_, errors = dbf.dbf_factorize(dev32(W), dev32(Om), passes=3, admm_steps=60)
    assert errors[-1] < 1e-5, errors


def test_finish_gives_the_dbf_form(dbf):
    n, m, k = 200, 256, 64
    W, Om = _problem(n, m, k, seed=5)
    f = F.factorize(W.astype(np.float64), Om.astype(np.float64), passes=2)
    L = f["a"][:, None] * f["A"] * np.sqrt(f["mid"])[None, :]
    R = np.sqrt(f["mid"])[:, None] * f["B"] * f["b"][None, :]
    pA, pB, a, mid, b = dbf.dbf_factorize_finish(dev32(L), dev32(R))
    torch.cuda.synchronize()
    A, bad_a = oracle.unpack_signs(pA.cpu().numpy().view(np.uint32), n, k)
    B, bad_b = oracle.unpack_signs(pB.cpu().numpy().view(np.uint32), k, m)
    assert bad_a == 0 and bad_b == 0
    assert np.array_equal(A, np.where(L < 0, -1, 1)) and np.array_equal(B, np.where(R < 0, -1, 1))
    Wd = dbf.dbf_reconstruct_dense(pA, pB, a, mid, b, n, k, m, W_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = L.astype(np.float64) @ R.astype(np.float64)
    got = Wd.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 2e-3
