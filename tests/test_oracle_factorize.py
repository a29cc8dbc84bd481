"""Pins of the reference DBF factorisation (oracle/factorize.py).

The pages (gist.science technical summary, section 2.2) describe the
optimisation as SVID projection, alternating minimisation and ADMM without
equations, so the reference is pinned by what the mathematics fixes:
  * SVID returns a matrix that already is sign (.) rank-one unchanged, and its
    factors are nonnegative;
  * k = 1 recovers W = a A mid B b exactly after one pass (W has rank one and a
    sign pattern with rank-one magnitudes: the left step's least squares is
    proportional to a (.) A, and SVID keeps it);
  * the error never rises over the passes, and the passes improve on the start;
  * the error falls as k grows (the analogue of the pages' error-vs-size
    curves), and at every k it is below 1 (the zero matrix);
  * the returned factors reconstruct, through the pinned C oracle's dense
    weight, exactly what the factorisation reports;
  * a converged ADMM solve sits at a fixed point of scaled ADMM: L = Z (the
    dual update stops) and Z = SVID(Z - grad f(Z) / rho) for the least-squares
    term f(L) = ||W - L R||_F^2 (the L step's stationarity fixes the scaled dual
    at U = -grad f(Z) / rho, and the Z step then projects Z + U);
  * a pass that would raise the error is not kept (on a seeded case where one
    does).
"""
import numpy as np
import pytest

import dbf_inputs as gen
from oracle import factorize as F


def _omega(m, k, seed=0):
    return gen.projection_signs(np.random.default_rng(seed), m, k)


def test_svid_keeps_sign_times_rank_one():
    rng = np.random.default_rng(1)
    u, v = np.abs(rng.standard_normal(17)) + 0.1, np.abs(rng.standard_normal(9)) + 0.1
    S = np.where(rng.random((17, 9)) < 0.5, -1, 1)
    M = u[:, None] * S * v[None, :]
    uu, SS, vv = F.svid(M)
    assert np.all(uu >= 0) and np.all(vv >= 0)
    assert np.array_equal(SS, S)
    assert np.allclose(uu[:, None] * SS * vv[None, :], M, rtol=1e-12, atol=1e-12)


def test_svid_is_the_best_rank_one_of_the_magnitudes():
    rng = np.random.default_rng(2)
    M = rng.standard_normal((30, 20))
    u, S, v = F.svid(M)
    assert np.array_equal(S, np.where(M < 0, -1, 1))
    U, sig, Vt = np.linalg.svd(np.abs(M))
    best = sig[0] * np.outer(U[:, 0], Vt[0])
    assert np.allclose(np.outer(u, v), np.abs(best), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("n,m", [(40, 30), (7, 64)])
def test_k1_recovers_a_dbf_layer_exactly(n, m):
    rng = np.random.default_rng(n + m)
    a, b = np.abs(rng.standard_normal(n)) + 0.1, np.abs(rng.standard_normal(m)) + 0.1
    A = np.where(rng.random((n, 1)) < 0.5, -1, 1)
    B = np.where(rng.random((1, m)) < 0.5, -1, 1)
    W = (a[:, None] * A * 0.7) @ (B * b[None, :])
    f = F.factorize(W, _omega(m, 1, n), passes=3, admm_steps=60)
    assert f["errors"][-1] < 1e-9, f["errors"]
    assert np.allclose(F.reconstruct(f), W, rtol=0, atol=1e-9 * np.abs(W).max())


def test_errors_never_rise_and_passes_help():
    rng = np.random.default_rng(3)
    W = rng.standard_normal((96, 80))
    f = F.factorize(W, _omega(80, 48), passes=6)
    e = f["errors"]
    assert all(e[i + 1] <= e[i] for i in range(len(e) - 1))
    assert e[-1] < 0.95 * e[0]


def test_error_falls_with_k():
    rng = np.random.default_rng(4)
    W = rng.standard_normal((128, 96))
    errs = [F.factorize(W, _omega(96, k), passes=6)["errors"][-1] for k in (8, 24, 48, 96)]
    assert all(0 < e < 1 for e in errs)
    assert all(errs[i + 1] < errs[i] for i in range(len(errs) - 1)), errs


def test_factors_reconstruct_through_the_dense_oracle(oracle_mod):
    rng = np.random.default_rng(5)
    W = rng.standard_normal((48, 40))
    f = F.factorize(W, _omega(40, 24), passes=4)
    assert f["A"].shape == (48, 24) and f["B"].shape == (24, 40)
    assert set(np.unique(f["A"])) <= {-1, 1} and set(np.unique(f["B"])) <= {-1, 1}
    Wd = oracle_mod.dense_weight(f["A"], f["B"], f["a"], f["mid"], f["b"])
    assert np.allclose(Wd, F.reconstruct(f), rtol=1e-12, atol=1e-12)
    assert np.linalg.norm(W - Wd) / np.linalg.norm(W) == pytest.approx(f["errors"][-1], rel=1e-9)


@pytest.mark.parametrize("seed", [300, 302])
def test_converged_admm_is_a_projected_gradient_fixed_point(seed):
    rng = np.random.default_rng(seed)
    n, m, k = 12, 10, 3
    W = rng.standard_normal((n, m))
    R = F.svid_matrix(rng.standard_normal((k, m)))
    Z0 = F.svid_matrix(rng.standard_normal((n, k)))
    rho = 2.0 * float(np.sum(R * R)) / k
    Z = F.admm_left(W, R, Z0, rho, 400)
    Z_next = F.admm_left(W, R, Z0, rho, 401)
    # these seeded cases converge (ADMM on a nonconvex set need not)
    assert np.linalg.norm(Z_next - Z) <= 1e-12 * np.linalg.norm(Z)
    grad = -2.0 * (W - Z @ R) @ R.T  # gradient of ||W - L R||_F^2 at L = Z
    assert np.linalg.norm(F.svid_matrix(Z - grad / rho) - Z) <= 1e-10 * np.linalg.norm(Z)


def test_a_pass_that_raises_the_error_is_not_kept():
    W = np.random.default_rng(202).standard_normal((16, 48))
    Om = gen.projection_signs(np.random.default_rng(2), 48, 8)
    L, R = F.start_factors(W, Om)
    free = [F.relative_error(W, L, R)]
    for _ in range(8):
        L, R = F.alternating_pass(W, L, R, 20)
        free.append(F.relative_error(W, L, R))
    assert any(free[i + 1] > free[i] for i in range(8)), "the case must contain a rising pass"
    e = F.factorize(W, Om, passes=8, admm_steps=20)["errors"]
    assert all(e[i + 1] <= e[i] for i in range(8))
    first_rise = next(i for i in range(8) if free[i + 1] > free[i])
    assert e[:first_rise + 1] == pytest.approx(free[:first_rise + 1], rel=1e-12)
    assert e[first_rise + 1] == e[first_rise]
