"""Pins of the oracle's Binary Quadratic Quantization (BQQ) weight and forward.

The sciencestack.ai page of "Binary Quadratic Quantization: Beyond First-Order
Quantization for Real-Valued Matrix Compression" (TL;DR) writes the compressed
matrix as W = sum_i (r_i Y_i Z_i + s_i Y_i 1_Z + t_i 1_Y Z_i) + u 1 with binary
Y_i (n x k), Z_i (k x m).  The binary alphabet is read as {0, 1}.  Pinned by:
  * a forward worked by hand (tests/golden/bqq_worked_example.txt);
  * Y Z against numpy's integer matmul (s = t = u = 0, r = 1);
  * the all-ones closed form W = sum_i k (r_i + s_i + t_i) + u;
  * the special case that is a DBF layer: with S = 1 - 2Y (a {0,1} matrix as
    signs), s_i = t_i = -r_i/2 and u = k sum_i r_i / 4, W equals
    sum_i (r_i / 4) S_Yi S_Zi, the oracle's (separately pinned) DBF weight with
    A = [S_Y0 .. S_Yp-1], mid = r_i / 4 on block i, a = b = 1;
  * rank: with r = 0 the weight is s-terms (constant along rows) plus t-terms
    (constant along columns) plus u: rank <= 2.
"""
import numpy as np
import pytest

from conftest import read_golden


def _random_bqq(rng, p, n, k, m):
    Y = rng.integers(0, 2, size=(p, n, k)).astype(np.int8)
    Z = rng.integers(0, 2, size=(p, k, m)).astype(np.int8)
    r, s, t = rng.standard_normal(p), rng.standard_normal(p), rng.standard_normal(p)
    return Y, Z, r, s, t, float(rng.standard_normal())


def test_bqq_hand_worked_example(oracle_mod):
    g = read_golden("bqq_worked_example.txt")
    Y = np.array([g["Y0"], g["Y1"]], dtype=np.int8).reshape(2, 2, 2)
    Z = np.array([g["Z0"], g["Z1"]], dtype=np.int8).reshape(2, 2, 2)
    x = np.array([g["x"]])
    W = oracle_mod.bqq_dense_weight(Y, Z, g["r"], g["s"], g["t"], g["u"][0])
    assert np.array_equal(W, np.array(g["W"]).reshape(2, 2))
    assert np.array_equal(oracle_mod.bqq_forward(x, Y, Z, g["r"], g["s"], g["t"], g["u"][0])[0], g["y"])
    W0 = oracle_mod.bqq_dense_weight(Y[:1], Z[:1], g["r"][:1], g["s"][:1], g["t"][:1], g["u"][0])
    assert np.array_equal(W0, np.array(g["W_term0"]).reshape(2, 2))
    assert np.array_equal(oracle_mod.bqq_forward(x, Y[:1], Z[:1], g["r"][:1], g["s"][:1], g["t"][:1], g["u"][0])[0],
                          g["y_term0"])


@pytest.mark.parametrize("n,k,m", [(3, 5, 7), (16, 8, 33), (64, 40, 48)])
def test_bqq_product_term_is_integer_matmul(oracle_mod, n, k, m):
    rng = np.random.default_rng(n * k * m)
    Y = rng.integers(0, 2, size=(n, k)).astype(np.int8)
    Z = rng.integers(0, 2, size=(k, m)).astype(np.int8)
    W = oracle_mod.bqq_dense_weight(Y, Z, [1.0], [0.0], [0.0], 0.0)
    assert np.array_equal(W, (Y.astype(np.int64) @ Z.astype(np.int64)).astype(np.float64))


def test_bqq_all_ones_closed_form(oracle_mod):
    p, n, k, m = 3, 5, 6, 4
    r, s, t, u = [0.5, -1.0, 2.0], [1.0, 0.25, -0.5], [-2.0, 1.0, 0.75], 0.125
    W = oracle_mod.bqq_dense_weight(np.ones((p, n, k)), np.ones((p, k, m)), r, s, t, u)
    expect = sum(k * (r[i] + s[i] + t[i]) for i in range(p)) + u
    assert np.array_equal(W, np.full((n, m), expect))


@pytest.mark.parametrize("p,n,k,m", [(1, 8, 16, 12), (3, 33, 24, 17), (2, 64, 64, 64)])
def test_bqq_reduces_to_dbf_weight(oracle_mod, p, n, k, m):
    """{0,1} matrices as signs S = 1 - 2 Y: Y Z = (1 - S_Y)(1 - S_Z) / 4, so
    s_i = t_i = -r_i / 2 and u = k sum(r) / 4 leave sum_i (r_i / 4) S_Yi S_Zi."""
    rng = np.random.default_rng(p * 100 + n)
    Y = rng.integers(0, 2, size=(p, n, k)).astype(np.int8)
    Z = rng.integers(0, 2, size=(p, k, m)).astype(np.int8)
    r = np.array([0.5, -2.0, 1.5][:p])
    W = oracle_mod.bqq_dense_weight(Y, Z, r, -r / 2, -r / 2, k * r.sum() / 4)
    A = np.concatenate([1 - 2 * Y[i].astype(np.int8) for i in range(p)], axis=1)
    B = np.concatenate([1 - 2 * Z[i].astype(np.int8) for i in range(p)], axis=0)
    mid = np.repeat(r / 4, k)
    W_dbf = oracle_mod.dense_weight(A, B, np.ones(n), mid, np.ones(m))
    assert np.allclose(W, W_dbf, rtol=0, atol=1e-12 * np.abs(W_dbf).max())


def test_bqq_without_product_terms_has_rank_two(oracle_mod):
    rng = np.random.default_rng(4)
    Y, Z, _, s, t, u = _random_bqq(rng, 3, 40, 16, 30)
    W = oracle_mod.bqq_dense_weight(Y, Z, np.zeros(3), s, t, u)
    sv = np.linalg.svd(W, compute_uv=False)
    assert sv[2] <= 1e-9 * sv[0] and sv[1] > 1e-6 * sv[0]


def test_bqq_forward_is_x_times_w_transposed(oracle_mod):
    rng = np.random.default_rng(6)
    Y, Z, r, s, t, u = _random_bqq(rng, 2, 24, 16, 40)
    x = rng.standard_normal((5, 40))
    W = oracle_mod.bqq_dense_weight(Y, Z, r, s, t, u)
    assert np.allclose(oracle_mod.bqq_forward(x, Y, Z, r, s, t, u), x @ W.T, rtol=1e-12, atol=1e-12)
