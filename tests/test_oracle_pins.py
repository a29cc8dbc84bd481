"""Pins for the fp64 oracle: each check ties it to something other than itself.

Sources of truth used here (none of them calls the oracle's C code):
  * a forward worked by hand (tests/golden/worked_example_2x2x3.txt);
  * exact integer arithmetic (numpy int64 / Python Fractions) on tiny shapes,
    exhaustively at n = k = m_in = 2;
  * the Sylvester-Hadamard closed form: with A = B = H_k, H_k H_k = k I, and the
    staged product equals a (.) FWHT(mid (.) FWHT(b (.) x)), with a butterfly
    FWHT written here;
  * the k = 1 rank-one closed form;
  * invariances of the factorisation (sign moves, middle permutation);
  * the bits/weight closed form against packed byte counts;
  * the documented packed layout table (tests/golden/packed_layout_bits.txt).
The factorisation and evaluation order follow "Addition is almost all you
need", gist.science technical summary section 2.1.
"""
from fractions import Fraction

import numpy as np
import pytest

import dbf_inputs as gen
from conftest import read_golden


# ---------------------------------------------------------------- worked example
def test_hand_worked_example(oracle_mod):
    g = read_golden("worked_example_2x2x3.txt")
    n, k, m_in = int(g["n"][0]), int(g["k"][0]), int(g["m_in"][0])
    A = np.array(g["A"], dtype=np.int8).reshape(n, k)
    B = np.array(g["B"], dtype=np.int8).reshape(k, m_in)
    x = np.array(g["x"]).reshape(1, m_in)
    y = oracle_mod.forward_staged(x, A, B, g["a"], g["mid"], g["b"])
    assert y.tolist() == [g["y"]]
    W = oracle_mod.dense_weight(A, B, g["a"], g["mid"], g["b"])
    assert W.reshape(-1).tolist() == g["W"]
    assert oracle_mod.forward_dense(x, W).tolist() == [g["y"]]


# ---------------------------------------------------------------- exact integer brute force
def _exact_int_forward(x, A, B, a, mid, b):
    """y = x W^T with W = diag(a) A diag(mid) B diag(b), all in int64."""
    W = (a[:, None] * A.astype(np.int64) * mid[None, :]) @ (B.astype(np.int64) * b[None, :])
    return x.astype(np.int64) @ W.T


def test_exhaustive_2x2x2(oracle_mod):
    """Every 2x2 sign pair (2^8 patterns) times every x in {-2..2}^2, integer scales."""
    xs = np.array([[p, q] for p in range(-2, 3) for q in range(-2, 3)], dtype=np.int64)
    a = np.array([3, -2], dtype=np.int64)
    mid = np.array([2, 5], dtype=np.int64)
    b = np.array([-1, 4], dtype=np.int64)
    for pattern in range(256):
        bits = [(pattern >> i) & 1 for i in range(8)]
        A = np.array([1 - 2 * v for v in bits[:4]], dtype=np.int8).reshape(2, 2)
        B = np.array([1 - 2 * v for v in bits[4:]], dtype=np.int8).reshape(2, 2)
        y = oracle_mod.forward_staged(xs, A, B, a, mid, b)
        assert np.array_equal(y, _exact_int_forward(xs, A, B, a, mid, b).astype(np.float64)), pattern


@pytest.mark.parametrize("n,k,m_in", [(1, 1, 1), (3, 2, 5), (5, 7, 3), (8, 4, 8), (2, 8, 6)])
def test_brute_force_fractions(oracle_mod, n, k, m_in):
    """Non-integer fp16-exact scales: compare to exact rational arithmetic."""
    rng = np.random.default_rng(17 + n * 100 + k * 10 + m_in)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    a = gen.abs_normal_scales(rng, n)
    mid = -gen.abs_normal_scales(rng, k)  # negative scales are legal too
    b = gen.abs_normal_scales(rng, m_in)
    x = gen.normal_activations(rng, 3, m_in)
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    F = lambda v: Fraction(float(v))  # fp16 -> float is exact, float -> Fraction is exact
    for t in range(3):
        for i in range(n):
            exact = sum(
                F(a[i]) * int(A[i, l]) * F(mid[l]) * int(B[l, j]) * F(b[j]) * F(x[t, j])
                for l in range(k)
                for j in range(m_in)
            )
            got = y[t, i]
            assert abs(Fraction(got) - exact) <= abs(exact) * Fraction(1, 10**12) + Fraction(1, 10**30)


# ---------------------------------------------------------------- associativity
@pytest.mark.parametrize("n,k,m_in,batch", [(256, 128, 256, 3), (96, 64, 320, 2), (40, 192, 64, 5)])
def test_staged_equals_dense(oracle_mod, n, k, m_in, batch):
    """Staged evaluation (computation process) vs dense reconstruction (factorisation)."""
    rng = np.random.default_rng(n + k + m_in)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    a, mid, b = gen.lognormal_scales(rng, n), gen.abs_normal_scales(rng, k), gen.lognormal_scales(rng, m_in)
    x = gen.normal_activations(rng, batch, m_in)
    y_staged = oracle_mod.forward_staged(x, A, B, a, mid, b)
    y_dense = oracle_mod.forward_dense(x, oracle_mod.dense_weight(A, B, a, mid, b))
    rel = np.linalg.norm(y_staged - y_dense) / np.linalg.norm(y_dense)
    assert rel < 1e-12
    # and against numpy's own matmul of the dense factors
    xf = x.astype(np.float64)
    W_np = (a.astype(np.float64)[:, None] * A * mid.astype(np.float64)[None, :]) @ (B * b.astype(np.float64)[None, :])
    rel_np = np.linalg.norm(y_staged - xf @ W_np.T) / np.linalg.norm(y_staged)
    assert rel_np < 1e-12


# ---------------------------------------------------------------- integer invariant
def test_integer_mode_is_exact(oracle_mod):
    shape = gen.CONFIGS["tiny_int"]
    L = gen.make_layer(shape, batch=4)
    y = oracle_mod.forward_staged(L["x"], L["A"], L["B"], L["a"], L["mid"], L["b"])
    assert np.all(y == np.round(y))
    one_n, one_k, one_m = (np.ones(s, dtype=np.int64) for s in (shape.n, shape.k, shape.m_in))
    exact = _exact_int_forward(L["x"].astype(np.int64), L["A"], L["B"], one_n, one_k, one_m)
    assert np.array_equal(y, exact.astype(np.float64))
    # the middle vector stays inside fp16's exact-integer range for this recipe
    _, v = oracle_mod.forward_staged(L["x"], L["A"], L["B"], L["a"], L["mid"], L["b"], return_v=True)
    assert np.abs(v).max() <= 2048


# ---------------------------------------------------------------- Hadamard closed form
def _fwht(v):
    """Unnormalised Walsh-Hadamard transform in Sylvester order, butterfly form, last axis."""
    v = np.array(v, dtype=np.float64, copy=True)
    h = 1
    size = v.shape[-1]
    while h < size:
        v = v.reshape(v.shape[:-1] + (size // (2 * h), 2, h))
        lo, hi = v[..., 0, :].copy(), v[..., 1, :].copy()
        v[..., 0, :], v[..., 1, :] = lo + hi, lo - hi
        v = v.reshape(v.shape[:-3] + (size,))
        h *= 2
    return v


def test_sylvester_pattern_matches_scipy():
    scipy_linalg = pytest.importorskip("scipy.linalg")
    for p in range(0, 7):
        assert np.array_equal(gen.sylvester_hadamard(p), scipy_linalg.hadamard(1 << p).astype(np.int8))


@pytest.mark.parametrize("p", [1, 3, 6, 8])
def test_hadamard_closed_form(oracle_mod, p):
    size = 1 << p
    H = gen.sylvester_hadamard(p)
    rng = np.random.default_rng(p)
    x = gen.integer_activations(rng, 3, size)
    ones = np.ones(size, dtype=np.float16)
    # unit scales: H H = size * I, so y = size * x exactly
    y = oracle_mod.forward_staged(x, H, H, ones, ones, ones)
    assert np.array_equal(y, size * x.astype(np.float64))
    # general scales: y = a (.) FWHT(mid (.) FWHT(b (.) x))
    a, mid, b = gen.abs_normal_scales(rng, size), gen.lognormal_scales(rng, size), gen.abs_normal_scales(rng, size)
    xn = gen.normal_activations(rng, 3, size)
    y = oracle_mod.forward_staged(xn, H, H, a, mid, b)
    closed = a.astype(np.float64) * _fwht(mid.astype(np.float64) * _fwht(b.astype(np.float64) * xn.astype(np.float64)))
    assert np.allclose(y, closed, rtol=1e-12, atol=1e-12 * np.abs(closed).max())


# ---------------------------------------------------------------- rank-one closed form
def test_k1_outer_product(oracle_mod):
    rng = np.random.default_rng(5)
    n, m_in = 37, 53
    A = gen.sign_matrix(rng, n, 1)
    B = gen.sign_matrix(rng, 1, m_in)
    a, mid, b = gen.lognormal_scales(rng, n), gen.abs_normal_scales(rng, 1), gen.abs_normal_scales(rng, m_in)
    x = gen.integer_activations(rng, 4, m_in)
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    inner = x.astype(np.float64) @ (B[0].astype(np.float64) * b.astype(np.float64))  # <B[0,:], b (.) x>
    closed = np.outer(inner * float(mid[0]), a.astype(np.float64) * A[:, 0])
    assert np.allclose(y, closed, rtol=1e-14, atol=0)


# ---------------------------------------------------------------- invariances
def _layer(seed, n=48, k=64, m_in=80, batch=3):
    rng = np.random.default_rng(seed)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    x = gen.integer_activations(rng, batch, m_in)
    a = rng.integers(-3, 4, n).astype(np.float16)
    mid = rng.integers(-3, 4, k).astype(np.float16)
    b = rng.integers(-3, 4, m_in).astype(np.float16)
    return x, A, B, a, mid, b


def test_invariance_row_sign_move(oracle_mod):
    x, A, B, a, mid, b = _layer(1)
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    A2, a2 = A.copy(), a.copy()
    A2[[3, 7, 11]] *= -1
    a2[[3, 7, 11]] *= -1
    assert np.array_equal(oracle_mod.forward_staged(x, A2, B, a2, mid, b), y)


def test_invariance_middle_sign_move(oracle_mod):
    x, A, B, a, mid, b = _layer(2)
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    cols = [0, 5, 63]
    A2, B2 = A.copy(), B.copy()
    A2[:, cols] *= -1
    B2[cols, :] *= -1
    assert np.array_equal(oracle_mod.forward_staged(x, A2, B2, a, mid, b), y)
    mid2 = mid.copy()
    mid2[cols] *= -1
    A3 = A.copy()
    A3[:, cols] *= -1
    assert np.array_equal(oracle_mod.forward_staged(x, A3, B, a, mid2, b), y)


def test_invariance_middle_permutation(oracle_mod):
    x, A, B, a, mid, b = _layer(3)
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    perm = np.random.default_rng(9).permutation(A.shape[1])
    assert np.array_equal(oracle_mod.forward_staged(x, A[:, perm], B[perm, :], a, mid[perm], b), y)


def test_orientation_is_not_transposed(oracle_mod):
    """b scales inputs (columns of B), a scales outputs (rows of A): check with one-hot scales."""
    x, A, B, a, mid, b = _layer(4, n=6, k=4, m_in=9, batch=1)
    x = np.ones((1, 9), dtype=np.float16)
    a = np.ones(6, dtype=np.float16)
    mid = np.ones(4, dtype=np.float16)
    b = np.zeros(9, dtype=np.float16)
    b[2] = 1  # only input column 2 survives
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    assert np.array_equal(y[0], (A.astype(np.float64) @ B[:, 2].astype(np.float64)))
    a = np.zeros(6, dtype=np.float16)
    a[4] = 1  # only output row 4 survives
    b = np.ones(9, dtype=np.float16)
    y = oracle_mod.forward_staged(x, A, B, a, mid, b)
    expect = np.zeros(6)
    expect[4] = A[4].astype(np.float64) @ B.astype(np.float64).sum(axis=1)
    assert np.array_equal(y[0], expect)


# ---------------------------------------------------------------- bits per weight
@pytest.mark.parametrize(
    "n,k,m_in,expect",
    [(4096, 2048, 4096, 1.0), (4096, 4096, 4096, 2.0), (14336, 4736, 4096, 4736 * 18432 / (14336 * 4096)),
     (256, 256, 256, 2.0), (256, 128, 256, 1.0)],
)
def test_bits_per_weight_closed_form(oracle_mod, n, k, m_in, expect):
    assert oracle_mod.bits_per_weight(n, k, m_in) == pytest.approx(expect, rel=1e-15)
    # packed sign storage: with k and m_in multiples of 256 there is no padding, so bits = k*n + k*m_in
    if k % 256 == 0 and m_in % 256 == 0:
        words = n * oracle_mod.words_per_row(k) + k * oracle_mod.words_per_row(m_in)
        assert words * 32 / (n * m_in) == pytest.approx(expect, rel=1e-15)


@pytest.mark.parametrize("n,k,m_in", [(4096, 2048, 4096), (4096, 4096, 4096), (14336, 4736, 4096), (1024, 832, 4096),
                                      (4096, 3200, 14336), (256, 128, 256), (3, 64, 5)])
def test_scale_bits_per_weight_counts_stored_vectors(oracle_mod, n, k, m_in):
    """The three scale vectors are stored as fp16 (sciencestack.ai Figure 1; gist.science section 2.1 names
    a, m, b as FP16 vectors): their storage, counted from real fp16 arrays of lengths n, k and m_in,
    spread over the n * m_in weights of the dense layer."""
    rng = np.random.default_rng(n + k + m_in)
    vecs = [gen.lognormal_scales(rng, n), gen.lognormal_scales(rng, k), gen.lognormal_scales(rng, m_in)]
    assert all(v.dtype == np.float16 for v in vecs)
    stored_bits = 8 * sum(v.nbytes for v in vecs)
    assert oracle_mod.scale_bits_per_weight(n, k, m_in) == pytest.approx(stored_bits / (n * m_in), rel=1e-15)


def test_bits_per_weight_rounding_rule():
    """k for a target bit rate: nearest multiple of 64, ties up (layer set recipe)."""
    def k_for(n, m_in, bits):
        exact = bits * n * m_in / (n + m_in)
        return int(np.floor(exact / 64 + 0.5)) * 64

    for bits, shapes in gen.LAYER_SET.items():
        for s in shapes:
            assert s.k == k_for(s.n, s.m_in, bits), s.name


# ---------------------------------------------------------------- packed layout
def _layout_table():
    rows = []
    from conftest import GOLDEN
    import os

    with open(os.path.join(GOLDEN, "packed_layout_bits.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(v) for v in line.split()))
    return rows


def test_layout_table(oracle_mod):
    for col, word, bit in _layout_table():
        cols = 768
        wpr = (cols + 255) // 256 * 8
        signs = np.ones((1, cols), dtype=np.int8)
        signs[0, col] = -1
        packed = oracle_mod.pack_signs(signs)
        expect = np.zeros(wpr, dtype=np.uint32)
        expect[word] = np.uint32(1 << bit)
        assert np.array_equal(packed, expect), (col, word, bit)
        back, bad = oracle_mod.unpack_signs(expect, 1, cols)
        assert bad == 0 and np.array_equal(back, signs)


def test_layout_hand_words(oracle_mod):
    # word 0 = 0x0000FFFF: bits 0..15 are pair 0, even column, of groups 0..15 -> columns 0, 16, ..., 240
    packed = np.zeros(8, dtype=np.uint32)
    packed[0] = 0x0000FFFF
    back, bad = oracle_mod.unpack_signs(packed, 1, 256)
    assert bad == 0
    assert [int(i) for i in np.nonzero(back[0] < 0)[0]] == list(range(0, 256, 16))
    # word 3 = 0xFFFF0000: bits 16..31 are pair 3, odd column -> columns 16g + 7
    packed[:] = 0
    packed[3] = 0xFFFF0000
    back, _ = oracle_mod.unpack_signs(packed, 1, 256)
    assert [int(i) for i in np.nonzero(back[0] < 0)[0]] == [16 * g + 7 for g in range(16)]
    # rows are 8 words apart for cols <= 256; second block of a row starts at word 8
    packed = np.zeros(32, dtype=np.uint32)
    packed[8] = 1 << 16  # row 0, column 257
    packed[16 + 15] = 1 << 31  # row 1, column 511
    back, bad = oracle_mod.unpack_signs(packed, 2, 512)
    assert bad == 0
    assert [int(i) for i in np.nonzero(back[0] < 0)[0]] == [257]
    assert [int(i) for i in np.nonzero(back[1] < 0)[0]] == [511]


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 128), (5, 192), (17, 320), (2, 1000), (4, 832)])
def test_layout_round_trip_and_padding(oracle_mod, rows, cols):
    rng = np.random.default_rng(rows * cols)
    s = gen.sign_matrix(rng, rows, cols)
    packed = oracle_mod.pack_signs(s)
    wpr = ((cols + 255) // 256) * 8
    assert packed.size == rows * wpr
    back, bad = oracle_mod.unpack_signs(packed, rows, cols)
    assert bad == 0 and np.array_equal(back, s)
    if cols % 256:
        corrupt = packed.copy()
        corrupt[wpr - 1] |= np.uint32(1 << 31)  # group 15, pair 7, odd: column 255 of the last block
        assert oracle_mod.unpack_signs(corrupt, rows, cols)[1] == 1


# ---------------------------------------------------------------- the transpose product dx = dy W
@pytest.mark.parametrize("n,k,m_in,batch", [(48, 64, 80, 3), (7, 5, 11, 2)])
def test_transposed_adjoint_identity(oracle_mod, n, k, m_in, batch):
    """<y(x), dy> = <x, dx(dy)> for every x and dy: the defining property of the transpose."""
    rng = np.random.default_rng(7 * n + k)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    a, mid, b = gen.lognormal_scales(rng, n), gen.abs_normal_scales(rng, k), gen.lognormal_scales(rng, m_in)
    x = gen.normal_activations(rng, batch, m_in).astype(np.float64)
    dy = gen.normal_activations(rng, batch, n).astype(np.float64)
    lhs = np.sum(oracle_mod.forward_staged(x, A, B, a, mid, b) * dy)
    rhs = np.sum(x * oracle_mod.forward_transposed(dy, A, B, a, mid, b))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


@pytest.mark.parametrize("n,k,m_in,batch", [(96, 64, 320, 2), (33, 64, 65, 3)])
def test_transposed_equals_dense(oracle_mod, n, k, m_in, batch):
    """dx = dy W against numpy's matmul with the dense factors written out here."""
    rng = np.random.default_rng(n * k + m_in)
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    a, mid, b = gen.abs_normal_scales(rng, n), gen.lognormal_scales(rng, k), gen.abs_normal_scales(rng, m_in)
    dy = gen.normal_activations(rng, batch, n).astype(np.float64)
    W_np = (a.astype(np.float64)[:, None] * A * mid.astype(np.float64)[None, :]) @ (B * b.astype(np.float64)[None, :])
    dx = oracle_mod.forward_transposed(dy, A, B, a, mid, b)
    assert np.linalg.norm(dx - dy @ W_np) <= 1e-12 * np.linalg.norm(dx)


@pytest.mark.parametrize("p", [3, 5])
def test_transposed_hadamard_closed_form(oracle_mod, p):
    """A = B = H (symmetric): dx = b (.) FWHT(mid (.) FWHT(a (.) dy))."""
    size = 1 << p
    H = gen.sylvester_hadamard(p)
    rng = np.random.default_rng(100 + p)
    a, mid, b = gen.abs_normal_scales(rng, size), gen.lognormal_scales(rng, size), gen.lognormal_scales(rng, size)
    dy = gen.normal_activations(rng, 2, size).astype(np.float64)
    dx = oracle_mod.forward_transposed(dy, H, H, a, mid, b)
    closed = b.astype(np.float64) * _fwht(mid.astype(np.float64) * _fwht(a.astype(np.float64) * dy))
    assert np.allclose(dx, closed, rtol=1e-12, atol=1e-12 * np.abs(closed).max())


def test_transposed_integer_exact(oracle_mod):
    """Unit scales, integer dy: dx equals the int64 product dy A B."""
    rng = np.random.default_rng(3)
    n, k, m_in = 40, 24, 56
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    dy = rng.integers(-8, 9, size=(3, n))
    ones = lambda s: np.ones(s, dtype=np.float16)
    dx = oracle_mod.forward_transposed(dy, A, B, ones(n), ones(k), ones(m_in))
    exact = dy.astype(np.int64) @ A.astype(np.int64) @ B.astype(np.int64)
    assert np.array_equal(dx, exact.astype(np.float64))


def test_transposed_uses_each_scale_once(oracle_mod):
    """One-hot scales pick single entries: dx[j] = b_j * B[l, j] * mid_l * A[i, l] * a_i * dy[i]."""
    rng = np.random.default_rng(11)
    n, k, m_in = 6, 4, 5
    A = gen.sign_matrix(rng, n, k)
    B = gen.sign_matrix(rng, k, m_in)
    i, l = 2, 1
    a = np.zeros(n, dtype=np.float16)
    a[i] = 3
    mid = np.zeros(k, dtype=np.float16)
    mid[l] = 5
    b = np.arange(1, m_in + 1).astype(np.float16)
    dy = np.zeros((1, n))
    dy[0, i] = 2
    dx = oracle_mod.forward_transposed(dy, A, B, a, mid, b)
    expect = b.astype(np.float64) * B[l].astype(np.float64) * 5 * A[i, l] * 3 * 2
    assert np.array_equal(dx[0], expect)
