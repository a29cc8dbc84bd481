"""fp64 reference of the offline DBF factorisation of a dense weight (test infrastructure).

Only ``tests/`` and ``bench.py``'s CPU legs may import this module; the product
never does.  It follows the optimisation of "Addition is almost all you need"
(gist.science technical summary, section 2.2, optimisation algorithm) in the
pages' order, with the steps the pages leave open filled in by the plainest
reading (each marked below):

1. SVID projection (Sign-Value-Independent Decomposition, as in OneBit): a real
   matrix M is projected onto {diag(u) S diag(v) : S in {+-1}, u, v >= 0} by
   S = sign(M) (0 taken as +1) and u v^T the best rank-one approximation of |M|
   (its leading singular pair; both vectors are nonnegative because |M| is).
2. Start (reading: a random projection of W's range, each factor projected by
   SVID): with Omega an m x k random sign matrix scaled by 1/sqrt(m) (an input,
   drawn by the caller), L = SVID(W Omega) (n x k) and R = SVID(Omega^T) (k x m),
   in the forms L = diag(a) A diag(mL), R = diag(mR) B diag(b); the middle
   vector is mL (.) mR.  (A truncated-SVD start was tried: after the same
   passes it ends 1-3% higher, and far higher when k exceeds W's rank.)
3. Alternating minimisation: with R fixed, the sign-constrained least-squares
   problem min_L ||W - L R||_F^2, L in the SVID set, is solved by ADMM (the
   pages name ADMM for the constrained problem; reading: scaled ADMM on the
   splitting L = Z, Z in the set):
       L <- (2 W R^T + rho (Z - U)) (2 R R^T + rho I)^-1
       Z <- SVID(L + U)
       U <- U + L - Z
   and then the same for R with L fixed (on the transposed problem).
   A pass is accepted only if it lowers the reconstruction error (reading: the
   pages report the error falling; accepting only improving passes makes the
   reported error monotone by construction).
Importance weighting (the pages' section 2.2 item 4) needs calibration
activations and gradients and is not included.
"""
from __future__ import annotations

import numpy as np


def sign_pm1(M: np.ndarray) -> np.ndarray:
    """+1 where M >= 0 (zeros included), -1 where M < 0, as int8."""
    return np.where(np.asarray(M) < 0, -1, 1).astype(np.int8)


def svid(M: np.ndarray):
    """SVID projection: returns (u, S, v) with M ~= diag(u) S diag(v), u, v >= 0."""
    M = np.asarray(M, dtype=np.float64)
    S = sign_pm1(M)
    U, sig, Vt = np.linalg.svd(np.abs(M), full_matrices=False)
    u = np.abs(U[:, 0]) * np.sqrt(sig[0])
    v = np.abs(Vt[0, :]) * np.sqrt(sig[0])
    return u, S, v


def svid_matrix(M: np.ndarray) -> np.ndarray:
    u, S, v = svid(M)
    return u[:, None] * S * v[None, :]


def relative_error(W: np.ndarray, L: np.ndarray, R: np.ndarray) -> float:
    return float(np.linalg.norm(W - L @ R) / np.linalg.norm(W))


def start_factors(W: np.ndarray, Omega: np.ndarray):
    """Step 2: L = SVID(W Omega), R = SVID(Omega^T) for an m x k projection Omega."""
    W = np.asarray(W, dtype=np.float64)
    Omega = np.asarray(Omega, dtype=np.float64)
    return svid_matrix(W @ Omega), svid_matrix(Omega.T)


def admm_left(W: np.ndarray, R: np.ndarray, Z0: np.ndarray, rho: float | None, steps: int) -> np.ndarray:
    """Step 3 for the left factor: min ||W - L R||^2, L in the SVID set (R fixed).
    rho defaults to the mean curvature of the least-squares term, trace(2 R R^T) / k
    (reading: the pages give no penalty; this scale worked best in a sweep of 0.25x..4x)."""
    k = R.shape[0]
    if rho is None:
        rho = 2.0 * float(np.sum(R * R)) / k or 1.0
    G = 2.0 * R @ R.T + rho * np.eye(k)
    WR = 2.0 * W @ R.T
    Z, Ud = Z0.copy(), np.zeros_like(Z0)
    for _ in range(steps):
        L = np.linalg.solve(G, (WR + rho * (Z - Ud)).T).T  # G is symmetric
        Z = svid_matrix(L + Ud)
        Ud = Ud + L - Z
    return Z


def alternating_pass(W: np.ndarray, L: np.ndarray, R: np.ndarray, admm_steps: int = 20, rho: float | None = None):
    """Step 3, one pass: the left factor with R fixed, then the right factor with the new L fixed."""
    Ln = admm_left(W, R, L, rho, admm_steps)
    Rn = admm_left(W.T, Ln.T, R.T, rho, admm_steps).T
    return Ln, Rn


def factorize(W: np.ndarray, Omega: np.ndarray, passes: int = 10, admm_steps: int = 20, rho: float | None = None):
    """DBF factorisation W ~= (a (.) A (.) mid^T)(B (.) b^T) with k = Omega.shape[1].

    Returns a dict with A (n x k int8), B (k x m int8), a, mid, b (fp64) and
    `errors`: the relative Frobenius error of the start and after each
    alternating pass (non-increasing)."""
    W = np.asarray(W, dtype=np.float64)
    L, R = start_factors(W, Omega)
    best = relative_error(W, L, R)
    errors = [best]
    for _ in range(passes):
        Ln, Rn = alternating_pass(W, L, R, admm_steps, rho)
        err = relative_error(W, Ln, Rn)
        if err < best:
            L, R, best = Ln, Rn, err
        errors.append(best)
    a, A, mL = svid(L)
    mR, B, b = svid(R)
    return {"A": A, "B": B, "a": a, "mid": mL * mR, "b": b, "errors": errors}


def reconstruct(f) -> np.ndarray:
    """(a (.) A (.) mid^T)(B (.) b^T) of a factorisation."""
    return (f["a"][:, None] * f["A"] * f["mid"][None, :]) @ (f["B"] * f["b"][None, :])
