"""CPU fp64 oracle of the LB-ADMM initialiser of the binary factorisation (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this module; the product package never does, and this module imports nothing from it.

What the method does (hardwired.dev, "NanoQuant jednoduse: 70B model na herni grafice",
section "Trikrokovy pipeline", step 2 "Inicializace binarni faktorizace (LB-ADMM)"): ADMM
finds the binary matrices and scaling factors that best approximate the layer's weights,
alternating two sub-problems, a closed-form least-squares solve for the continuous
parameters and a projection onto the binary constraint by the sign operation; magnitude
balancing of the scaling factors follows.  The initialiser's routines are named
power_iteration, rank1_approx, svid and factorize_admm_nanoquant (codewithpapers.app record
of arXiv 2602.06694, code-sample list); their bodies are not given.  The pages give no
formula, so this module states a reading of its own (every point also listed in the
repository's design notes).  Of the named routines it keeps the power iteration (as a block
power iteration for the start); a rank-one or sign-value decomposition has no step in it
(with r = 1 the whole factorisation is the rank-one problem, which the tests use as a pin):

  objective   min || W - diag(s1) U V^T diag(s2) ||_F,  U in {+-1}^{m x r}, V in {+-1}^{n x r},
              written as W ~= A B^T with the latent real factors A (m x r), B (n x r)
              constrained to the row-scaled sign sets C = { diag(s) S : S in {+-1}^{. x r} }
              (A = diag(s1) U and B = diag(s2) V give the stored form exactly);
  splitting   A = Z_A, B = Z_B with Z_A, Z_B in C, scaled duals L_A, L_B;
  LS step     A <- argmin_A ||W - A B^T||^2 + rho_A ||A - (Z_A - L_A)||^2
                 = (W B + rho_A (Z_A - L_A)) (B^T B + rho_A I)^-1        (closed form)
              then the same for B with W^T and the new A (Gauss-Seidel order: A, then B);
  penalty     rho_A = lam_k tr(B^T B) / r, rho_B = lam_k tr(A^T A) / r (the scale of the
              fixed factor, so the step is invariant to rescaling W), lam_k = lam0 growth^k;
  projection  Z = Pi(A + L_A): per row, the signs S = sign(row) (sign(0) = +1, as the
              packed storage) and the least-squares scale s = mean_k |row_k| (for fixed
              signs the best scale of a row is <row, S> / r);
  dual        L_A <- L_A + A - Z_A (likewise B);
  init        a block power iteration from a seeded Gaussian n x r start Omega: Q = orth(W
              Omega), q times Q = orth(W (W^T Q)), orth by Cholesky-QR (Y L^-T with
              L L^T = Y^T Y); A0 = Q, B0 = W^T Q (the least-squares fit to Q), then each
              column pair rescaled to equal norms (product unchanged); Z = Pi(A0), Pi(B0),
              duals zero;
  result      U, s_A from Z_A and V, s_B from Z_B after the last iteration;
  balancing   s1 = c s_A, s2 = s_B / c with c = sqrt(rms(s_B) / rms(s_A)), so that both
              scale vectors have the same root-mean-square (the product is unchanged).

Library primitives serve as steps (numpy's matmul, Cholesky and linear solve); nothing is
blocked, fused or reordered beyond the steps above.
"""
from __future__ import annotations

import numpy as np


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact: bfloat16 is the top half of a binary32)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def project(M: np.ndarray):
    """Pi: the nearest row-scaled sign matrix.  Returns (S int8 in {+-1}, s per row, Z)."""
    M = np.asarray(M, dtype=np.float64)
    S = np.where(M >= 0.0, 1, -1).astype(np.int8)
    s = np.abs(M).sum(axis=1) / M.shape[1]
    return S, s, s[:, None] * S


def penalty(F: np.ndarray, lam: float) -> float:
    """rho for the update of the factor paired with F: lam * tr(F^T F) / r."""
    return lam * float(np.sum(F * F)) / F.shape[1]


def ls_update(W: np.ndarray, F: np.ndarray, C: np.ndarray, rho: float) -> np.ndarray:
    """argmin_X ||W - X F^T||_F^2 + rho ||X - C||_F^2 = (W F + rho C)(F^T F + rho I)^-1."""
    r = F.shape[1]
    H = F.T @ F + rho * np.eye(r)
    R = W @ F + rho * C
    return np.linalg.solve(H, R.T).T  # H is symmetric: X H = R  <=>  H X^T = R^T


def orthonormalize(Y: np.ndarray) -> np.ndarray:
    """Cholesky-QR: Y L^-T with L L^T = Y^T Y (orthonormal columns spanning Y's)."""
    L = np.linalg.cholesky(Y.T @ Y)
    return np.linalg.solve(L, Y.T).T


def power_iteration_init(W: np.ndarray, Omega: np.ndarray, q: int):
    """Latent start (A0, B0): block power iteration from Omega, then column balancing."""
    Q = orthonormalize(W @ Omega)
    for _ in range(q):
        Q = orthonormalize(W @ (W.T @ Q))
    A = Q
    B = W.T @ Q
    c = np.sqrt(np.linalg.norm(B, axis=0) / np.linalg.norm(A, axis=0))
    return A * c, B / c


def admm_step(W: np.ndarray, st: dict, lam: float) -> dict:
    """One iteration: the A update, its projection and dual, then the same for B."""
    A = ls_update(W, st["B"], st["ZA"] - st["LA"], penalty(st["B"], lam))
    SA, sA, ZA = project(A + st["LA"])
    LA = st["LA"] + A - ZA
    B = ls_update(W.T, A, st["ZB"] - st["LB"], penalty(A, lam))
    SB, sB, ZB = project(B + st["LB"])
    LB = st["LB"] + B - ZB
    return dict(A=A, B=B, ZA=ZA, ZB=ZB, LA=LA, LB=LB, SA=SA, SB=SB, sA=sA, sB=sB)


def start_state(A0: np.ndarray, B0: np.ndarray) -> dict:
    SA, sA, ZA = project(A0)
    SB, sB, ZB = project(B0)
    return dict(A=A0, B=B0, ZA=ZA, ZB=ZB, LA=np.zeros_like(A0), LB=np.zeros_like(B0), SA=SA, SB=SB, sA=sA, sB=sB)


def magnitude_balance(sA: np.ndarray, sB: np.ndarray):
    """(c sA, sB / c) with c = sqrt(rms(sB) / rms(sA)): equal root-mean-squares."""
    rA = np.sqrt(np.mean(sA * sA))
    rB = np.sqrt(np.mean(sB * sB))
    if rA == 0.0 or rB == 0.0:
        return sA.copy(), sB.copy()
    c = np.sqrt(rB / rA)
    return sA * c, sB / c


def reconstruction_error(W: np.ndarray, U, V, s1, s2) -> float:
    """||W - diag(s1) U V^T diag(s2)||_F / ||W||_F."""
    W = np.asarray(W, dtype=np.float64)
    P = (np.asarray(s1, np.float64)[:, None] * np.asarray(U, np.float64)) @ \
        (np.asarray(s2, np.float64)[:, None] * np.asarray(V, np.float64)).T
    return float(np.linalg.norm(W - P) / np.linalg.norm(W))


def factorize(W: np.ndarray, Omega: np.ndarray, iters: int, lam0: float = 0.2, growth: float = 1.05,
              q: int = 1, history: bool = False):
    """The whole initialiser on a real m x n W (float64) with the start Omega (n x r).

    Returns (U int8 m x r, V int8 n x r, s1, s2) and, with history=True, also the relative
    reconstruction error of the projected factors after the start and after each iteration.
    """
    W = np.asarray(W, dtype=np.float64)
    A0, B0 = power_iteration_init(W, np.asarray(Omega, dtype=np.float64), q)
    st = start_state(A0, B0)
    hist = [reconstruction_error(W, st["SA"], st["SB"], st["sA"], st["sB"])] if history else None
    lam = lam0
    for _ in range(iters):
        st = admm_step(W, st, lam)
        lam *= growth
        if history:
            hist.append(reconstruction_error(W, st["SA"], st["SB"], st["sA"], st["sB"]))
    s1, s2 = magnitude_balance(st["sA"], st["sB"])
    out = (st["SA"].copy(), st["SB"].copy(), s1, s2)
    return (out + (hist,)) if history else out
