"""Pins of the LB-ADMM oracle (oracle/admm.py): each checks it against something other than
itself -- brute force, a differently computed library routine, an exact algebraic identity,
or a planted answer -- chosen so that a plausible mistake in any step fails one of them.

Every pin takes the module under test as its argument, so that the planted-mistake tests
(tests/test_admm_pins.py) can run them against altered copies.
"""
from __future__ import annotations

import itertools

import numpy as np


def _rng(*tags):
    return np.random.default_rng([0xAD33, *tags])


def _planted(m, n, r, seed, noise=0.0):
    """W = diag(s1) U V^T diag(s2) (+ Gaussian noise of `noise` times W's rms)."""
    g = _rng(seed)
    U = np.where(g.standard_normal((m, r)) >= 0, 1, -1).astype(np.int8)
    V = np.where(g.standard_normal((n, r)) >= 0, 1, -1).astype(np.int8)
    s1 = g.uniform(0.5, 1.5, m)
    s2 = g.uniform(0.5, 1.5, n)
    W = (s1[:, None] * U) @ (s2[:, None] * V).T
    if noise:
        W = W + noise * np.sqrt(np.mean(W * W)) * g.standard_normal((m, n))
    return W, U, V, s1, s2


def pin_projection_is_nearest_row_scaled_sign_vector(adm):
    """Brute force over all 2^r sign patterns (r <= 8): no pattern with its best
    non-negative scale is nearer to a row than Pi's pattern and scale."""
    g = _rng(1)
    for r in (1, 3, 8):
        M = g.standard_normal((6, r)) * g.uniform(0.1, 10.0, (6, 1))
        S, s, Z = adm.project(M)
        for i in range(M.shape[0]):
            best = np.inf
            for pat in itertools.product((-1.0, 1.0), repeat=r):
                p = np.array(pat)
                c = max(0.0, float(M[i] @ p) / r)
                best = min(best, float(np.sum((M[i] - c * p) ** 2)))
            got = float(np.sum((M[i] - Z[i]) ** 2))
            assert got <= best * (1 + 1e-12) + 1e-300, (r, i, got, best)
            assert np.all(Z[i] == s[i] * S[i])


def pin_projection_idempotent_and_sign_of_zero(adm):
    g = _rng(2)
    M = g.standard_normal((9, 16))
    M[0, 3] = 0.0
    S, s, Z = adm.project(M)
    S2, s2, Z2 = adm.project(Z)
    assert np.array_equal(S, S2) and np.array_equal(Z, Z2)
    assert S[0, 3] == 1  # the packed storage's sign(0) = +1
    assert set(np.unique(S)) <= {-1, 1}
    # the scale is least squares for the chosen signs: the residual is orthogonal to them
    assert np.max(np.abs(np.sum((M - Z) * S, axis=1))) <= 1e-12 * np.max(np.abs(M)) * 16


def pin_ls_update_matches_augmented_lstsq(adm):
    """The closed form against numpy's least squares on the stacked system
    [F; sqrt(rho) I] x = [w; sqrt(rho) c] row by row, and the gradient vanishing there."""
    g = _rng(3)
    m, n, r = 7, 11, 4
    W, F, C = g.standard_normal((m, n)), g.standard_normal((n, r)), g.standard_normal((m, r))
    rho = 0.37
    X = adm.ls_update(W, F, C, rho)
    stack = np.vstack([F, np.sqrt(rho) * np.eye(r)])
    for i in range(m):
        rhs = np.concatenate([W[i], np.sqrt(rho) * C[i]])
        x, *_ = np.linalg.lstsq(stack, rhs, rcond=None)
        assert np.max(np.abs(x - X[i])) <= 1e-12 * max(1.0, np.max(np.abs(x)))
    grad = (X @ F.T - W) @ F + rho * (X - C)
    assert np.max(np.abs(grad)) <= 1e-11


def pin_penalty_scale(adm):
    """rho = lam * (sum of squares of F) / r, checked on a hand-sized F."""
    F = np.array([[1.0, 2.0], [3.0, -4.0], [0.0, 0.5]])  # sum of squares 30.25, r = 2
    assert abs(adm.penalty(F, 0.2) - 0.2 * 30.25 / 2) <= 1e-15


def pin_orthonormalize(adm):
    """Q^T Q = I, and Y = Q R with R = Q^T Y upper triangular (the same column span, in
    order), against numpy's Householder QR up to column signs."""
    g = _rng(4)
    Y = g.standard_normal((40, 6))
    Q = adm.orthonormalize(Y)
    assert np.max(np.abs(Q.T @ Q - np.eye(6))) <= 1e-12
    R = Q.T @ Y
    assert np.max(np.abs(np.tril(R, -1))) <= 1e-12 * np.max(np.abs(R))
    Qh, _ = np.linalg.qr(Y)
    assert np.max(np.abs(np.abs(Qh.T @ Q) - np.eye(6))) <= 1e-10


def pin_init_spans_and_balances(adm):
    """A W of rank k <= r is reproduced exactly by the start A0 B0^T (the power iteration
    spans W's range); every column pair has equal norms."""
    g = _rng(5)
    m, n, k, r = 30, 25, 5, 5  # Cholesky-QR needs W Omega of full column rank: rank(W) >= r
    W = g.standard_normal((m, k)) @ g.standard_normal((k, n))
    for q in (0, 1, 2):
        A0, B0 = adm.power_iteration_init(W, g.standard_normal((n, r)), q)
        assert np.linalg.norm(W - A0 @ B0.T) <= 1e-10 * np.linalg.norm(W)
        assert np.max(np.abs(np.linalg.norm(A0, axis=0) - np.linalg.norm(B0, axis=0))) <= 1e-10 * np.max(
            np.linalg.norm(A0, axis=0))
    # and for a full-rank W the start is the projection of W onto the span of W Omega
    W = g.standard_normal((m, n))
    Om = g.standard_normal((n, r))
    A0, B0 = adm.power_iteration_init(W, Om, 0)
    Qh, _ = np.linalg.qr(W @ Om)
    assert np.linalg.norm(A0 @ B0.T - Qh @ (Qh.T @ W)) <= 1e-10 * np.linalg.norm(W)


def pin_rank_one_exact(adm):
    """r = 1: W = diag(s1) u v^T diag(s2) is recovered exactly (signs up to one common
    flip), and the balanced scales have equal root-mean-squares."""
    W, U, V, s1, s2 = _planted(40, 24, 1, 6)
    Ug, Vg, t1, t2 = adm.factorize(W, _rng(7).standard_normal((24, 1)), 5)
    assert adm.reconstruction_error(W, Ug, Vg, t1, t2) <= 1e-12
    flip = 1 if Ug[0, 0] == U[0, 0] else -1
    assert np.array_equal(Ug, flip * U) and np.array_equal(Vg, flip * V)
    assert abs(np.sqrt(np.mean(t1 ** 2)) - np.sqrt(np.mean(t2 ** 2))) <= 1e-12 * np.sqrt(np.mean(t1 ** 2))
    assert np.max(np.abs(np.outer(t1, t2) - np.outer(s1, s2))) <= 1e-12 * np.max(np.outer(s1, s2))


def pin_planted_low_rank_binary_recovered(adm):
    """A planted diag(s1) U V^T diag(s2) of rank 8 (noise-free): the sign product U V^T is
    found exactly (the factors up to a signed permutation of their columns) and the scales
    converge, the error falling below 1e-6 by 60 iterations; with 10 % noise the error
    stays at the noise floor (the planted factors' own error)."""
    W, U, V, s1, s2 = _planted(96, 80, 8, 8)
    Ug, Vg, t1, t2 = adm.factorize(W, _rng(9).standard_normal((80, 8)), 60)
    assert np.array_equal(Ug.astype(np.int64) @ Vg.T.astype(np.int64), U.astype(np.int64) @ V.T.astype(np.int64))
    assert adm.reconstruction_error(W, Ug, Vg, t1, t2) <= 1e-6
    Wn, U, V, s1, s2 = _planted(96, 80, 8, 10, noise=0.1)
    floor = adm.reconstruction_error(Wn, U, V, s1, s2)
    Ug, Vg, t1, t2 = adm.factorize(Wn, _rng(11).standard_normal((80, 8)), 40)
    assert adm.reconstruction_error(Wn, Ug, Vg, t1, t2) <= floor * 1.02


def pin_beats_projected_truncated_svd(adm):
    """On a dense Gaussian W with row and column scale spread, the factorisation beats the
    plain alternative the method is compared with: sign-and-scale projection of the
    truncated SVD factors (numpy's SVD), and the ADMM improves on its own start."""
    g = _rng(12)
    m, n, r = 128, 96, 24
    W = np.exp(0.5 * g.standard_normal(m))[:, None] * g.standard_normal((m, n)) * np.exp(0.5 * g.standard_normal(n))
    Uu, S, Vt = np.linalg.svd(W, full_matrices=False)
    A = Uu[:, :r] * np.sqrt(S[:r])
    B = Vt[:r].T * np.sqrt(S[:r])
    SA = np.where(A >= 0, 1, -1)
    SB = np.where(B >= 0, 1, -1)
    svd_err = adm.reconstruction_error(W, SA, SB, np.abs(A).mean(axis=1), np.abs(B).mean(axis=1))
    U, V, s1, s2, hist = adm.factorize(W, g.standard_normal((n, r)), 40, history=True)
    err = adm.reconstruction_error(W, U, V, s1, s2)
    assert err < 0.9 * svd_err, (err, svd_err)
    assert err < 0.9 * hist[0]
    assert abs(err - hist[-1]) <= 1e-12  # balancing does not change the product


def pin_negation_symmetry(adm):
    """factorize(-W) negates U and keeps V and the scales, bit for bit (negation is exact
    and every step is odd in W)."""
    g = _rng(13)
    W = g.standard_normal((32, 24))
    Om = g.standard_normal((24, 6))
    U, V, s1, s2 = adm.factorize(W, Om, 10)
    Un, Vn, t1, t2 = adm.factorize(-W, Om, 10)
    assert np.array_equal(Un, -U) and np.array_equal(Vn, V)
    assert np.array_equal(t1, s1) and np.array_equal(t2, s2)


def pin_balance_keeps_product(adm):
    g = _rng(14)
    a, b = g.uniform(0.1, 3.0, 7) * 100, g.uniform(0.1, 3.0, 5) * 0.01
    s1, s2 = adm.magnitude_balance(a, b)
    assert np.max(np.abs(np.outer(s1, s2) - np.outer(a, b))) <= 1e-13 * np.max(np.outer(a, b))
    assert abs(np.sqrt(np.mean(s1 ** 2)) - np.sqrt(np.mean(s2 ** 2))) <= 1e-12 * np.sqrt(np.mean(s1 ** 2))


def pin_one_step_by_hand(adm):
    """One iteration on a 2 x 2, r = 2 problem, every quantity worked out by hand in
    fractions: W = [[3, 1], [1, 3]], B = I, Z_A = [[1, 1], [1, -1]], Z_B = [[1, 1], [-1, 1]],
    duals zero, lam = 1/2.
      rho_A = 1/2 * tr(I) / 2 = 1/2;  A = (W I + 1/2 Z_A) / (1 + 1/2) = [[7/3, 1], [1, 5/3]]
      Z_A rows: [5/3, 5/3], [4/3, 4/3];  L_A = [[2/3, -2/3], [-1/3, 1/3]]
      rho_B = 1/2 * (49/9 + 1 + 1 + 25/9) / 2 = 23/9
      H = A^T A + rho_B I = [[9, 4], [4, 19/3]] (det 41);  W^T A + rho_B Z_B =
        [[95/9, 65/9], [25/9, 77/9]];  B = that H^-1 = [[25/27, 5/9], [-449/1107, 593/369]]
      Z_B rows: [20/27, 20/27], [-1114/1107, 1114/1107]
      L_B = [[5/27, -5/27], [665/1107, 665/1107]]"""
    W = np.array([[3.0, 1.0], [1.0, 3.0]])
    st = dict(A=np.zeros((2, 2)), B=np.eye(2), ZA=np.array([[1.0, 1.0], [1.0, -1.0]]),
              ZB=np.array([[1.0, 1.0], [-1.0, 1.0]]), LA=np.zeros((2, 2)), LB=np.zeros((2, 2)))
    out = adm.admm_step(W, st, 0.5)
    expect = {
        "A": [[7 / 3, 1.0], [1.0, 5 / 3]],
        "ZA": [[5 / 3, 5 / 3], [4 / 3, 4 / 3]],
        "LA": [[2 / 3, -2 / 3], [-1 / 3, 1 / 3]],
        "B": [[25 / 27, 5 / 9], [-449 / 1107, 593 / 369]],
        "ZB": [[20 / 27, 20 / 27], [-1114 / 1107, 1114 / 1107]],
        "LB": [[5 / 27, -5 / 27], [665 / 1107, 665 / 1107]],
    }
    for key, val in expect.items():
        assert np.max(np.abs(out[key] - np.array(val))) <= 1e-14, key
    assert np.array_equal(out["SB"], np.array([[1, 1], [-1, 1]]))


ALL = [
    pin_projection_is_nearest_row_scaled_sign_vector,
    pin_projection_idempotent_and_sign_of_zero,
    pin_ls_update_matches_augmented_lstsq,
    pin_penalty_scale,
    pin_orthonormalize,
    pin_init_spans_and_balances,
    pin_rank_one_exact,
    pin_planted_low_rank_binary_recovered,
    pin_beats_projected_truncated_svd,
    pin_negation_symmetry,
    pin_balance_keeps_product,
    pin_one_step_by_hand,
]
