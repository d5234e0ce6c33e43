"""Pins for the oracle's factor refresh (CPU only).

Checked against: the published SplitMix64 output stream, LAPACK (numpy
eigh / qr) as library cross-checks, closed-form spectra, exact low-rank
factors, and convergence of subspace iteration to the exact eigenpairs.
"""
import numpy as np
import pytest

from oracle import gift_oracle as O


def test_splitmix64_published_stream():
    # SplitMix64 seeded with 1234567: first five outputs of the reference generator
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    x = 1234567
    got = []
    for _ in range(5):
        got.append(O.splitmix64(x))
        x = (x + 0x9E3779B97F4A7C15) & ((1 << 64) - 1)
    assert got == want


def test_rademacher_start_is_balanced_and_seeded():
    a = O.rademacher_start(256, 48, 42)
    b = O.rademacher_start(256, 48, 42)
    c = O.rademacher_start(256, 48, 43)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert set(np.unique(a)) == {-1.0, 1.0}
    assert abs(a.mean()) < 0.05


def test_householder_q_vs_lapack():
    rng = np.random.default_rng(0)
    Y = rng.standard_normal((300, 40)) @ np.diag(np.logspace(0, -6, 40))
    Q = O.householder_q(Y)
    assert np.allclose(Q.T @ Q, np.eye(40), atol=1e-13)
    R = Q.T @ Y
    assert np.allclose(np.tril(R, -1), 0, atol=1e-12 * np.abs(R).max())
    Ql, _ = np.linalg.qr(Y)
    # same columns up to sign
    s = np.sign(np.sum(Q * Ql, axis=0))
    assert np.allclose(Q, Ql * s, atol=1e-9)


@pytest.mark.parametrize("n", [5, 17, 48])
def test_jacobi_vs_lapack_eigh(n):
    rng = np.random.default_rng(n)
    B = rng.standard_normal((n, n))
    B = B + B.T
    w, V = O.jacobi_eigh(B)
    wl, Vl = np.linalg.eigh(B)
    assert np.allclose(w, wl[::-1], rtol=1e-12, atol=1e-12 * np.abs(wl).max())
    assert np.allclose(V.T @ V, np.eye(n), atol=1e-12)
    assert np.allclose(B @ V, V * w[None, :], atol=1e-11 * np.abs(wl).max())


def test_input_factor_closed_form():
    # X = rows sqrt(N s_i) e_i  =>  X^T X / N = diag(s) exactly
    d = 64
    s = 4.0 ** -np.arange(d, dtype=np.float64)   # even powers: sqrt(N s) exact
    N = d
    X = np.diag(np.sqrt(N * s))
    A = O.input_factor(X)
    assert np.array_equal(A, np.diag(s))


def test_refresh_diagonal_closed_form():
    # A = diag(s) with a strictly decreasing power law: the top-32 Ritz values
    # converge to s[:32]; rho to mean(s[32:]) once converged.
    d = 256
    s = np.arange(1, d + 1, dtype=np.float64) ** -2.0
    s[:5] *= 100.0
    A = np.diag(s)
    U, lam, rho, flags = O.factor_refresh(A, 32, 16, iters=60, seed=1)
    assert flags == 0
    assert np.allclose(lam, s[:32], rtol=1e-10)
    assert np.isclose(rho, s[32:].mean(), rtol=1e-10)
    # U spans the first 32 coordinate axes
    P = U @ U.T
    assert np.allclose(P, np.diag(np.r_[np.ones(32), np.zeros(d - 32)]), atol=1e-8)


def test_refresh_exact_low_rank_one_iteration():
    # rank(A) = 20 <= 32: range(A Q) = range(A) after one product, so one
    # iteration reproduces the exact nonzero eigenpairs.
    rng = np.random.default_rng(4)
    d, k = 200, 20
    B = np.linalg.qr(rng.standard_normal((d, k)))[0]
    ev = np.linspace(5.0, 1.0, k)
    A = B @ np.diag(ev) @ B.T
    U, lam, rho, flags = O.factor_refresh(A, 32, 16, iters=1, seed=9)
    wl = np.linalg.eigh(A)[0][::-1]
    assert np.allclose(lam[:k], wl[:k], rtol=1e-10)
    assert np.allclose(lam[k:], 0, atol=1e-10)
    # trace identity: rho = (tr A - sum lam)/(d - 32) ~ 0 -> floored
    assert flags == 1 and rho == pytest.approx(2.0 ** -24 * lam[0])


def test_refresh_converges_to_eigh_and_rho_matches_tail_mean():
    rng = np.random.default_rng(8)
    d = 192
    Q = np.linalg.qr(rng.standard_normal((d, d)))[0]
    ev = np.arange(1, d + 1, dtype=np.float64) ** -1.2
    ev[:5] *= 100
    A = Q @ np.diag(ev) @ Q.T
    errs = []
    for it in (1, 4, 40):
        U, lam, rho, _ = O.factor_refresh(A, 32, 16, iters=it, seed=3)
        errs.append(np.max(np.abs(lam - ev[:32]) / ev[:32]))
    assert errs[2] < 1e-9
    assert errs[0] > errs[1] > errs[2]
    U, lam, rho, _ = O.factor_refresh(A, 32, 16, iters=40, seed=3)
    assert rho == pytest.approx(ev[32:].mean(), rel=1e-9)
    # Rayleigh-Ritz: U orthonormal and U^T A U = diag(lam) at any iteration count
    U4, lam4, _, _ = O.factor_refresh(A, 32, 16, iters=4, seed=3)
    assert np.allclose(U4.T @ U4, np.eye(32), atol=1e-12)
    assert np.allclose(U4.T @ A @ U4, np.diag(lam4), atol=1e-12 * lam4[0])


def test_refresh_full_rank_gives_exact_inverse_sqrt():
    rng = np.random.default_rng(2)
    d, N = 24, 400
    X = rng.standard_normal((N, d)) @ np.diag(np.linspace(3, 0.2, d))
    A = O.input_factor(X)
    U, lam, rho, _ = O.factor_refresh(A, d)
    assert rho == 0.0
    M = O.transform_matrix(U, lam, rho)
    Xw = X @ M
    assert np.allclose(Xw.T @ Xw / N, np.eye(d), atol=1e-10)
