"""Pins of the oracle's inverse roots, power iteration and Chebyshev fit.

Every check compares the oracle with something other than itself: a closed
form, an invariant of the recurrence, a numpy.polynomial routine, or a
hand-written Jacobi eigensolver.
"""

import numpy as np
import pytest
from numpy.polynomial import chebyshev as npcheb

from oracle import roots, jacobi
from matrix_inverse_roots_stack_b200 import workloads


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(b)


def random_spd(b, kappa, seed):
    rng = np.random.default_rng(seed)
    U = workloads.haar_orthogonal(b, rng)
    w = np.geomspace(1.0, 1.0 / kappa, b)
    return (U * w) @ U.T, U, w


# ---------------------------------------------------------------- level 1

def test_identity_closed_form_all_levels():
    alpha, b = 3.7, 8
    A = alpha * np.eye(b)
    expect = alpha ** -0.25 * np.eye(b)
    assert rel(roots.inv_root_eigh(A), expect) < 1e-14
    V0 = workloads.pi_start_vectors(b, 32, seed=3)[:b]
    lam, _ = roots.power_iteration(A, V0, 10)
    assert abs(lam - alpha) < 1e-13 * alpha
    # c*lambda = 1/2 exactly: both Newton-DB stages converge to double precision
    assert rel(roots.ndb_inv4root_spectral(A, lam, 14, 14), expect) < 1e-13
    assert rel(roots.ndb_inv4root_matmul(A, lam, 14, 14), expect) < 1e-13


def test_diagonal_closed_form():
    lam = np.array([1.0, 0.3, 0.05, 1e-3, 2e-4, 7.5])
    A = np.diag(lam)
    assert rel(roots.inv_root_eigh(A), np.diag(lam ** -0.25)) < 1e-14
    # converged truncated method reaches the same closed form
    X = roots.ndb_inv4root_matmul(A, lam.max(), 40, 40)
    assert rel(X, np.diag(lam ** -0.25)) < 1e-12


def sqrt2x2(A):
    # sqrt(A) = (A + s I)/t, s = sqrt(det A), t = sqrt(tr A + 2 s)
    s = np.sqrt(np.linalg.det(A))
    t = np.sqrt(np.trace(A) + 2.0 * s)
    return (A + s * np.eye(2)) / t


def inv2x2(A):
    a, b, c, d = A[0, 0], A[0, 1], A[1, 0], A[1, 1]
    return np.array([[d, -b], [-c, a]]) / (a * d - b * c)


def test_2x2_closed_form():
    rng = np.random.default_rng(11)
    for _ in range(20):
        M = rng.standard_normal((2, 2))
        A = M @ M.T + 0.05 * np.eye(2)
        expect = inv2x2(sqrt2x2(sqrt2x2(A)))
        assert rel(roots.inv_root_eigh(A), expect) < 1e-12


def test_4x4_hadamard_block_closed_form():
    H = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], float)
    Q = 0.5 * H  # orthogonal and symmetric
    rng = np.random.default_rng(5)
    for _ in range(10):
        M1, M2 = rng.standard_normal((2, 2)), rng.standard_normal((2, 2))
        A1, A2 = M1 @ M1.T + 0.1 * np.eye(2), M2 @ M2.T + 0.1 * np.eye(2)
        D = np.zeros((4, 4))
        D[:2, :2], D[2:, 2:] = A1, A2
        A = Q @ D @ Q.T
        R = np.zeros((4, 4))
        R[:2, :2] = inv2x2(sqrt2x2(sqrt2x2(A1)))
        R[2:, 2:] = inv2x2(sqrt2x2(sqrt2x2(A2)))
        assert rel(roots.inv_root_eigh(A), Q @ R @ Q.T) < 1e-12


def test_jacobi_brute_force_4x4():
    rng = np.random.default_rng(2)
    for _ in range(10):
        M = rng.standard_normal((4, 4))
        A = M @ M.T + 0.01 * np.eye(4)
        w, V = jacobi.jacobi_eigh(A.tolist())
        wl = np.linalg.eigvalsh(A)
        assert np.max(np.abs(np.array(w) - wl)) < 1e-13 * wl.max()
        V = np.array(V)
        assert np.linalg.norm(V.T @ V - np.eye(4)) < 1e-13
        assert rel(np.array(jacobi.inv_root_jacobi(A.tolist())), roots.inv_root_eigh(A)) < 1e-12


def test_level1_invariants():
    A, _, _ = random_spd(32, 1e4, seed=1)
    X = roots.inv_root_eigh(A)
    X4 = X @ X @ X @ X
    assert np.linalg.norm(X4 @ A - np.eye(32)) / np.sqrt(32) < 1e-9
    assert np.linalg.norm(X - X.T) < 1e-12 * np.linalg.norm(X)
    assert np.linalg.norm(X @ A - A @ X) < 1e-12 * np.linalg.norm(X) * np.linalg.norm(A)


def test_level1_known_eigenvectors():
    # config-2 construction: A = U diag(lam) U^T with lam known in closed form
    A, U, lam = workloads.spd_stack_decaying(n=2, b=64, n_cols=1024, floor=1e-6, seed=4)
    for i in range(2):
        M = (U[i] * lam) @ U[i].T
        assert rel(roots.inv_root_eigh(M), (U[i] * lam ** -0.25) @ U[i].T) < 1e-10
        # the stored float32 matrix is that matrix rounded
        assert np.max(np.abs(A[i] - M)) < 1e-7 * lam.max()


# ---------------------------------------------------------------- Newton-DB

def ns_product_map(p, iters):
    # the product p = y z obeys p <- p (3 - p)^2 / 4, and y / z stays equal to x
    for _ in range(iters):
        p = p * (3.0 - p) ** 2 / 4.0
    return p


@pytest.mark.parametrize("iters", [0, 1, 3, 8, 14])
def test_ndb_scalar_invariants(iters):
    x = np.geomspace(1e-7, 1.5, 40)
    y, z = roots.ndb_scalar(x, iters)
    p = ns_product_map(x.copy(), iters)
    assert np.allclose(y, np.sqrt(x * p), rtol=1e-12, atol=0)
    assert np.allclose(z, np.sqrt(p / x), rtol=1e-12, atol=0)


def test_ndb_matrix_diagonal_matches_invariant_form():
    x = np.array([0.5, 0.1, 1e-3, 0.9, 0.25])
    for T in (1, 5, 9):
        Y, Z = roots.ndb_matrix(np.diag(x), T)
        p = ns_product_map(x.copy(), T)
        assert rel(np.diag(Y), np.sqrt(x * p)) < 1e-13
        assert rel(np.diag(Z), np.sqrt(p / x)) < 1e-13
        assert np.linalg.norm(Y - np.diag(np.diag(Y))) == 0.0


@pytest.mark.parametrize("T1,T2", [(8, 8), (14, 14), (3, 10)])
def test_ndb_level2_matches_level3(T1, T2):
    A, _, w = random_spd(48, 1e3, seed=7)
    lam = w.max() * 0.999
    assert rel(roots.ndb_inv4root_spectral(A, lam, T1, T2),
               roots.ndb_inv4root_matmul(A, lam, T1, T2)) < 1e-10


def test_ndb_converges_to_exact():
    A, _, w = random_spd(48, 1e3, seed=8)
    assert rel(roots.ndb_inv4root_spectral(A, w.max(), 30, 30), roots.inv_root_eigh(A)) < 1e-10


def test_ndb_config2_convergence_profile():
    # on the decaying spectrum (kappa ~ 963) 14 iterations per stage converge
    lam = workloads.decaying_spectrum(256, 1024, 1e-6)
    phi = roots.ndb_phi(lam, lam.max(), 14, 14)
    assert np.max(np.abs(phi / lam ** -0.25 - 1.0)) < 1e-12
    phi8 = roots.ndb_phi(lam, lam.max(), 8, 8)
    assert np.max(np.abs(phi8 / lam ** -0.25 - 1.0)) > 1e-2


# ---------------------------------------------------------------- coupled Newton


@pytest.mark.parametrize("iters", [0, 1, 4, 12])
def test_cn_scalar_keeps_the_coupling_invariant(iters):
    # every coupled-Newton step keeps m = x^4 * m0 (C multiplies x once and
    # m four times), so a wrong power or a dropped factor breaks it
    m0 = np.geomspace(1e-6, 4.9, 60)
    x, m = roots.cn_scalar(m0, iters)
    assert np.allclose(m, x ** 4 * m0, rtol=1e-12, atol=0)


def test_cn_scalar_converges_to_inverse_fourth_root():
    m0 = np.geomspace(1e-6, 4.5, 60)
    x, m = roots.cn_scalar(m0, 60)
    assert np.max(np.abs(x / m0 ** -0.25 - 1.0)) < 1e-12
    assert np.max(np.abs(m - 1.0)) < 1e-12
    # outside (0, p + 1) = (0, 5) the iteration leaves the basin
    x, _ = roots.cn_scalar(np.array([5.5]), 30)
    assert not np.isfinite(x[0]) or abs(x[0] - 5.5 ** -0.25) > 1e-3


def test_cn_matrix_keeps_the_coupling_invariant():
    A, _, w = random_spd(24, 1e2, seed=11)
    M0 = A / (2.0 * w.max())
    for T in (1, 3, 6):
        X, M = roots.cn_matrix(M0, T)
        assert rel(M, np.linalg.matrix_power(X, 4) @ M0) < 1e-12


@pytest.mark.parametrize("delta", [1e-2, 1e-3, 1e-4])
def test_cn_newton_step_contracts_quadratically(delta):
    # Guo-Higham Newton step for p = 4 near the fixed point: with
    # m = 1 - delta, C = (5 - m)/4 = 1 + delta/4 and
    # 1 - C^4 m = (5/8) delta^2 + (5/16) delta^3 + O(delta^4): the constant is
    # (p + 1)/(2p).  Any other affine C_k (e.g. (3 - m)/2) loses the quadratic
    # term or changes its constant, and the coupling invariant cannot see it.
    x, m = roots.cn_scalar(np.array([1.0 - delta]), 1)
    assert abs(x[0] - (1.0 + delta / 4.0)) < 1e-15
    ratio = (1.0 - m[0]) / delta ** 2
    assert abs(ratio - 0.625) < 0.4 * delta, ratio


def test_cn_one_and_two_steps_closed_form():
    # T = 1 and T = 2 written out from the step's definition, on the
    # eigenvalues of M0 (not through cn_scalar): X1 = C0 = (5I - M0)/4,
    # M1 = C0^4 M0, X2 = C0 (5I - M1)/4.
    A, U, w = random_spd(20, 50.0, seed=14)
    lam = 1.05 * w.max()
    c = 1.0 / (2.0 * lam)
    m0 = c * w
    c0 = (5.0 - m0) / 4.0
    x1 = c0
    m1 = c0 ** 4 * m0
    x2 = c0 * (5.0 - m1) / 4.0
    for T, x in ((1, x1), (2, x2)):
        expect = (U * (c ** 0.25 * x)) @ U.T
        assert rel(roots.cn_inv4root_spectral(A, lam, T), expect) < 1e-13
        assert rel(roots.cn_inv4root_matmul(A, lam, T), expect) < 1e-12


def test_cn_level2_matches_level3():
    A, _, w = random_spd(48, 1e3, seed=12)
    lam = w.max() * 0.999
    for T in (3, 9, 16):
        assert rel(roots.cn_inv4root_spectral(A, lam, T), roots.cn_inv4root_matmul(A, lam, T)) < 1e-10


def test_cn_converges_to_exact():
    A, _, w = random_spd(48, 1e3, seed=13)
    assert rel(roots.cn_inv4root_spectral(A, w.max(), 30), roots.inv_root_eigh(A)) < 1e-10
    # identity: lambda_est = alpha exactly, M0 = 1/2 I, X -> alpha^(-1/4) I
    X = roots.cn_inv4root_matmul(3.0 * np.eye(5), 3.0, 25)
    assert rel(X, 3.0 ** -0.25 * np.eye(5)) < 1e-12


# ---------------------------------------------------------------- Chebyshev

@pytest.mark.parametrize("degree,delta", [(4, 0.1), (16, 1e-3), (16, 1e-6), (60, 1e-3)])
def test_cheb_coeffs_match_numpy_interpolant(degree, delta):
    c = roots.cheb_inv4root_coeffs(degree, delta)
    # numpy's interpolant on [-1, 1] of the mapped function, its c0 not halved
    f = lambda t: (delta + 0.5 * (t + 1.0)) ** -0.25
    ref = npcheb.chebinterpolate(f, degree)
    ours = c.copy()
    ours[0] *= 0.5
    assert np.max(np.abs(ours - ref)) < 1e-12 * np.max(np.abs(ref))


def test_cheb_interpolates_at_nodes():
    d, delta = 16, 1e-3
    c = roots.cheb_inv4root_coeffs(d, delta)
    j = np.arange(d + 1)
    t = np.cos(np.pi * (j + 0.5) / (d + 1))
    x = delta + 0.5 * (t + 1.0)
    assert np.max(np.abs(roots.clenshaw_scalar(c, t) / x ** -0.25 - 1.0)) < 1e-13


def test_clenshaw_matches_chebval():
    rng = np.random.default_rng(0)
    c = rng.standard_normal(13)
    t = np.linspace(-1, 1, 101)
    cc = c.copy()
    cc[0] *= 0.5
    assert np.max(np.abs(roots.clenshaw_scalar(c, t) - npcheb.chebval(t, cc))) < 1e-13


def test_cheb_matrix_diagonal_matches_chebval():
    w = np.array([1.0, 0.4, 0.01, 1e-4, 0.77])
    lam, d, delta = 1.0, 16, 1e-3
    X = roots.cheb_inv4root_matmul(np.diag(w), lam, d, delta)
    c = roots.cheb_inv4root_coeffs(d, delta)
    cc = c.copy()
    cc[0] *= 0.5
    # spectral scaling 1/(2 lam): t = w/lam - 1, undone by (2 lam)^(-1/4)
    expect = npcheb.chebval(w / lam - 1.0, cc) * (2.0 * lam) ** -0.25
    assert rel(np.diag(X), expect) < 1e-13


def test_cheb_level2_matches_level3():
    A, _, w = random_spd(40, 1e3, seed=9)
    lam = w.max()
    for d, delta in ((16, 1e-3), (24, 1e-6)):
        assert rel(roots.cheb_inv4root_spectral(A, lam, d, delta),
                   roots.cheb_inv4root_matmul(A, lam, d, delta)) < 1e-10


def test_cheb_high_degree_approaches_shifted_target():
    # p approximates x^(-1/4) on [delta, 1+delta]; with c = 1/(2 lam) the
    # matrix result c^(1/4) p(c A + delta I) ~ (A + 2 delta lam I)^(-1/4)
    A, _, w = random_spd(24, 50.0, seed=10)
    lam, delta = w.max(), 0.05
    X = roots.cheb_inv4root_spectral(A, lam, 40, delta)
    assert rel(X, roots.inv_root_eigh(A + 2.0 * delta * lam * np.eye(24))) < 1e-9


def test_cheb_spectrum_stays_inside_interval():
    # with the 1/(2 lam) scaling an estimate up to 2x below lam_max still maps
    # the spectrum into [delta, 1 + delta], i.e. t in [-1, 1]
    w = np.linspace(1e-3, 1.0, 50)
    for lam in (1.0, 0.9, 0.5):
        t = 2.0 * roots.ndb_scale(lam) * w - 1.0
        assert t.min() >= -1.0 and t.max() <= 1.0


# ---------------------------------------------------------------- power iteration

def test_power_iteration_diagonal_closed_form():
    a = np.array([2.0, 1.5, 0.3, 0.01, 1.9])
    V0 = workloads.pi_start_vectors(5, 8, seed=1).astype(np.float64)
    T = 6
    lam, rq = roots.power_iteration(np.diag(a), V0, T)
    # normalisations cancel in the quotient of the last product
    num = np.sum((a[:, None] ** (2 * T - 1)) * V0 ** 2, axis=0)
    den = np.sum((a[:, None] ** (2 * T - 2)) * V0 ** 2, axis=0)
    assert np.max(np.abs(rq - num / den)) < 1e-13
    assert lam == pytest.approx(np.max(num / den), rel=1e-14)


def test_power_iteration_bound_and_gap():
    rng = np.random.default_rng(3)
    V0 = workloads.pi_start_vectors(64, 32, seed=2).astype(np.float64)
    for s in range(5):
        A, _, w = random_spd(64, 1e5, seed=20 + s)
        lam, _ = roots.power_iteration(A, V0, 10)
        assert lam <= w.max() * (1 + 1e-12)
    U = workloads.haar_orthogonal(64, rng)
    w = np.concatenate([[1.0], np.linspace(0.5, 1e-3, 63)])
    lam, _ = roots.power_iteration((U * w) @ U.T, V0, 10)
    assert abs(lam - 1.0) < 1e-3
