"""Inverse fourth roots, power iteration and the Chebyshev fit, in float64.

Test infrastructure only (see the package docstring).  Three "levels":

* level 1 -- the exact principal inverse root V diag(lambda^(-1/p)) V^T from a
  symmetric eigendecomposition (the accuracy reference the DASH explainer calls
  EVD, "Step-by-step", solver option (c)).
* level 2 -- the truncated method as specified.  Newton-DB and the Clenshaw
  polynomial are polynomials in the input matrix, so their exact result is
  V diag(phi(lambda)) V^T where phi is the same recurrence run on scalars.
* level 3 -- the same recurrences written out step by step with float64
  matrix products, in the page's order and notation.
"""

import numpy as np


# --------------------------------------------------------------------------
# level 1
# --------------------------------------------------------------------------

def inv_root_eigh(A, p=4):
    """Exact A^(-1/p) of a symmetric positive definite A via eigh.

    DASH explainer, "Step-by-step", solver (c) EVD: decompose A = Q Lambda Q^T,
    take Lambda^(-1/p), reassemble.
    """
    A = np.asarray(A, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (A + A.T))
    if w[0] <= 0:
        raise ValueError("matrix is not positive definite")
    return (Q * w ** (-1.0 / p)) @ Q.T


# --------------------------------------------------------------------------
# power iteration (multi-start)
# --------------------------------------------------------------------------

def power_iteration(A, V0, iters):
    """Largest-eigenvalue estimate by multi-start power iteration.

    DASH explainer, "Building blocks" (Multi-Power-Iteration) and
    "Step-by-step" (scale each block): start from K random vectors, multiply by
    A repeatedly, keep the largest Rayleigh quotient.

    Reading of the unspecified details: ``iters`` products W = A V are taken;
    after every product but the last the columns are normalised to unit
    length; the estimate is max_j (v_j . A v_j) / (v_j . v_j) taken with the
    vectors that entered the last product.  A column whose norm is zero is
    left at zero and contributes a quotient of 0.

    Returns (lambda_est, rayleigh_quotients).
    """
    A = np.asarray(A, dtype=np.float64)
    V = np.array(V0, dtype=np.float64, copy=True)
    if iters < 1:
        raise ValueError("iters must be >= 1")
    for t in range(iters):
        W = A @ V
        if t == iters - 1:
            num = np.sum(V * W, axis=0)
            den = np.sum(V * V, axis=0)
            rq = np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)
            return float(np.max(rq)), rq
        nrm = np.linalg.norm(W, axis=0)
        V = np.where(nrm > 0, W / np.where(nrm > 0, nrm, 1.0), 0.0)
    raise AssertionError("unreachable")


# --------------------------------------------------------------------------
# Newton-DB (Denman-Beavers in coupled Newton-Schulz form)
# --------------------------------------------------------------------------

def ndb_scalar(x, iters):
    """The Newton-DB recurrence on scalars (element-wise on arrays).

    DASH explainer, "Building blocks" (Newton-DB): Y0 = x, Z0 = 1;
    E = (3 - Z Y)/2; Y <- Y E; Z <- E Z (both from the old values).
    Returns (y, z) after ``iters`` iterations; y -> sqrt(x), z -> 1/sqrt(x)
    for 0 < x < 3.
    """
    y = np.array(x, dtype=np.float64, copy=True)
    z = np.ones_like(y)
    for _ in range(iters):
        e = 0.5 * (3.0 - z * y)
        y, z = y * e, e * z
    return y, z


def ndb_scale(lam_est):
    """Spectral scaling c = 1/(2 lambda_est), used by both solvers.

    DASH explainer, "Building blocks" (spectral scaling) and "Step-by-step"
    (scale each block, before the solver is chosen): divide the block by
    about 2*lambda_est.  Read literally as the factor 2.
    """
    return 1.0 / (2.0 * float(lam_est))


def ndb_phi(w, lam_est, iters1, iters2):
    """Scalar map of the chained Newton-DB inverse fourth root.

    Stage 1 runs on c*w; stage 2 runs again on the stage-1 Y ("chain twice",
    "run again on Y"); the result is c^(1/4) * z2, which tends to w^(-1/4).
    """
    c = ndb_scale(lam_est)
    y1, _ = ndb_scalar(c * np.asarray(w, dtype=np.float64), iters1)
    _, z2 = ndb_scalar(y1, iters2)
    return c ** 0.25 * z2


def ndb_inv4root_spectral(A, lam_est, iters1, iters2):
    """Level 2: the truncated chained Newton-DB result, evaluated exactly."""
    A = np.asarray(A, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (A + A.T))
    return (Q * ndb_phi(w, lam_est, iters1, iters2)) @ Q.T


def ndb_matrix(Y0, iters):
    """Newton-DB with matrices, step by step (level 3), from Z0 = I."""
    Y = np.array(Y0, dtype=np.float64, copy=True)
    n = Y.shape[0]
    I = np.eye(n)
    Z = I.copy()
    for _ in range(iters):
        E = 0.5 * (3.0 * I - Z @ Y)
        Y, Z = Y @ E, E @ Z
    return Y, Z


def ndb_inv4root_matmul(A, lam_est, iters1, iters2):
    """Level 3: chained Newton-DB inverse fourth root with matrix products.

    Y0 = c A, Z0 = I, ``iters1`` iterations; then again on Y with Z reset to
    I, ``iters2`` iterations; X = c^(1/4) Z.
    """
    c = ndb_scale(lam_est)
    Y1, _ = ndb_matrix(c * np.asarray(A, dtype=np.float64), iters1)
    _, Z2 = ndb_matrix(Y1, iters2)
    return c ** 0.25 * Z2


# --------------------------------------------------------------------------
# Coupled Newton
# --------------------------------------------------------------------------

def cn_scalar(m0, iters, p=4):
    """The coupled-Newton recurrence on scalars (element-wise on arrays).

    DASH explainer, "Building blocks" (Coupled-Newton): X_k ~ A^(-1/p) with a
    stabiliser M_k; C_k is computed from M_k, X_{k+1} = X_k C_k and
    M_{k+1} = C_k^p M_k.  Reading for the unstated C_k: the Newton step
    C_k = ((p+1) - M_k)/p.  From x0 = 1, m0 = c*w: x -> m0^(-1/p) for
    0 < m0 < p+1, and m = x^p * m0 at every step.  Returns (x, m).
    """
    m = np.array(m0, dtype=np.float64, copy=True)
    x = np.ones_like(m)
    for _ in range(iters):
        c = ((p + 1.0) - m) / p
        x, m = x * c, c ** p * m
    return x, m


def cn_phi(w, lam_est, iters):
    """Scalar map of the coupled-Newton inverse fourth root: the common
    scaling c = 1/(2 lambda_est), M0 = c w, X0 = 1, result c^(1/4) x."""
    c = ndb_scale(lam_est)
    x, _ = cn_scalar(c * np.asarray(w, dtype=np.float64), iters)
    return c ** 0.25 * x


def cn_inv4root_spectral(A, lam_est, iters):
    """Level 2: the truncated coupled-Newton result, evaluated exactly."""
    A = np.asarray(A, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (A + A.T))
    return (Q * cn_phi(w, lam_est, iters)) @ Q.T


def cn_matrix(M0, iters, p=4):
    """Coupled Newton with matrices, step by step (level 3), from X0 = I:
    C = ((p+1) I - M)/p; X <- X C; M <- C^p M."""
    M = np.array(M0, dtype=np.float64, copy=True)
    I = np.eye(M.shape[0])
    X = I.copy()
    for _ in range(iters):
        C = ((p + 1.0) * I - M) / p
        X, M = X @ C, np.linalg.matrix_power(C, p) @ M
    return X, M


def cn_inv4root_matmul(A, lam_est, iters):
    """Level 3: coupled-Newton inverse fourth root with matrix products,
    M0 = c A, X0 = I, X = c^(1/4) X_T."""
    c = ndb_scale(lam_est)
    X, _ = cn_matrix(c * np.asarray(A, dtype=np.float64), iters)
    return c ** 0.25 * X


# --------------------------------------------------------------------------
# Chebyshev / Clenshaw
# --------------------------------------------------------------------------

def cheb_fit(f, degree, lo, hi):
    """Chebyshev interpolant of f on [lo, hi] at the first-kind nodes.

    DASH explainer, "Building blocks" (Chebyshev): coefficients are pre-fit on
    an interval.  Reading: interpolation at the degree+1 Chebyshev points of
    the first kind, in float64.  Convention f ~ c0/2 + sum_{k>=1} c_k T_k(t)
    with t = (2x - lo - hi)/(hi - lo).
    """
    n = degree + 1
    j = np.arange(n)
    theta = np.pi * (j + 0.5) / n
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(theta)
    fx = f(x)
    k = np.arange(n)
    c = (2.0 / n) * (np.cos(np.outer(k, theta)) @ fx)
    return c


def cheb_inv4root_coeffs(degree, delta):
    """Coefficients of x^(-1/4) on [delta, 1 + delta]."""
    return cheb_fit(lambda x: x ** -0.25, degree, delta, 1.0 + delta)


def clenshaw_scalar(c, t):
    """Clenshaw evaluation of c0/2 + sum c_k T_k(t) (element-wise)."""
    t = np.asarray(t, dtype=np.float64)
    b1 = np.zeros_like(t)
    b2 = np.zeros_like(t)
    for k in range(len(c) - 1, 0, -1):
        b1, b2 = c[k] + 2.0 * t * b1 - b2, b1
    return 0.5 * c[0] + t * b1 - b2


def cheb_phi(w, lam_est, degree, delta):
    """Scalar map of the Chebyshev inverse fourth root.

    DASH explainer, "Step-by-step": each block is first scaled by
    c = 1/(2 lambda_est) (step "Scale each block using multi-Power-Iteration",
    which precedes the choice of solver), then solver (d) maps the spectrum
    into [delta, 1 + delta]: x = c w + delta.  The polynomial p ~ x^(-1/4) is
    evaluated at the Chebyshev variable t = 2(x - delta) - 1 = 2 c w - 1, and
    the scaling is undone: the result c^(1/4) p approximates
    (w + delta / c)^(-1/4).
    """
    c = ndb_scale(lam_est)
    cf = cheb_inv4root_coeffs(degree, delta)
    t = 2.0 * c * np.asarray(w, dtype=np.float64) - 1.0
    return c ** 0.25 * clenshaw_scalar(cf, t)


def cheb_inv4root_spectral(A, lam_est, degree, delta):
    """Level 2: the Chebyshev/Clenshaw result, evaluated exactly."""
    A = np.asarray(A, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (A + A.T))
    return (Q * cheb_phi(w, lam_est, degree, delta)) @ Q.T


def cheb_inv4root_matmul(A, lam_est, degree, delta):
    """Level 3: the matrix Clenshaw recurrence with float64 products.

    c = 1/(2 lambda_est); T = 2 c A - I; b_k = c_k I + 2 T b_{k+1} - b_{k+2}
    for k = d..1; p = c0/2 I + T b1 - b2; X = c^(1/4) p.
    """
    A = np.asarray(A, dtype=np.float64)
    n = A.shape[0]
    I = np.eye(n)
    s = ndb_scale(lam_est)
    c = cheb_inv4root_coeffs(degree, delta)
    T = 2.0 * s * A - I
    b1 = np.zeros((n, n))
    b2 = np.zeros((n, n))
    for k in range(degree, 0, -1):
        b1, b2 = c[k] * I + 2.0 * T @ b1 - b2, b1
    P = 0.5 * c[0] * I + T @ b1 - b2
    return s ** 0.25 * P
