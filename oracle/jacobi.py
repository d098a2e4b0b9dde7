"""Cyclic Jacobi eigensolver, written out by hand (no LAPACK).

Test infrastructure only.  Used to pin the oracle's eigendecomposition-based
inverse roots on tiny matrices by brute force, independently of numpy.linalg.
The method is the classical cyclic-by-row Jacobi rotation scheme (Golub & Van
Loan, "Matrix Computations", section 8.5): sweep over all (p, q) pairs, zero
A[p, q] with a plane rotation, repeat until the off-diagonal mass vanishes.
"""

import math


def jacobi_eigh(A, tol=1e-15, max_sweeps=100):
    """Return (eigenvalues, eigenvectors) of a small symmetric matrix.

    ``A`` is a list of lists or a 2-D array-like; the result is a pair of
    plain Python lists: w[i] and V[row][i] (column i is the eigenvector of
    w[i]), sorted by ascending eigenvalue.
    """
    n = len(A)
    a = [[float(A[i][j]) for j in range(n)] for i in range(n)]
    v = [[1.0 if i == j else 0.0 for j in range(n)] for i in range(n)]
    scale = math.sqrt(sum(a[i][j] ** 2 for i in range(n) for j in range(n))) or 1.0
    for _ in range(max_sweeps):
        off = math.sqrt(sum(a[i][j] ** 2 for i in range(n) for j in range(n) if i != j))
        if off <= tol * scale:
            break
        for p in range(n - 1):
            for q in range(p + 1, n):
                apq = a[p][q]
                if apq == 0.0:
                    continue
                theta = (a[q][q] - a[p][p]) / (2.0 * apq)
                t = (1.0 if theta >= 0 else -1.0) / (abs(theta) + math.sqrt(theta * theta + 1.0))
                c = 1.0 / math.sqrt(t * t + 1.0)
                s = t * c
                for k in range(n):  # A <- A J  (columns p, q)
                    akp, akq = a[k][p], a[k][q]
                    a[k][p] = c * akp - s * akq
                    a[k][q] = s * akp + c * akq
                for k in range(n):  # A <- J^T A  (rows p, q)
                    apk, aqk = a[p][k], a[q][k]
                    a[p][k] = c * apk - s * aqk
                    a[q][k] = s * apk + c * aqk
                for k in range(n):  # V <- V J
                    vkp, vkq = v[k][p], v[k][q]
                    v[k][p] = c * vkp - s * vkq
                    v[k][q] = s * vkp + c * vkq
    w = [a[i][i] for i in range(n)]
    order = sorted(range(n), key=lambda i: w[i])
    return [w[i] for i in order], [[v[r][i] for i in order] for r in range(n)]


def inv_root_jacobi(A, p=4):
    """A^(-1/p) of a small SPD matrix from the Jacobi eigenpairs (lists)."""
    w, V = jacobi_eigh(A)
    n = len(w)
    if min(w) <= 0:
        raise ValueError("matrix is not positive definite")
    f = [x ** (-1.0 / p) for x in w]
    return [[sum(V[i][k] * f[k] * V[j][k] for k in range(n)) for j in range(n)]
            for i in range(n)]
