"""Seeded synthetic inputs for the batched block-Shampoo step.

This module holds no arithmetic of the method itself: it only draws the
inputs (gradients, parameters, SPD test stacks, power-iteration start
vectors) with the shapes and value distributions of the workloads that the
DASH explainer's "The test and why" section describes (a ~1B Llama-style
model; its C4 gradients are not available, so seeded synthetic gradients of
the same layer shapes stand in for them).  Both the CUDA path's tests and
the float64 oracle consume these arrays.

All generators are deterministic functions of ``seed``.
"""

import numpy as np


# ---------------------------------------------------------------------------
# parameter-set shapes
# ---------------------------------------------------------------------------

def gpt2_124m_shapes(with_embeddings=True):
    """GPT-2 small: 12 layers x {QKV 768x2304, attn-out 768x768,
    MLP 768x3072, 3072x768}, plus wte 50257x768 and wpe 1024x768."""
    shapes = []
    for _ in range(12):
        shapes += [(768, 2304), (768, 768), (768, 3072), (3072, 768)]
    if with_embeddings:
        shapes += [(50257, 768), (1024, 768)]
    return shapes


def llama_1b_shapes(with_embeddings=True):
    """~1B Llama-style: 24 layers x {Q, K, V, O 2048x2048; SwiGLU gate/up
    2048x5632, down 5632x2048}, plus embedding and head 32000x2048."""
    shapes = []
    for _ in range(24):
        shapes += [(2048, 2048)] * 4 + [(2048, 5632), (2048, 5632), (5632, 2048)]
    if with_embeddings:
        shapes += [(32000, 2048), (32000, 2048)]
    return shapes


def mixed_shapes():
    """Block-size sweep set: 1024x4096, 4096x1024, 2048x2048."""
    return [(1024, 4096), (4096, 1024), (2048, 2048)]


# ---------------------------------------------------------------------------
# gradients
# ---------------------------------------------------------------------------

def spiked_gradient(rows=512, cols=512, rank=8, scale=10.0, seed=0):
    """G = Z + S with Z ~ N(0,1) and a rank-``rank`` spike
    S = scale * A B^T / sqrt(rank), A, B ~ N(0,1): spike entries have RMS
    ``scale`` relative to the unit-variance noise.  float32."""
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((rows, cols))
    A = rng.standard_normal((rows, rank))
    Bm = rng.standard_normal((cols, rank))
    return (Z + scale * (A @ Bm.T) / np.sqrt(rank)).astype(np.float32)


def gaussian_gradients(shapes, std=0.1, seed=0, row_lognormal_sigma=None):
    """Per-parameter float32 gradients N(0, std^2); optionally every row is
    multiplied by s_r ~ LogNormal(0, row_lognormal_sigma)."""
    rng = np.random.default_rng(seed)
    out = []
    for (r, c) in shapes:
        g = rng.standard_normal((r, c), dtype=np.float32) * np.float32(std)
        if row_lognormal_sigma is not None:
            s = rng.lognormal(0.0, row_lognormal_sigma, size=(r, 1)).astype(np.float32)
            g *= s
        out.append(g)
    return out


def student_t_gradients(shapes, nu=3.0, seed=0):
    """Heavy-tailed float32 gradients, Student-t with ``nu`` degrees of freedom."""
    rng = np.random.default_rng(seed)
    return [rng.standard_t(nu, size=s).astype(np.float32) for s in shapes]


def parameters(shapes, std=0.02, seed=1):
    """Float32 parameters N(0, std^2) (their values do not enter the update)."""
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(s, dtype=np.float32) * np.float32(std) for s in shapes]


def torch_gaussian_gradients(shapes, device, std=0.1, seed=0, row_lognormal_sigma=None):
    """Device-side variant of :func:`gaussian_gradients` for large parameter
    sets (drawn with torch's generator on ``device``; not bit-identical to the
    numpy variant)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for (r, c) in shapes:
        x = torch.randn((r, c), generator=g, device=device, dtype=torch.float32) * std
        if row_lognormal_sigma is not None:
            s = torch.randn((r, 1), generator=g, device=device, dtype=torch.float32)
            x *= torch.exp(s * row_lognormal_sigma)
        out.append(x)
    return out


def torch_student_t_gradients(shapes, device, nu=3.0, seed=0):
    """Device-side Student-t(nu) gradients: z / sqrt(chi2_nu / nu)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for (r, c) in shapes:
        z = torch.randn((r, c), generator=g, device=device, dtype=torch.float32)
        chi = torch.zeros((r, c), device=device, dtype=torch.float32)
        for _ in range(int(nu)):
            e = torch.randn((r, c), generator=g, device=device, dtype=torch.float32)
            chi += e * e
        out.append(z / torch.sqrt(chi / nu))
    return out


# ---------------------------------------------------------------------------
# standalone SPD stacks
# ---------------------------------------------------------------------------

def haar_orthogonal(n, rng):
    """Haar-distributed n x n orthogonal matrix: QR of a Gaussian matrix with
    the signs of R's diagonal folded into Q."""
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def decaying_spectrum(b=256, n_cols=1024, floor=1e-6):
    """Eigenvalues of G G^T / n_cols + floor*I when G's singular values are
    1/k, k = 1..b: 1/(n_cols k^2) + floor (descending)."""
    k = np.arange(1, b + 1, dtype=np.float64)
    return 1.0 / (n_cols * k * k) + floor


def spd_stack_decaying(n=256, b=256, n_cols=1024, floor=1e-6, seed=0):
    """Stack of n SPD matrices A_i = G_i G_i^T / n_cols + floor*I with
    G_i = U_i diag(1/k) V_i^T (U_i Haar b x b, V_i with orthonormal columns).
    Since V_i^T V_i = I the product equals U_i diag(1/k^2) U_i^T, which is how
    it is formed.  Returns (A float32 (n,b,b), U float64 (n,b,b), spectrum)."""
    rng = np.random.default_rng(seed)
    lam = decaying_spectrum(b, n_cols, floor)
    A = np.empty((n, b, b), dtype=np.float32)
    Us = np.empty((n, b, b), dtype=np.float64)
    for i in range(n):
        U = haar_orthogonal(b, rng)
        M = (U * lam) @ U.T
        A[i] = (0.5 * (M + M.T)).astype(np.float32)
        Us[i] = U
    return A, Us, lam


def spd_stack_geometric(n, b, kappa, seed=0, lam_max=1.0):
    """Stack of n SPD matrices with eigenvalues geometrically spaced from
    lam_max down to lam_max/kappa and Haar eigenvectors.  float32."""
    rng = np.random.default_rng(seed)
    lam = lam_max * np.geomspace(1.0, 1.0 / kappa, b)
    A = np.empty((n, b, b), dtype=np.float32)
    for i in range(n):
        U = haar_orthogonal(b, rng)
        M = (U * lam) @ U.T
        A[i] = (0.5 * (M + M.T)).astype(np.float32)
    return A


def pi_start_vectors(B, K=32, seed=0):
    """Power-iteration start block V0 (B x K), N(0,1) float32, column-major in
    meaning (column j is start vector j); stored row-major (B, K)."""
    rng = np.random.default_rng(seed + 7919)
    return rng.standard_normal((B, K)).astype(np.float32)
