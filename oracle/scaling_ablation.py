"""Frobenius versus spectral scaling: Newton-DB iterations to the exact root.

Test infrastructure (see the package docstring): a float64 computation on the
oracle alone, run by hand to produce the ablation table of the DASH explainer's
comparison of the two scale estimates ("Building blocks": power-iteration
scaling instead of the Frobenius norm, which overestimates the top eigenvalue
and so costs iterations; "Scoreboard": Newton-DB with Frobenius versus
power-iteration scaling).

For a factor A = F + eps I with eigenvalues w, the truncated Newton-DB result
at T iterations per stage is V diag(phi_T(w)) V^T (level 2), and the exact
root is V diag(w^(-1/4)) V^T (level 1), so their relative Frobenius distance
is ||phi_T(w) - w^(-1/4)|| / ||w^(-1/4)||: only the eigenvalues are needed.
For each factor and each scale estimate (the multi-start power iteration of
the step, or ||A||_F) this finds the smallest T (equal in both stages) whose
distance is at most the root tolerance 1e-3.

    python -m oracle.scaling_ablation [--quick]
"""

import argparse
import sys

import numpy as np

from . import roots, step

TOL = 1e-3
T_MAX = 120


def iterations_to_tolerance(w, lam, tol=TOL, t_max=T_MAX):
    """Smallest T (iterations per stage) with level-2 within tol of level 1,
    or None if T_MAX is not enough."""
    w = np.asarray(w, dtype=np.float64)
    exact = w ** -0.25
    norm = np.linalg.norm(exact)
    lo, hi = 1, t_max
    if np.linalg.norm(roots.ndb_phi(w, lam, hi, hi) - exact) > tol * norm:
        return None
    while lo < hi:  # the distance falls monotonically with T once the spectrum is inside (0, 2)
        mid = (lo + hi) // 2
        if np.linalg.norm(roots.ndb_phi(w, lam, mid, mid) - exact) <= tol * norm:
            hi = mid
        else:
            lo = mid + 1
    return lo


def factor_spectra(shapes, grads, B, hp, V0):
    """Eigenvalues, power-iteration estimate and Frobenius norm of every
    step-1 factor F + eps I (F = beta init I + (1 - beta) G G^T or G^T G)."""
    out = []
    for (r, c), G in zip(shapes, grads):
        G = G.astype(np.float64)
        for (r0, r1, c0, c1) in step.block_grid(r, c, B):
            Gb = G[r0:r1, c0:c1]
            for P in (Gb @ Gb.T, Gb.T @ Gb):
                n = P.shape[0]
                A = hp.beta * hp.init_scale * np.eye(n) + (1.0 - hp.beta) * P + hp.eps * np.eye(n)
                w = np.linalg.eigvalsh(A)
                lam_pi, _ = roots.power_iteration(A, V0[:n], hp.pi_iters)
                out.append((w, lam_pi, np.linalg.norm(w)))
    return out


def summarise(name, spectra):
    t_pi = [iterations_to_tolerance(w, l) for (w, l, _) in spectra]
    t_fr = [iterations_to_tolerance(w, f) for (w, _, f) in spectra]
    kap = [w[-1] / w[0] for (w, _, _) in spectra]
    ratio = [f / l for (_, l, f) in spectra]

    def stats(ts):
        ok = [t for t in ts if t is not None]
        miss = len(ts) - len(ok)
        if not ok:
            return f"none within {T_MAX}"
        s = f"median {int(np.median(ok))}, max {max(ok)}"
        return s + (f", {miss} beyond {T_MAX}" if miss else "")

    return (f"| {name} | {len(spectra)} | {min(kap):.1e}-{max(kap):.1e} | "
            f"{np.median(ratio):.1f} | {stats(t_pi)} | {stats(t_fr)} |")


def main(argv=None):
    from matrix_inverse_roots_stack_b200 import workloads as wl
    p = argparse.ArgumentParser()
    p.add_argument("--quick", action="store_true", help="fewer Llama-shaped parameters")
    args = p.parse_args(argv)
    rows = []
    V0_256 = wl.pi_start_vectors(256, 32, seed=0).astype(np.float64)
    # standalone roots: 256 matrices of 256 with one closed-form spectrum
    A, _, w = wl.spd_stack_decaying(n=4, b=256, seed=0)
    spectra = []
    for i in range(A.shape[0]):
        Ai = A[i].astype(np.float64)
        lam, _ = roots.power_iteration(Ai, V0_256, 10)
        spectra.append((np.linalg.eigvalsh(Ai), lam, np.linalg.norm(Ai)))
    rows.append(summarise("standalone roots, 256 of 256 (4 sampled), eps = 0", spectra))
    # Llama ~1B shapes, B = 1024, step-1 factors (a sample of parameters)
    hp = step.HParams(block_size=1024)
    V0 = wl.pi_start_vectors(1024, 32, seed=0).astype(np.float64)
    shapes = [(2048, 2048), (2048, 5632), (5632, 2048)] + ([] if args.quick else [(32000, 2048)])
    grads = wl.gaussian_gradients(shapes, std=0.1, seed=0, row_lognormal_sigma=1.0)
    rows.append(summarise("Llama ~1B shapes, B = 1024 (" + ", ".join(f"{r}x{c}" for r, c in shapes) + ")",
                          factor_spectra(shapes, grads, 1024, hp, V0)))
    # GPT-2 124M shapes, B = 512, N(0, 0.1^2) gradients (no row scaling: a
    # flatter spectrum, where the Frobenius norm is many times lambda_max)
    hp512 = step.HParams(block_size=512)
    V0_512 = wl.pi_start_vectors(512, 32, seed=0).astype(np.float64)
    shapes = [(768, 2304), (768, 768), (768, 3072), (3072, 768)]
    grads = wl.gaussian_gradients(shapes, std=0.1, seed=0)
    rows.append(summarise("GPT-2 124M shapes, B = 512 (one layer: " + ", ".join(f"{r}x{c}" for r, c in shapes) + ")",
                          factor_spectra(shapes, grads, 512, hp512, V0_512)))
    # mixed sweep, Student-t gradients, B = 1024 and 2048
    shapes = wl.mixed_shapes()
    grads = wl.student_t_gradients(shapes, seed=0)
    for B in (1024, 2048):
        hpB = step.HParams(block_size=B)
        V0B = wl.pi_start_vectors(B, 32, seed=0).astype(np.float64)
        rows.append(summarise(f"mixed shapes, Student-t(3), B = {B}", factor_spectra(shapes, grads, B, hpB, V0B)))
    print("| workload | factors | kappa | ||A||_F / lambda_PI (median) | "
          f"iterations per stage to {TOL:g} of the exact root, power iteration | same, Frobenius |")
    print("|---|---|---|---|---|---|")
    for r in rows:
        print(r)
    return 0


if __name__ == "__main__":
    sys.exit(main())
