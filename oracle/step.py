"""Blocking, factor EMA, preconditioning, Adam grafting: the full step, float64.

Test infrastructure only (see the package docstring).  Follows the DASH
explainer's "High-level flow" and "Step-by-step" sections, in that order:
build/EMA the preconditioners L, R per block; scale each block by a
multi-start power-iteration estimate; compute inverse fourth roots; graft the
preconditioned direction to Adam's norm; apply the update.

The oracle does not pad edge blocks: an edge block of size b_r x b_c has its
own b_r x b_r and b_c x b_c factors.  Nothing here is shared with the CUDA
library.
"""

from dataclasses import dataclass

import numpy as np

from . import roots


@dataclass
class HParams:
    """Hyper-parameters of one step (names follow the pages' notation).

    Readings where the pages are silent: beta=0.95 for the factor EMA,
    eps=1e-6 added at root time only, initial factors init_scale*I with
    init_scale=1e-6, textbook bias-corrected Adam (beta1=0.9, beta2=0.999,
    adam_eps=1e-8), per-block grafting, power iteration with ``pi_iters``
    products, Newton-DB ``ndb_iters1`` + ``ndb_iters2`` iterations, Chebyshev
    degree ``cheb_degree`` on [cheb_delta, 1 + cheb_delta], coupled Newton
    ``cn_iters`` iterations.

    ``scaling``: the scale estimate of each factor ("Building blocks",
    scaling): "spectral" (multi-start power iteration) or "frobenius"
    (lambda = ||L + eps I||_F, which bounds lambda_max from above).
    ``root_every``: roots are recomputed on steps 1, 1 + f, 1 + 2f, ... and
    reused in between, while the factors, moments and parameters are updated
    every step (the update-frequency variant the pages time).
    """
    block_size: int = 128
    beta: float = 0.95
    eps: float = 1e-6
    init_scale: float = 1e-6
    beta1: float = 0.9
    beta2: float = 0.999
    adam_eps: float = 1e-8
    lr: float = 1e-3
    solver: str = "ndb"          # "ndb" | "cheb" | "cn"
    ndb_iters1: int = 14
    ndb_iters2: int = 14
    cheb_degree: int = 16
    cheb_delta: float = 1e-3
    cn_iters: int = 16
    pi_iters: int = 10
    root_level: int = 2          # 1 exact, 2 truncated method (spectral), 3 matmul
    scaling: str = "spectral"    # "spectral" | "frobenius"
    root_every: int = 1


def block_grid(rows, cols, B):
    """Tile an m x n matrix into B x B blocks, edge blocks smaller.

    DASH explainer, "Step-by-step" (split into blocks and stack): break layers
    into B x B blocks.  Reading: cuts at multiples of B, the last row/column
    chunk partial.  Returns a list of (r0, r1, c0, c1) in row-major order.
    """
    if B < 1:
        raise ValueError("block size must be positive")
    out = []
    for r0 in range(0, rows, B):
        for c0 in range(0, cols, B):
            out.append((r0, min(r0 + B, rows), c0, min(c0 + B, cols)))
    return out


def factor_ema(L, R, G, beta):
    """L <- beta L + (1-beta) G G^T ; R <- beta R + (1-beta) G^T G.

    DASH explainer, "Step-by-step" (build preconditioners): exponential moving
    averages of G G^T and G^T G.  No bias correction (the page has none).
    """
    G = np.asarray(G, dtype=np.float64)
    return beta * L + (1.0 - beta) * (G @ G.T), beta * R + (1.0 - beta) * (G.T @ G)


def inverse_fourth_root(Abar, V0, hp, lam_est=None):
    """Inverse fourth root of one regularised factor at the chosen level.

    Returns (X, lambda_est).  ``lam_est`` overrides the power-iteration
    estimate (the estimate depends on the random starts, so a parity check
    evaluates the truncated method at the estimate the GPU used).
    """
    b = Abar.shape[0]
    if lam_est is None:
        if hp.scaling == "frobenius":
            lam_est = float(np.linalg.norm(Abar, "fro"))
        elif hp.scaling == "spectral":
            lam_est, _ = roots.power_iteration(Abar, V0[:b], hp.pi_iters)
        else:
            raise ValueError("unknown scaling")
    if hp.solver == "ndb":
        if hp.root_level == 1:
            X = roots.inv_root_eigh(Abar, 4)
        elif hp.root_level == 2:
            X = roots.ndb_inv4root_spectral(Abar, lam_est, hp.ndb_iters1, hp.ndb_iters2)
        else:
            X = roots.ndb_inv4root_matmul(Abar, lam_est, hp.ndb_iters1, hp.ndb_iters2)
    elif hp.solver == "cn":
        if hp.root_level == 1:
            X = roots.inv_root_eigh(Abar, 4)
        elif hp.root_level == 2:
            X = roots.cn_inv4root_spectral(Abar, lam_est, hp.cn_iters)
        else:
            X = roots.cn_inv4root_matmul(Abar, lam_est, hp.cn_iters)
    elif hp.solver == "cheb":
        if hp.root_level == 1:
            shift = hp.cheb_delta / roots.ndb_scale(lam_est)
            X = roots.inv_root_eigh(Abar + shift * np.eye(b), 4)
        elif hp.root_level == 2:
            X = roots.cheb_inv4root_spectral(Abar, lam_est, hp.cheb_degree, hp.cheb_delta)
        else:
            X = roots.cheb_inv4root_matmul(Abar, lam_est, hp.cheb_degree, hp.cheb_delta)
    else:
        raise ValueError("unknown solver")
    return X, lam_est


def adam_direction(G, m, v, t, hp):
    """Bias-corrected Adam moments and direction P = m_hat/(sqrt(v_hat)+eps).

    DASH explainer, "Step-by-step" (grafting): P is the Adam-like direction.
    Reading: textbook Adam (Kingma & Ba 2015).  Returns (m, v, P).
    """
    G = np.asarray(G, dtype=np.float64)
    m = hp.beta1 * m + (1.0 - hp.beta1) * G
    v = hp.beta2 * v + (1.0 - hp.beta2) * G * G
    mh = m / (1.0 - hp.beta1 ** t)
    vh = v / (1.0 - hp.beta2 ** t)
    return m, v, mh / (np.sqrt(vh) + hp.adam_eps)


def graft_scale(P, U):
    """s = ||P||_F / ||U||_F (0 when U vanishes).

    DASH explainer, "Step-by-step" (grafting with Adam's magnitude).
    """
    nu = np.linalg.norm(U)
    return 0.0 if nu == 0.0 else float(np.linalg.norm(P) / nu)


def init_state(shapes, hp):
    """Per-parameter state: factors L = R = init_scale*I per block, m = v = 0."""
    state = []
    for (rows, cols) in shapes:
        blocks = []
        for (r0, r1, c0, c1) in block_grid(rows, cols, hp.block_size):
            blocks.append({
                "L": hp.init_scale * np.eye(r1 - r0),
                "R": hp.init_scale * np.eye(c1 - c0),
            })
        state.append({"blocks": blocks, "m": np.zeros((rows, cols)),
                      "v": np.zeros((rows, cols))})
    return {"params": state, "t": 0}


def shampoo_step(thetas, grads, state, hp, V0, lam_override=None):
    """One batched block-Shampoo step (every step preconditioned).

    ``thetas``, ``grads``: lists of 2-D arrays.  ``V0``: (block_size, K) start
    vectors for the power iteration (an edge factor of size b uses the first b
    rows).  ``lam_override``: optional sequence of per-factor estimates in the
    library's factor order (for block k in parameter order and row-major block
    order: factor 2k is its L, 2k+1 its R).

    Returns (new_thetas, new_state, info) with info = {"lam": [...],
    "graft": [...], "U": [...], "P": [...], "root_step": bool}; on steps that
    reuse roots, "lam" holds the estimates of the step that computed them.
    """
    t = state["t"] + 1
    f_every = max(1, int(hp.root_every))
    root_step = (t - 1) % f_every == 0
    new_thetas, new_params = [], []
    lam_out, graft_out, U_out, P_out = [], [], [], []
    f = 0
    for th, G, ps in zip(thetas, grads, state["params"]):
        th = np.array(th, dtype=np.float64, copy=True)
        G = np.asarray(G, dtype=np.float64)
        m, v, P = adam_direction(G, ps["m"], ps["v"], t, hp)
        U_full = np.zeros_like(th)
        new_blocks = []
        for (r0, r1, c0, c1), blk in zip(block_grid(*th.shape, hp.block_size), ps["blocks"]):
            Gb = G[r0:r1, c0:c1]
            L, R = factor_ema(blk["L"], blk["R"], Gb, hp.beta)
            if root_step or "XL" not in blk:
                XL, lamL = inverse_fourth_root(
                    L + hp.eps * np.eye(L.shape[0]), V0, hp,
                    None if lam_override is None else lam_override[f])
                XR, lamR = inverse_fourth_root(
                    R + hp.eps * np.eye(R.shape[0]), V0, hp,
                    None if lam_override is None else lam_override[f + 1])
            else:  # reuse the roots of the last root step
                XL, XR, lamL, lamR = blk["XL"], blk["XR"], blk["lamL"], blk["lamR"]
            new_blocks.append({"L": L, "R": R, "XL": XL, "XR": XR, "lamL": lamL, "lamR": lamR})
            lam_out += [lamL, lamR]
            f += 2
            Ub = XL @ Gb @ XR
            s = graft_scale(P[r0:r1, c0:c1], Ub)
            graft_out.append(s)
            U_full[r0:r1, c0:c1] = Ub
            th[r0:r1, c0:c1] -= hp.lr * s * Ub
        new_thetas.append(th)
        new_params.append({"blocks": new_blocks, "m": m, "v": v})
        U_out.append(U_full)
        P_out.append(P)
    info = {"lam": lam_out, "graft": graft_out, "U": U_out, "P": P_out, "root_step": root_step}
    return new_thetas, {"params": new_params, "t": t}, info


def first_step_block_update(Gb, Pb, hp, lam_L, lam_R):
    """Delta theta of one block on the first step, from its gradient block.

    Same arithmetic as :func:`shampoo_step` restricted to one block (factors
    start at init_scale*I; P is that block of the Adam direction), so that
    sampled blocks of a large parameter set can be checked one by one.
    Returns (delta, U, s).
    """
    Gb = np.asarray(Gb, dtype=np.float64)
    br, bc = Gb.shape
    L, R = factor_ema(hp.init_scale * np.eye(br), hp.init_scale * np.eye(bc), Gb, hp.beta)
    XL, _ = inverse_fourth_root(L + hp.eps * np.eye(br), None, hp, lam_L)
    XR, _ = inverse_fourth_root(R + hp.eps * np.eye(bc), None, hp, lam_R)
    U = XL @ Gb @ XR
    s = graft_scale(Pb, U)
    return -hp.lr * s * U, U, s

