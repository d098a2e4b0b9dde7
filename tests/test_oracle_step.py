"""Pins of the oracle's blocking, factor EMA, preconditioning and grafting."""

import os

import numpy as np
import pytest

from oracle import step
from matrix_inverse_roots_stack_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(b)


def test_block_grid_partitions_exactly():
    for (m, n, B) in [(512, 512, 128), (768, 2304, 512), (50257, 768, 512), (5, 7, 3)]:
        cover = np.zeros((m, n), dtype=np.int32)
        for (r0, r1, c0, c1) in step.block_grid(m, n, B):
            assert 0 < r1 - r0 <= B and 0 < c1 - c0 <= B
            cover[r0:r1, c0:c1] += 1
        assert cover.min() == 1 and cover.max() == 1


def test_block_grid_embedding_golden():
    with open(os.path.join(GOLDEN, "embedding_blocks_b1024.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    m, n, B, full, edge, er, ec = map(int, rows[0])
    blocks = step.block_grid(m, n, B)
    sizes = [(r1 - r0, c1 - c0) for (r0, r1, c0, c1) in blocks]
    assert sum(1 for s in sizes if s == (B, B)) == full
    edges = [s for s in sizes if s != (B, B)]
    assert len(edges) == edge and all(s == (er, ec) for s in edges)


def test_factor_ema_brute_force():
    rng = np.random.default_rng(0)
    G = rng.standard_normal((3, 5))
    L0, R0 = np.diag([1.0, 2.0, 3.0]), np.eye(5) * 0.5
    beta = 0.9
    L, R = step.factor_ema(L0, R0, G, beta)
    for i in range(3):
        for j in range(3):
            s = sum(G[i, k] * G[j, k] for k in range(5))
            assert L[i, j] == pytest.approx(beta * L0[i, j] + (1 - beta) * s, abs=1e-14)
    for i in range(5):
        for j in range(5):
            s = sum(G[k, i] * G[k, j] for k in range(3))
            assert R[i, j] == pytest.approx(beta * R0[i, j] + (1 - beta) * s, abs=1e-14)


def one_block_step(G, hp, level=1):
    hp.root_level = level
    state = step.init_state([G.shape], hp)
    V0 = workloads.pi_start_vectors(hp.block_size, 32, seed=0)
    th = np.zeros(G.shape)
    return step.shampoo_step([th], [G], state, hp, V0)


def test_precondition_closed_form_rectangular():
    # G = U diag(s) V^T; after one step from init_scale*I the factors are
    # U diag(a s^2) U^T + e I and V diag(a s^2) V^T + e I (a = 1-beta,
    # e = beta*init_scale + eps), so X_L G X_R = U diag(s (a s^2 + e)^-1/2) V^T.
    rng = np.random.default_rng(1)
    br, bc, r = 12, 7, 5
    U, _ = np.linalg.qr(rng.standard_normal((br, r)))
    V, _ = np.linalg.qr(rng.standard_normal((bc, r)))
    s = np.array([3.0, 1.0, 0.5, 0.1, 0.02])
    G = (U * s) @ V.T
    hp = step.HParams(block_size=16)
    _, _, info = one_block_step(G, hp, level=1)
    a, e = 1 - hp.beta, hp.beta * hp.init_scale + hp.eps
    expect = (U * (s / np.sqrt(a * s * s + e))) @ V.T
    assert rel(info["U"][0], expect) < 1e-9


def test_precondition_closed_form_orthogonal():
    rng = np.random.default_rng(2)
    Q = workloads.haar_orthogonal(16, rng)
    sigma = 0.7
    hp = step.HParams(block_size=16)
    _, _, info = one_block_step(sigma * Q, hp, level=1)
    scale = ((1 - hp.beta) * sigma ** 2 + hp.beta * hp.init_scale + hp.eps) ** -0.5
    assert rel(info["U"][0], sigma * Q * scale) < 1e-12


def test_graft_norm_invariant():
    G = workloads.spiked_gradient(40, 56, rank=3, scale=10.0, seed=3).astype(np.float64)
    hp = step.HParams(block_size=16, ndb_iters1=8, ndb_iters2=8)
    state = step.init_state([G.shape], hp)
    V0 = workloads.pi_start_vectors(16, 32, seed=0)
    th0 = workloads.parameters([G.shape], seed=5)[0].astype(np.float64)
    new, _, info = step.shampoo_step([th0], [G], state, hp, V0)
    d = new[0] - th0
    for (r0, r1, c0, c1) in step.block_grid(*G.shape, 16):
        pn = np.linalg.norm(info["P"][0][r0:r1, c0:c1])
        assert np.linalg.norm(d[r0:r1, c0:c1]) == pytest.approx(hp.lr * pn, rel=1e-12)


def test_adam_first_step_closed_form():
    hp = step.HParams()
    G = np.array([[1.0, -2.0], [1e-9, 0.0]])
    m, v, P = step.adam_direction(G, np.zeros_like(G), np.zeros_like(G), 1, hp)
    assert np.allclose(P, G / (np.abs(G) + hp.adam_eps), rtol=1e-12, atol=0)
    assert np.allclose(m, (1 - hp.beta1) * G) and np.allclose(v, (1 - hp.beta2) * G * G)


def test_adam_bias_correction_constant_gradient():
    hp = step.HParams()
    g = np.array([[0.3, -4.0, 2e-3]])
    m = v = np.zeros_like(g)
    for t in range(1, 8):
        m, v, P = step.adam_direction(g, m, v, t, hp)
        assert np.allclose(P, g / (np.abs(g) + hp.adam_eps), rtol=1e-12, atol=0)


def test_zero_block_grafts_to_zero():
    G = np.zeros((16, 16))
    G[:8, :8] = np.random.default_rng(0).standard_normal((8, 8))
    hp = step.HParams(block_size=8, ndb_iters1=8, ndb_iters2=8)
    state = step.init_state([G.shape], hp)
    V0 = workloads.pi_start_vectors(8, 32, seed=0)
    new, _, info = step.shampoo_step([np.zeros_like(G)], [G], state, hp, V0)
    assert info["graft"][1] == 0.0 and np.all(new[0][:8, 8:] == 0.0)


def test_edge_blocks_are_independent_problems():
    # a 20 x 13 gradient at B=8: each block's update equals the update of that
    # block run as a parameter of its own
    G = workloads.student_t_gradients([(20, 13)], seed=4)[0].astype(np.float64)
    hp = step.HParams(block_size=8, ndb_iters1=10, ndb_iters2=10)
    V0 = workloads.pi_start_vectors(8, 32, seed=1)
    new, _, _ = step.shampoo_step([np.zeros_like(G)], [G], step.init_state([G.shape], hp), hp, V0)
    for (r0, r1, c0, c1) in step.block_grid(20, 13, 8):
        Gb = G[r0:r1, c0:c1]
        nb, _, _ = step.shampoo_step([np.zeros_like(Gb)], [Gb],
                                     step.init_state([Gb.shape], hp), hp, V0)
        assert rel(new[0][r0:r1, c0:c1], nb[0]) < 1e-13


def test_converged_truncated_step_matches_exact_step():
    G = workloads.gaussian_gradients([(24, 40)], std=0.1, seed=6)[0].astype(np.float64)
    V0 = workloads.pi_start_vectors(16, 32, seed=2)
    out = {}
    for level in (1, 2, 3):
        hp = step.HParams(block_size=16, ndb_iters1=40, ndb_iters2=40, root_level=level,
                          eps=1e-3)
        new, _, _ = step.shampoo_step([np.zeros_like(G)], [G],
                                      step.init_state([G.shape], hp), hp, V0)
        out[level] = new[0]
    assert rel(out[2], out[1]) < 1e-9
    assert rel(out[3], out[2]) < 1e-9


def test_first_step_block_update_matches_full_step():
    G = workloads.gaussian_gradients([(40, 24)], std=0.1, seed=11)[0].astype(np.float64)
    hp = step.HParams(block_size=16, ndb_iters1=9, ndb_iters2=9)
    V0 = workloads.pi_start_vectors(16, 32, seed=0)
    th0 = np.zeros(G.shape)
    new, _, info = step.shampoo_step([th0], [G], step.init_state([G.shape], hp), hp, V0)
    for k, (r0, r1, c0, c1) in enumerate(step.block_grid(40, 24, 16)):
        d, _, s = step.first_step_block_update(G[r0:r1, c0:c1], info["P"][0][r0:r1, c0:c1], hp,
                                               info["lam"][2 * k], info["lam"][2 * k + 1])
        assert rel(d, new[0][r0:r1, c0:c1]) < 1e-13 and s == pytest.approx(info["graft"][k], rel=1e-13)


def test_frobenius_scale_is_the_frobenius_norm_diagonal():
    # diagonal factor: ||A||_F = sqrt(sum lambda_i^2), an upper bound of
    # lambda_max; with enough iterations the truncated root at that scale is
    # the exact diag(lambda^-1/4)
    lam = np.array([3.0, 1.0, 0.5, 0.25, 0.1, 0.05, 0.02, 0.01])
    A = np.diag(lam)
    hp = step.HParams(block_size=8, scaling="frobenius", ndb_iters1=40, ndb_iters2=40, root_level=2)
    X, lam_est = step.inverse_fourth_root(A, None, hp)
    assert lam_est == pytest.approx(np.sqrt(np.sum(lam ** 2)), rel=1e-15)
    assert lam_est >= lam.max()
    assert rel(X, np.diag(lam ** -0.25)) < 1e-10
    hp.scaling = "nonsense"
    with pytest.raises(ValueError):
        step.inverse_fourth_root(A, None, hp)


def test_root_every_reuses_the_last_root_step_closed_form():
    # gradients sigma_t Q_t with Q_t orthogonal keep every factor a multiple of
    # I: after step t, L = R = a_t I with a_t = beta a_{t-1} + (1-beta) sigma_t^2,
    # a_0 = init_scale.  Exact roots (level 1) give U_t = sigma_t Q_t (a + eps)^-1/2
    # where a is a_t on root steps and the last root step's a otherwise.
    rng = np.random.default_rng(7)
    b, sig = 8, [0.7, 1.9, 0.4, 1.1]
    Qs = [workloads.haar_orthogonal(b, rng) for _ in sig]
    V0 = workloads.pi_start_vectors(b, 32, seed=0)
    for every, roots_at in [(1, [1, 2, 3, 4]), (2, [1, 3]), (3, [1, 4])]:
        hp = step.HParams(block_size=b, root_level=1, root_every=every)
        state = step.init_state([(b, b)], hp)
        th = [np.zeros((b, b))]
        a, a_root = hp.init_scale, None
        for t, (s_t, Q) in enumerate(zip(sig, Qs), start=1):
            th, state, info = step.shampoo_step(th, [s_t * Q], state, hp, V0)
            a = hp.beta * a + (1 - hp.beta) * s_t ** 2
            if t in roots_at:
                a_root = a
            assert info["root_step"] == (t in roots_at)
            assert rel(info["U"][0], s_t * Q * (a_root + hp.eps) ** -0.5) < 1e-12
