"""Full-size GPU runs of the step on the workloads' parameter sets, checked on
sampled blocks against the float64 oracle block by block.

The whole step runs on the GPU exactly as bench.py launches it; the oracle
recomputes a few blocks (first, middle, last -- edge blocks included) from
their gradient blocks, at the GPU's power-iteration estimates (level 2).

Tolerance on each sampled block's update (relative Frobenius error): 5e-3
when both of its factors (with the root-time damping) have condition number
<= 1e6, the regime the root tolerance is stated for.  First-step factors of
these workloads reach 1e7 and more; there the error of any fp32-precision
evaluation of the truncated iteration grows with the condition number, and
the bound used is 5e-3 * kappa / 1e6.  The in-regime variants damp the
factors (eps = 1e-2) so that every block satisfies kappa <= 1e6 and hold all
of them to 5e-3.
"""

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import workloads
from oracle import step as ostep
from tests.gpu_util import rel, cuda_or_skip

pytestmark = pytest.mark.gpu

UPDATE_TOL = 5e-3
KAPPA_REGIME = 1e6


@pytest.fixture(scope="module")
def torch():
    return cuda_or_skip()


def f32(x):
    return float(np.float32(x))


def kappa(M):
    w = np.linalg.eigvalsh(M)
    return w[-1] / w[0]


def run_and_check(torch, shapes, grads, B, solver="ndb", iters=14, degree=16, n_sample=6, eps=1e-6,
                  require_regime=False):
    from matrix_inverse_roots_stack_b200 import binding as bd
    dev = grads[0].device
    params = [torch.zeros_like(g) for g in grads]
    hpb = bd.make_hparams(block_size=B, solver=bd.SOLVER_NEWTON_DB if solver == "ndb" else bd.SOLVER_CHEBYSHEV,
                          ndb_iters1=iters, ndb_iters2=iters, cheb_degree=degree, eps=eps)
    opt = bd.Shampoo(params, grads, hp=hpb, v0=torch.from_numpy(workloads.pi_start_vectors(B, 32, seed=0)).to(dev))
    opt.step()
    rc, flags = opt.status()
    assert rc == 0, bd.strerror(rc)
    lam = opt.lam.cpu().numpy().astype(np.float64)
    table = opt.block_table()
    hp = ostep.HParams(block_size=B, solver=solver, ndb_iters1=iters, ndb_iters2=iters, cheb_degree=degree,
                       beta=f32(0.95), eps=f32(eps), init_scale=f32(1e-6), beta1=f32(0.9), beta2=f32(0.999),
                       adam_eps=f32(1e-8), lr=f32(1e-3), cheb_delta=f32(1e-3))
    nb = len(table)
    picks = sorted(set([0, 1, nb // 3, nb // 2, (2 * nb) // 3, nb - 1][:n_sample]))
    rows = []
    for k in picks:
        p, r0, c0, br, bc, fl, fr = (int(x) for x in table[k])
        Gb = grads[p][r0:r0 + br, c0:c0 + bc].cpu().numpy().astype(np.float64)
        _, _, Pb = ostep.adam_direction(Gb, np.zeros_like(Gb), np.zeros_like(Gb), 1, hp)
        d_ref, _, _ = ostep.first_step_block_update(Gb, Pb, hp, lam[fl], lam[fr])
        d_gpu = params[p][r0:r0 + br, c0:c0 + bc].cpu().numpy().astype(np.float64)
        if np.linalg.norm(d_ref) == 0:
            continue
        L, R = ostep.factor_ema(hp.init_scale * np.eye(br), hp.init_scale * np.eye(bc), Gb, hp.beta)
        kap = max(kappa(L + hp.eps * np.eye(br)), kappa(R + hp.eps * np.eye(bc)))
        tol = UPDATE_TOL * max(1.0, kap / KAPPA_REGIME)
        rows.append((k, br, bc, kap, rel(d_gpu, d_ref), tol))
    assert rows
    if require_regime:
        assert all(r[3] <= KAPPA_REGIME for r in rows), rows
    assert all(r[4] < r[5] for r in rows), rows
    return rows


def test_gpt2_124m_b512(torch):
    shapes = workloads.gpt2_124m_shapes()
    grads = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0)
    run_and_check(torch, shapes, grads, 512)


def test_llama_1b_b1024(torch):
    shapes = workloads.llama_1b_shapes()
    grads = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0, row_lognormal_sigma=1.0)
    run_and_check(torch, shapes, grads, 1024, n_sample=5)


@pytest.mark.parametrize("B", [128, 256, 512, 1024, 2048])
def test_mixed_shapes_block_sweep(torch, B):
    shapes = workloads.mixed_shapes()
    grads = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=0)
    run_and_check(torch, shapes, grads, B, n_sample=4)


@pytest.mark.parametrize("B", [512, 2048])
def test_mixed_shapes_chebyshev(torch, B):
    shapes = workloads.mixed_shapes()
    grads = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=1)
    run_and_check(torch, shapes, grads, B, solver="cheb", degree=16, n_sample=4)


@pytest.mark.parametrize("B", [256, 1024, 2048])
def test_mixed_shapes_in_regime(torch, B):
    # root-time damping eps = 1e-2 bounds every factor's condition number by
    # 1e6 here, so every sampled block is held to the stated 5e-3
    shapes = workloads.mixed_shapes()
    grads = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=2)
    run_and_check(torch, shapes, grads, B, n_sample=4, eps=1e-2, require_regime=True)
