"""Full-size GPU runs of the step on the workloads' parameter sets, checked on
sampled blocks against the float64 oracle block by block.

The whole step runs on the GPU exactly as bench.py launches it; the oracle
recomputes a few blocks (first, middle, last -- edge blocks included) from
their gradient blocks, at the GPU's power-iteration estimates (level 2).
Tolerance: relative Frobenius error <= 5e-3 on each sampled block's update.
"""

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import workloads
from oracle import step as ostep
from tests.gpu_util import rel, cuda_or_skip

pytestmark = pytest.mark.gpu

UPDATE_TOL = 5e-3


@pytest.fixture(scope="module")
def torch():
    return cuda_or_skip()


def f32(x):
    return float(np.float32(x))


def run_and_check(torch, shapes, grads, B, solver="ndb", iters=14, degree=16, n_sample=6):
    from matrix_inverse_roots_stack_b200 import binding as bd
    dev = grads[0].device
    params = [torch.zeros_like(g) for g in grads]
    hpb = bd.make_hparams(block_size=B, solver=bd.SOLVER_NEWTON_DB if solver == "ndb" else bd.SOLVER_CHEBYSHEV,
                          ndb_iters1=iters, ndb_iters2=iters, cheb_degree=degree)
    opt = bd.Shampoo(params, grads, hp=hpb, v0=torch.from_numpy(workloads.pi_start_vectors(B, 32, seed=0)).to(dev))
    opt.step()
    rc, flags = opt.status()
    assert rc == 0, bd.strerror(rc)
    lam = opt.lam.cpu().numpy().astype(np.float64)
    table = opt.block_table()
    hp = ostep.HParams(block_size=B, solver=solver, ndb_iters1=iters, ndb_iters2=iters, cheb_degree=degree,
                       beta=f32(0.95), eps=f32(1e-6), init_scale=f32(1e-6), beta1=f32(0.9), beta2=f32(0.999),
                       adam_eps=f32(1e-8), lr=f32(1e-3), cheb_delta=f32(1e-3))
    nb = len(table)
    picks = sorted(set([0, 1, nb // 3, nb // 2, (2 * nb) // 3, nb - 1][:n_sample]))
    errs = []
    for k in picks:
        p, r0, c0, br, bc, fl, fr = (int(x) for x in table[k])
        Gb = grads[p][r0:r0 + br, c0:c0 + bc].cpu().numpy().astype(np.float64)
        _, _, Pb = ostep.adam_direction(Gb, np.zeros_like(Gb), np.zeros_like(Gb), 1, hp)
        d_ref, _, _ = ostep.first_step_block_update(Gb, Pb, hp, lam[fl], lam[fr])
        d_gpu = params[p][r0:r0 + br, c0:c0 + bc].cpu().numpy().astype(np.float64)
        if np.linalg.norm(d_ref) > 0:
            errs.append((k, br, bc, rel(d_gpu, d_ref)))
    worst = max(e[3] for e in errs)
    assert worst < UPDATE_TOL, errs
    return errs


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
