"""Full-size GPU runs of the step on the workloads' parameter sets, checked on
sampled blocks against the float64 oracle block by block.

The whole step runs on the GPU exactly as bench.py launches it; the oracle
recomputes the sampled blocks from their gradient blocks, at the GPU's
power-iteration estimates (level 2).  The sample holds one block of every
distinct block shape of the parameter set (edge blocks: 256 x 1024 rows of
the embedding, 512-wide blocks of 5632, the 768 -> 512 + 256 and 50257 edges
of GPT-2) and evenly spaced blocks up to at least 32 (all blocks when there
are fewer).

Tolerance on a sampled block's update (relative Frobenius error of its
Delta theta): 5e-3, the parameter-update tolerance.  It holds for every
sampled block of the GPT-2 and Llama parameter sets (factor condition numbers
up to ~1e9) and for every block whose factors have kappa <= 1e6, the regime
the root tolerance is stated for.  The heavy-tailed Student-t sweep also has
blocks with kappa of 1e7 and beyond, where each K=16 partial product that the
tensor core rounds toward zero into tensor memory limits any fp32-level
evaluation of the truncated iteration.  Plain fp32 arithmetic rounded to
nearest does worse there.  Those blocks are held to 5e-2, which still
catches a wrong kernel, and their measured errors are printed.
"""

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import workloads
from oracle import step as ostep
from tests.gpu_util import assert_mirrored_blocks, rel, cuda_or_skip

pytestmark = pytest.mark.gpu

UPDATE_TOL = 5e-3
KAPPA_REGIME = 1e6
BEYOND_REGIME_TOL = 5e-2
MIN_SAMPLE = 32


@pytest.fixture(scope="module")
def torch():
    return cuda_or_skip()


def f32(x):
    return float(np.float32(x))


def kappa(M):
    w = np.linalg.eigvalsh(M)
    return w[-1] / w[0]


def sample_blocks(table, n_sample):
    """One block of every distinct (b_r, b_c) shape, then evenly spaced
    blocks until n_sample (or every block)."""
    nb = len(table)
    picks = {}
    for k in range(nb):
        picks.setdefault((int(table[k][3]), int(table[k][4])), k)
    chosen = set(picks.values())
    for k in np.linspace(0, nb - 1, num=min(nb, n_sample)).round().astype(int):
        if len(chosen) >= max(n_sample, len(picks)):
            break
        chosen.add(int(k))
    k = 0
    while len(chosen) < min(nb, n_sample):
        chosen.add(k)
        k += 1
    return sorted(chosen)


def run_and_check(torch, shapes, grads, B, solver="ndb", iters=14, degree=16, n_sample=MIN_SAMPLE, eps=1e-6,
                  require_regime=False, flat=True, cn_iters=16):
    from matrix_inverse_roots_stack_b200 import binding as bd
    dev = grads[0].device
    params = [torch.zeros_like(g) for g in grads]
    code = {"ndb": bd.SOLVER_NEWTON_DB, "cheb": bd.SOLVER_CHEBYSHEV, "cn": bd.SOLVER_COUPLED_NEWTON}[solver]
    hpb = bd.make_hparams(block_size=B, solver=code, ndb_iters1=iters, ndb_iters2=iters, cheb_degree=degree,
                          eps=eps, cn_iters=cn_iters)
    opt = bd.Shampoo(params, grads, hp=hpb, v0=torch.from_numpy(workloads.pi_start_vectors(B, 32, seed=0)).to(dev))
    opt.step()
    rc, flags = opt.status()
    assert rc == 0, bd.strerror(rc)
    assert_mirrored_blocks(torch, opt.factors)
    lam = opt.lam.cpu().numpy().astype(np.float64)
    table = opt.block_table()
    hp = ostep.HParams(block_size=B, solver=solver, ndb_iters1=iters, ndb_iters2=iters, cheb_degree=degree,
                       cn_iters=cn_iters, beta=f32(0.95), eps=f32(eps), init_scale=f32(1e-6), beta1=f32(0.9), beta2=f32(0.999),
                       adam_eps=f32(1e-8), lr=f32(1e-3), cheb_delta=f32(1e-3))
    rows = []
    for k in sample_blocks(table, n_sample):
        p, r0, c0, br, bc, fl, fr = (int(x) for x in table[k])
        Gb = grads[p][r0:r0 + br, c0:c0 + bc].cpu().numpy().astype(np.float64)
        _, _, Pb = ostep.adam_direction(Gb, np.zeros_like(Gb), np.zeros_like(Gb), 1, hp)
        d_ref, _, _ = ostep.first_step_block_update(Gb, Pb, hp, lam[fl], lam[fr])
        d_gpu = params[p][r0:r0 + br, c0:c0 + bc].cpu().numpy().astype(np.float64)
        if np.linalg.norm(d_ref) == 0:
            assert np.all(d_gpu == 0.0), k
            continue
        L, R = ostep.factor_ema(hp.init_scale * np.eye(br), hp.init_scale * np.eye(bc), Gb, hp.beta)
        kap = max(kappa(L + hp.eps * np.eye(br)), kappa(R + hp.eps * np.eye(bc)))
        rows.append((k, br, bc, kap, rel(d_gpu, d_ref)))
    assert len(rows) >= min(n_sample, len(table)) - 1
    if require_regime:
        assert all(r[3] <= KAPPA_REGIME for r in rows), rows
    worst = max(rows, key=lambda r: r[4])
    print(f"B={B} {solver}: {len(rows)} blocks, worst update error {worst[4]:.2e} (block {worst[0]}, "
          f"{worst[1]}x{worst[2]}, kappa {worst[3]:.1e}); kappa up to {max(r[3] for r in rows):.1e}")
    tol = lambda r: UPDATE_TOL if (flat or r[3] <= KAPPA_REGIME) else BEYOND_REGIME_TOL
    beyond = [r for r in rows if tol(r) > UPDATE_TOL]
    if beyond:
        print(f"  {len(beyond)} blocks beyond kappa {KAPPA_REGIME:.0e}: errors " +
              ", ".join(f"{r[4]:.1e} (kappa {r[3]:.1e})" for r in beyond))
    assert all(r[4] < tol(r) for r in rows), [r for r in rows if r[4] >= tol(r)]
    return rows


def test_gpt2_124m_b512(torch):
    shapes = workloads.gpt2_124m_shapes()
    grads = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0)
    run_and_check(torch, shapes, grads, 512)


def test_llama_1b_b1024(torch):
    shapes = workloads.llama_1b_shapes()
    grads = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0, row_lognormal_sigma=1.0)
    run_and_check(torch, shapes, grads, 1024)


@pytest.mark.parametrize("B", [128, 256, 512, 1024, 2048])
def test_mixed_shapes_block_sweep(torch, B):
    shapes = workloads.mixed_shapes()
    grads = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=0)
    run_and_check(torch, shapes, grads, B, flat=False)


@pytest.mark.parametrize("B,degree", [(512, 16), (2048, 16), (1024, 60), (2048, 60)])
def test_mixed_shapes_chebyshev(torch, B, degree):
    # degree 60 is the explainer's figure for the Chebyshev solver
    shapes = workloads.mixed_shapes()
    grads = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=1)
    run_and_check(torch, shapes, grads, B, solver="cheb", degree=degree, flat=False)


@pytest.mark.parametrize("degree", [16, 60])
def test_llama_1b_b1024_chebyshev(torch, degree):
    shapes = workloads.llama_1b_shapes()
    grads = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0, row_lognormal_sigma=1.0)
    run_and_check(torch, shapes, grads, 1024, solver="cheb", degree=degree)


def test_llama_1b_b1024_coupled_newton(torch):
    # split-fp16 coupled Newton, 16 iterations, on upper-triangle tiles
    shapes = workloads.llama_1b_shapes()
    grads = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0, row_lognormal_sigma=1.0)
    run_and_check(torch, shapes, grads, 1024, solver="cn")


@pytest.mark.parametrize("B", [256, 1024, 2048])
def test_mixed_shapes_in_regime(torch, B):
    # root-time damping eps = 3e-2 bounds every factor's condition number by
    # 1e6 here, the regime the root tolerance is stated for
    shapes = workloads.mixed_shapes()
    grads = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=2)
    run_and_check(torch, shapes, grads, B, eps=3e-2, require_regime=True)
