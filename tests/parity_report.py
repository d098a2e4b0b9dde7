"""Parity of the GPU path against the float64 oracle on each workload
configuration, printed as one JSON object.

The GPU parity tests assert these quantities against their tolerances; this
script reports the values themselves (relative Frobenius errors), for the
measurement table:

    python tests/parity_report.py > parity.json

Level 2 is the truncated method evaluated exactly at the GPU's power-
iteration estimates; level 1 the exact inverse root (eigendecomposition).
Needs a CUDA device.
"""

import dataclasses
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def spiked(torch, out):
    from matrix_inverse_roots_stack_b200 import workloads
    from oracle import step as ostep
    from tests import test_gpu_step as ts
    from tests.gpu_util import rel
    G = workloads.spiked_gradient(512, 512, rank=8, scale=10.0, seed=0)
    th = workloads.parameters([(512, 512)], seed=1)
    hp = ostep.HParams(block_size=128, ndb_iters1=8, ndb_iters2=8)
    gpu = ts.run_gpu(torch, th, [[G]], hp)
    d_gpu = gpu["theta"][0] - th[0].astype(np.float64)
    res = {}
    for level in (2, 1):
        h = dataclasses.replace(hp, root_level=level)
        ref, _, _ = ts.run_oracle(th, [[G]], h, gpu["lam"])
        res[f"dtheta_rel_level{level}"] = rel(d_gpu, ref[0] - th[0].astype(np.float64))
    res["tol_level2"] = 5e-3
    out["config1_spiked512_B128_ndb8+8"] = res


def standalone(torch, out):
    from matrix_inverse_roots_stack_b200 import binding as bd, workloads
    from oracle import roots
    from tests.gpu_util import rel
    A, U, lamv = workloads.spd_stack_decaying(n=256, b=256, seed=0)
    At = torch.from_numpy(A).cuda()
    vt = torch.from_numpy(workloads.pi_start_vectors(256, 32, seed=0)).cuda()
    exact = lambda i: (U[i] * lamv ** -0.25) @ U[i].T  # closed-form level 1
    sample = range(0, 256, 32)
    for name, call, lvl2 in (
            ("ndb14+14", lambda: bd.inv_root_newton_db(At, vt, iters1=14, iters2=14, eps=0.0),
             lambda Ai, l: roots.ndb_inv4root_spectral(Ai, l, 14, 14)),
            ("cheb16_delta1e-3", lambda: bd.inv_root_chebyshev(At, vt, degree=16, delta=1e-3, eps=0.0),
             lambda Ai, l: roots.cheb_inv4root_spectral(Ai, l, 16, 1e-3)),
            ("cn16", lambda: bd.inv_root_coupled_newton(At, vt, iters=16, eps=0.0),
             lambda Ai, l: roots.cn_inv4root_spectral(Ai, l, 16))):
        X, lam, ws = call()
        rc, _ = bd.read_status(ws)
        X = X.cpu().numpy().astype(np.float64)
        lam = lam.cpu().numpy().astype(np.float64)
        e2 = [rel(X[i], lvl2(A[i].astype(np.float64), lam[i])) for i in sample]
        e1 = [rel(X[i], exact(i)) for i in sample]
        out[f"config2_roots256x256_{name}"] = {"status": rc, "root_rel_level2_max": max(e2),
                                               "root_rel_level1_max": max(e1), "matrices_sampled": len(e2),
                                               "tol_level2": 1e-3}


def fullsize(torch, out):
    from matrix_inverse_roots_stack_b200 import workloads
    from tests.test_gpu_fullsize import run_and_check

    def record(key, rows):
        out[key] = {"blocks_sampled": len(rows),
                    "dtheta_rel_level2_max": max(r[4] for r in rows),
                    "kappa_max": max(r[3] for r in rows),
                    "tol_applied_max": max(r[5] for r in rows),
                    "per_block": [[int(r[0]), int(r[1]), int(r[2]), float(r[3]), float(r[4])] for r in rows]}

    shapes = workloads.gpt2_124m_shapes()
    g = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0)
    record("config3_gpt2_124m_B512_ndb14+14", run_and_check(torch, shapes, g, 512))
    del g
    shapes = workloads.llama_1b_shapes()
    g = workloads.torch_gaussian_gradients(shapes, "cuda", std=0.1, seed=0, row_lognormal_sigma=1.0)
    record("config4_llama1b_B1024_ndb14+14", run_and_check(torch, shapes, g, 1024, n_sample=5))
    del g
    torch.cuda.empty_cache()
    shapes = workloads.mixed_shapes()
    for B in (128, 256, 512, 1024, 2048):
        g = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=0)
        record(f"config5_mixed_B{B}_ndb14+14", run_and_check(torch, shapes, g, B, n_sample=4))
    for B in (512, 2048):
        g = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=1)
        record(f"config5_mixed_B{B}_cheb16", run_and_check(torch, shapes, g, B, solver="cheb", n_sample=4))
    for B in (256, 1024, 2048):
        g = workloads.torch_student_t_gradients(shapes, "cuda", nu=3.0, seed=2)
        record(f"config5_mixed_B{B}_ndb14+14_eps1e-2",
               run_and_check(torch, shapes, g, B, n_sample=4, eps=1e-2, require_regime=True))


def main():
    import torch
    from matrix_inverse_roots_stack_b200 import build
    build.build()
    out = {}
    spiked(torch, out)
    standalone(torch, out)
    fullsize(torch, out)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
