"""The entry point that allocates nothing: shampoo_inv_root_newton_db_static.

It serves callers that cannot call cudaMalloc (for instance a plug-in inside a
host framework that owns all device memory): its scratch is a fixed array in
the library's device memory instead of a caller workspace.  This test calls it
through the C ABI twice in a row, on different inputs, and checks each result
against the workspace entry point shampoo_inv_root_newton_db on the same
inputs, within the root tolerance the other GPU tests use, and reads the
status word the entry point keeps in its scratch after each call.  It also
checks that a problem larger than the scratch is rejected.  The file is named to be
collected last so that a run stopping at the first failure has already run
every other test.
"""

import ctypes

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import workloads
from tests.gpu_util import rel, cuda_or_skip

pytestmark = pytest.mark.gpu

ROOT_TOL = 1e-3


@pytest.fixture(scope="module")
def torch():
    return cuda_or_skip()


def call_static(torch, lib, At, vt, it, stream):
    n, B = At.shape[0], At.shape[1]
    X = torch.empty_like(At)
    lam = torch.empty(n, dtype=torch.float32, device=At.device)
    rc = lib.shampoo_inv_root_newton_db_static(ctypes.c_void_p(At.data_ptr()), ctypes.c_void_p(X.data_ptr()), n, B,
                                               it, it, 1e-6, ctypes.c_void_p(vt.data_ptr()), 10,
                                               ctypes.c_void_p(lam.data_ptr()), stream)
    return rc, X, lam


def test_static_scratch_matches_workspace_entry_point(torch):
    from matrix_inverse_roots_stack_b200 import binding as bd
    lib = bd.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    vt = torch.from_numpy(workloads.pi_start_vectors(256, 32, seed=0)).cuda()
    for call, (kappa, seed, it) in enumerate([(1e3, 11, 12), (1e4, 12, 16)]):
        A = workloads.spd_stack_geometric(6, 256, kappa, seed=seed)
        At = torch.from_numpy(A).cuda()
        rc, X, lam = call_static(torch, lib, At, vt, it, stream)
        assert rc == bd.SHAMPOO_OK, (call, bd.strerror(rc))
        # the scratch's status word reports a clean call
        assert bd.read_static_status() == (bd.SHAMPOO_OK, 0)
        torch.cuda.synchronize()
        Xw, lamw, ws = bd.inv_root_newton_db(At, vt, iters1=it, iters2=it, eps=1e-6, pi_iters=10)
        assert bd.read_status(ws)[0] == bd.SHAMPOO_OK
        X, Xw = X.cpu().numpy().astype(np.float64), Xw.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(X))
        assert np.allclose(lam.cpu().numpy(), lamw.cpu().numpy(), rtol=1e-6, atol=0)
        for i in range(6):
            assert rel(X[i], Xw[i]) < ROOT_TOL, (call, i, rel(X[i], Xw[i]))


def test_static_scratch_rejects_oversized_problem(torch):
    from matrix_inverse_roots_stack_b200 import binding as bd
    lib = bd.load()
    B = 1024
    n = 1
    while lib.shampoo_inv_root_workspace_bytes(n, B, 0) <= bd.STATIC_SCRATCH_BYTES:
        n += 1  # smallest stack that does not fit the 64 MiB scratch
    At = torch.zeros((n, B, B), dtype=torch.float32, device="cuda")
    vt = torch.zeros((B, 32), dtype=torch.float32, device="cuda")
    rc, _, _ = call_static(torch, lib, At, vt, 4, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == bd.SHAMPOO_EWORKSPACE
