"""The standalone root calls inside a CUDA graph.

The calls are stream-ordered, allocate no device memory and make no
non-stream CUDA calls after the first launch of each kernel on a device, so a
call can be captured once and replayed: a replay must reproduce the eager
call on the same inputs, and recompute from new inputs copied into the same
buffers.  Replays may differ from the eager call only in the summation order
of the power iteration's fp32 atomic column sums.
"""

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import workloads
from tests.gpu_util import rel, cuda_or_skip

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    return cuda_or_skip()


@pytest.mark.parametrize("solver", ["ndb", "cheb", "cn"])
def test_standalone_roots_replay_from_a_cuda_graph(torch, solver):
    from matrix_inverse_roots_stack_b200 import binding as bd
    n, B = 6, 256
    A1 = torch.from_numpy(workloads.spd_stack_geometric(n, B, 1e3, seed=3)).cuda()
    A2 = torch.from_numpy(workloads.spd_stack_geometric(n, B, 1e2, seed=4)).cuda()
    v0 = torch.from_numpy(workloads.pi_start_vectors(B, 32, seed=0)).cuda()
    code = {"ndb": bd.SOLVER_NEWTON_DB, "cheb": bd.SOLVER_CHEBYSHEV, "cn": bd.SOLVER_COUPLED_NEWTON}[solver]
    A = A1.clone()
    X = torch.empty_like(A)
    lam = torch.empty(n, dtype=torch.float32, device="cuda")
    ws = torch.empty(bd.inv_root_workspace_bytes(n, B, code), dtype=torch.uint8, device="cuda")

    def call(stream=None):
        if solver == "ndb":
            bd.inv_root_newton_db(A, v0, 14, 14, 1e-6, 10, X, lam, ws, stream)
        elif solver == "cheb":
            bd.inv_root_chebyshev(A, v0, 16, 1e-3, 1e-6, 10, X, lam, ws, stream)
        else:
            bd.inv_root_coupled_newton(A, v0, 16, False, 1e-6, 10, X, lam, ws, stream)

    eager = {}
    for name, src in (("A1", A1), ("A2", A2)):
        A.copy_(src)
        call()
        torch.cuda.synchronize()
        assert bd.read_status(ws)[0] == 0
        eager[name] = (X.clone(), lam.clone())

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    A.copy_(A1)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        call()
    for name, src in (("A1", A1), ("A2", A2), ("A1", A1)):
        X.zero_()
        A.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        assert bd.read_status(ws)[0] == 0
        Xe, le = eager[name]
        assert rel(lam.cpu().numpy(), le.cpu().numpy()) < 1e-5, (solver, name)
        for i in range(n):
            assert rel(X[i].cpu().numpy(), Xe[i].cpu().numpy()) < 1e-5, (solver, name, i)


def test_full_step_replays_from_a_cuda_graph(torch):
    # after one eager step, a step whose number comes from the device counter
    # (step = 0 at the C ABI) is captured once and replayed for the later
    # steps; it must match a twin optimizer stepped eagerly with explicit
    # step numbers (Adam bias correction included)
    from matrix_inverse_roots_stack_b200 import binding as bd
    shapes = [(300, 200), (128, 256), (5, 7)]
    B = 128
    hp = bd.make_hparams(block_size=B, ndb_iters1=12, ndb_iters2=12)
    v0 = torch.from_numpy(workloads.pi_start_vectors(B, 32, seed=0)).cuda()
    theta = workloads.parameters(shapes, seed=2)
    steps = [workloads.gaussian_gradients(shapes, std=0.1, seed=20 + k) for k in range(4)]

    def make():
        P = [torch.from_numpy(t.copy()).cuda() for t in theta]
        G = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
        return P, G, bd.Shampoo(P, G, hp=hp, v0=v0)

    def load(G, gs):
        for g, x in zip(G, gs):
            g.copy_(torch.from_numpy(x))

    Pe, Ge, ref = make()
    for gs in steps:
        load(Ge, gs)
        ref.step()
    Pg, Gg, opt = make()
    load(Gg, steps[0])
    opt.step()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        opt.step(device_step=True)
    for gs in steps[1:]:
        load(Gg, gs)
        g.replay()
    torch.cuda.synchronize()
    assert ref.status()[0] == 0 and opt.status()[0] == 0
    for i in range(len(shapes)):
        d_ref = Pe[i].cpu().numpy().astype(np.float64) - theta[i]
        d_got = Pg[i].cpu().numpy().astype(np.float64) - theta[i]
        assert rel(d_got, d_ref) < 1e-5, i
        assert rel(opt.m[i].cpu().numpy(), ref.m[i].cpu().numpy()) < 1e-6, i
        assert rel(opt.v[i].cpu().numpy(), ref.v[i].cpu().numpy()) < 1e-6, i
