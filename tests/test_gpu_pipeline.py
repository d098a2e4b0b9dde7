"""The host-buffer step with overlapped copies against the device-resident step.

Grouping the parameters changes no block's arithmetic (every block is an
independent problem), so after the same steps from the same inputs the
pipelined step's host parameters must equal the device-resident step's
parameters up to the order of the fp32 atomic sums in the per-block Adam
norms.  The device-resident step itself is held to the float64 oracle in
test_gpu_step.py.
"""

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import workloads
from tests.gpu_util import cuda_or_skip

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    return cuda_or_skip()


@pytest.mark.parametrize("groups", [1, 3])
def test_pipelined_host_step_matches_device_step(torch, groups):
    from matrix_inverse_roots_stack_b200 import binding as bd
    from matrix_inverse_roots_stack_b200.pipeline import HostPipelinedShampoo
    shapes = [(300, 200), (128, 520), (5, 7), (256, 256), (130, 129)]
    B = 128
    hp = bd.make_hparams(block_size=B, ndb_iters1=12, ndb_iters2=12)
    v0 = torch.from_numpy(workloads.pi_start_vectors(B, 32, seed=0)).cuda()
    theta = [torch.from_numpy(t.astype(np.float32)) for t in workloads.parameters(shapes, seed=4)]
    steps = [workloads.gaussian_gradients(shapes, std=0.1, seed=10 + s) for s in range(2)]

    # device-resident reference
    P = [t.cuda() for t in theta]
    G = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    ref = bd.Shampoo(P, G, hp=hp, v0=v0)
    for gs in steps:
        for g, x in zip(G, gs):
            g.copy_(torch.from_numpy(x.astype(np.float32)))
        ref.step()
    torch.cuda.synchronize()
    assert ref.status()[0] == 0

    pipe = HostPipelinedShampoo(shapes, hp=hp, v0=v0, groups=groups)
    assert sorted(i for g in pipe.groups for i in g) == list(range(len(shapes)))
    assert len(pipe.groups) == min(groups, len(shapes))
    host_p = [t.clone().pin_memory() for t in theta]
    pipe.load_params(host_p)
    for gs in steps:
        host_g = [torch.from_numpy(x.astype(np.float32)).pin_memory() for x in gs]
        pipe.step(host_g, host_p)
    torch.cuda.synchronize()
    assert pipe.status()[0] == 0

    for i, (hp_i, p_ref, t0) in enumerate(zip(host_p, P, theta)):
        got = hp_i.numpy().astype(np.float64)
        want = p_ref.cpu().numpy().astype(np.float64)
        moved = np.linalg.norm(want - t0.numpy())
        assert moved > 0, i
        # the updates agree to fp32 rounding of the norms' summation order
        assert np.linalg.norm(got - want) <= 1e-5 * moved + 1e-12, (i, np.linalg.norm(got - want), moved)
