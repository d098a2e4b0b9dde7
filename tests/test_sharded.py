"""Greedy ownership and the parameter exchange of the multi-GPU step, on CPU.

The exchange logic is tested with two gloo ranks: each rank steps the
parameters it owns with the float64 oracle (standing in for the library's
local step, which needs a GPU), the all-gather distributes the results, and
every rank must then hold exactly what one process stepping all parameters
computes.
"""

import os
import socket

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import distributed as sd
from matrix_inverse_roots_stack_b200 import workloads


def test_block_sizes_cover_the_parameter():
    for (r, c, B) in [(300, 200, 128), (50257, 768, 512), (5, 7, 3), (1024, 1024, 1024)]:
        bs = sd.block_sizes(r, c, B)
        assert sum(br * bc for br, bc in bs) == r * c
        assert all(0 < br <= B and 0 < bc <= B for br, bc in bs)


def test_partition_is_a_balanced_deterministic_assignment():
    shapes = workloads.llama_1b_shapes()
    B = 1024
    costs = [sd.root_cost(s, B) for s in shapes]
    for world in (1, 2, 3, 8):
        owner = sd.partition(shapes, B, world)
        assert owner == sd.partition(shapes, B, world)
        assert len(owner) == len(shapes) and all(0 <= o < world for o in owner)
        load = [sum(c for c, o in zip(costs, owner) if o == r) for r in range(world)]
        # list-scheduling bound: no rank exceeds the mean by more than one item
        assert max(load) <= sum(costs) / world + max(costs)
        if world <= len(shapes):
            assert min(load) > 0
    assert sd.partition([(4, 4)], 128, 3) == [0]
    with pytest.raises(ValueError):
        sd.partition([(4, 4)], 128, 0)


def test_pipeline_groups_cover_every_parameter_once():
    from matrix_inverse_roots_stack_b200.pipeline import parameter_groups
    shapes = workloads.llama_1b_shapes()
    for groups in (1, 2, 4, 8):
        gs = parameter_groups(shapes, 1024, groups)
        assert len(gs) == groups and all(gs)
        assert sorted(i for g in gs for i in g) == list(range(len(shapes)))
        assert all(g == sorted(g) for g in gs)
        # balanced by root cost like the multi-GPU ownership
        load = [sum(sd.root_cost(shapes[i], 1024) for i in g) for g in gs]
        assert max(load) <= sum(load) / groups + max(sd.root_cost(s, 1024) for s in shapes)
    # two parameters, five groups asked: two groups, the costlier parameter first
    assert parameter_groups([(4, 4), (8, 8)], 128, 5) == [[1], [0]]
    assert parameter_groups([], 128, 3) == []
    with pytest.raises(ValueError):
        parameter_groups([(4, 4)], 128, 0)


def test_partition_greedy_order_small_case():
    # costs (B = 4): 4x4 -> 2*64 = 128, 8x4 -> 2*(64+64) = 256, 2x2 -> 16
    shapes = [(4, 4), (8, 4), (2, 2), (4, 4)]
    assert sd.partition(shapes, 4, 2) == [1, 0, 0, 1]


class OracleLocal:
    """Local step on CPU float64 tensors with the oracle (test stand-in)."""

    def __init__(self, params, grads, hp, V0):
        from oracle import step as ostep
        self.ostep, self.hp, self.V0 = ostep, hp, V0
        self.params, self.grads = params, grads
        self.state = ostep.init_state([tuple(p.shape) for p in params], hp)

    def step(self):
        th = [p.numpy() for p in self.params]
        g = [x.numpy() for x in self.grads]
        new, self.state, _ = self.ostep.shampoo_step(th, g, self.state, self.hp, self.V0)
        for p, n in zip(self.params, new):
            p.copy_(__import__("torch").from_numpy(n))


def _shapes():
    return [(40, 24), (16, 16), (33, 7), (24, 40), (8, 70)]


def _inputs(step):
    shapes = _shapes()
    th = workloads.parameters(shapes, seed=31)
    gs = workloads.gaussian_gradients(shapes, std=0.1, seed=40 + step)
    return shapes, th, gs


def _rank_main(rank, world, port, out_path):
    import torch
    import torch.distributed as dist
    from oracle import step as ostep
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        hp = ostep.HParams(block_size=16, ndb_iters1=10, ndb_iters2=10)
        V0 = workloads.pi_start_vectors(16, 32, seed=0)
        shapes, th, _ = _inputs(0)
        params = [torch.from_numpy(t.astype(np.float64)) for t in th]
        grads = [torch.zeros(s, dtype=torch.float64) for s in shapes]
        opt = sd.ShardedShampoo(params, grads, 16, make_local=lambda ps, gs: OracleLocal(ps, gs, hp, V0))
        for s in range(2):
            _, _, gs = _inputs(s)
            for g, x in zip(grads, gs):
                g.copy_(torch.from_numpy(x.astype(np.float64)))
            opt.step()
        np.savez(out_path + f".{rank}.npz", owner=np.array(opt.owner), *[p.numpy() for p in params])
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_match_one_process(tmp_path):
    import torch.multiprocessing as mp
    from oracle import step as ostep
    world = 2
    out = str(tmp_path / "res")
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    # reference: one process steps all parameters
    hp = ostep.HParams(block_size=16, ndb_iters1=10, ndb_iters2=10)
    V0 = workloads.pi_start_vectors(16, 32, seed=0)
    shapes, th, _ = _inputs(0)
    state = ostep.init_state(shapes, hp)
    cur = [t.astype(np.float64) for t in th]
    for s in range(2):
        _, _, gs = _inputs(s)
        cur, state, _ = ostep.shampoo_step(cur, [g.astype(np.float64) for g in gs], state, hp, V0)
    res = [np.load(out + f".{r}.npz") for r in range(world)]
    owner = res[0]["owner"]
    assert set(owner.tolist()) == {0, 1}  # both ranks own something
    assert np.array_equal(owner, res[1]["owner"])
    for r in range(world):
        for i, ref in enumerate(cur):
            got = res[r][f"arr_{i}"]
            assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref)), (r, i)
