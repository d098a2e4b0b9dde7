"""Multi-GPU block Shampoo: greedy ownership of parameters and one all-gather.

DASH explainer, "High-level flow" (the last step: load-balance across GPUs and
sync): every Shampoo block is an independent problem, so each GPU owns a
share of the parameters, runs the whole step (factor EMA, roots,
preconditioning, Adam graft, update) for the blocks of the parameters it
owns, and the updated parameters are then exchanged so that every GPU holds
all of them.  Ownership is decided once, greedily: parameters in decreasing
order of root cost (sum of b^3 over their factors) each go to the currently
least-loaded rank.

One process per GPU, ``torch.distributed`` for the exchange: NCCL over
NVLink on GPUs (one all-gather of the owned parameters packed into equal-size
buffers per step), gloo on CPU for the tests.  The local step is any object
with ``step()`` built by ``make_local`` from the owned parameters and
gradients -- by default the library's :class:`binding.Shampoo`.
"""

from typing import Callable, List, Optional, Sequence, Tuple


def block_sizes(rows: int, cols: int, B: int) -> List[Tuple[int, int]]:
    """(b_r, b_c) of every block of a rows x cols parameter cut at multiples of B."""
    rs = [min(B, rows - r0) for r0 in range(0, rows, B)]
    cs = [min(B, cols - c0) for c0 in range(0, cols, B)]
    return [(br, bc) for br in rs for bc in cs]


def root_cost(shape: Sequence[int], B: int) -> int:
    """Root work of one parameter per step: sum of b^3 over its L and R factors."""
    return sum(br ** 3 + bc ** 3 for br, bc in block_sizes(int(shape[0]), int(shape[1]), B))


def partition(shapes: Sequence[Sequence[int]], B: int, world: int) -> List[int]:
    """Owner rank of every parameter: longest-processing-time-first greedy.

    Parameters are taken in decreasing root cost (ties by index) and each is
    given to the rank with the least cost so far (ties to the lowest rank).
    Deterministic, so every rank computes the same table.
    """
    if world < 1:
        raise ValueError("world size must be positive")
    costs = [root_cost(s, B) for s in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-costs[i], i))
    load = [0] * world
    owner = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += costs[i]
    return owner


class ShardedShampoo:
    """Block Shampoo over ``torch.distributed`` ranks with greedy ownership.

    ``params``, ``grads``: the full list of parameter / gradient tensors, the
    same on every rank (data-parallel replicas; gradients already averaged).
    Each rank steps the parameters it owns and :meth:`sync` all-gathers the
    updated parameters.  ``make_local(owned_params, owned_grads)`` builds the
    local optimizer (called only when the rank owns something).
    """

    def __init__(self, params, grads, block_size: int, make_local: Optional[Callable] = None, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.params = list(params)
        self.grads = list(grads)
        self.owner = partition([tuple(p.shape) for p in self.params], block_size, self.world)
        self.owned = [i for i, r in enumerate(self.owner) if r == self.rank]
        if make_local is None:
            from . import binding
            make_local = lambda ps, gs: binding.Shampoo(ps, gs, hp=binding.make_hparams(block_size=block_size))
        self.local = make_local([self.params[i] for i in self.owned],
                                [self.grads[i] for i in self.owned]) if self.owned else None
        # pack layout: rank r's owned parameters, flattened, in index order
        self.numel = [[self.params[i].numel() for i, o in enumerate(self.owner) if o == r] for r in range(self.world)]
        self.span = max([sum(n) for n in self.numel] + [1])
        p0 = self.params[0]
        self.send = p0.new_empty(self.span)
        self.recv = [p0.new_empty(self.span) for _ in range(self.world)]

    def step(self):
        """Local step on the owned parameters, then the exchange."""
        if self.local is not None:
            self.local.step()
        self.sync()

    def sync(self):
        """All-gather the owned parameters so every rank holds all of them."""
        if self.world == 1:
            return
        off = 0
        for i in self.owned:
            n = self.params[i].numel()
            self.send[off:off + n].copy_(self.params[i].reshape(-1))
            off += n
        self.dist.all_gather(self.recv, self.send, group=self.group)
        for r in range(self.world):
            if r == self.rank:
                continue
            off = 0
            for i, o in enumerate(self.owner):
                if o != r:
                    continue
                n = self.params[i].numel()
                self.params[i].reshape(-1).copy_(self.recv[r][off:off + n])
                off += n
