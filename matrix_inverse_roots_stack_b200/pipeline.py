"""Block-Shampoo step with host-resident gradients and parameters, the copies
overlapped with the device work.

When gradients arrive in pinned host memory and the updated parameters go
back to it, a step is upload -> step -> download, and done one after the
other the two copies add their full PCIe time to the step.  Here the
parameters are split into ``groups`` sets balanced by root cost (the greedy
rule of :func:`distributed.partition`), each with its own library context.
Per step the gradient uploads run on one copy stream, each group's step on
the compute stream as soon as its gradients have landed, and each group's
parameter download on a second copy stream as soon as its update is done.
Only the first group's upload and the last group's download are left
outside the tensor-core work.  Every block is an independent problem, so the
grouping does not change the arithmetic of any block.
"""

from typing import List, Sequence

from . import binding
from .distributed import partition


def parameter_groups(shapes: Sequence[Sequence[int]], B: int, groups: int) -> List[List[int]]:
    """Indices of the parameters in each group: at most ``groups`` non-empty
    groups balanced by root cost (greedy, as the multi-GPU ownership), each
    in increasing index order."""
    if groups < 1:
        raise ValueError("groups must be positive")
    if not shapes:
        return []
    owner = partition(shapes, B, min(groups, len(shapes)))
    return [g for g in ([i for i, o in enumerate(owner) if o == k] for k in range(max(owner) + 1)) if g]


class HostPipelinedShampoo:
    """``shapes``: the (rows, cols) of every parameter.  Device copies of the
    parameters, gradients and moments are allocated here; ``load_params``
    sets the parameters, ``step(host_grads, host_params)`` runs one step."""

    def __init__(self, shapes: Sequence[Sequence[int]], hp=None, v0=None, device="cuda", groups: int = 4):
        import torch
        self.hp = hp if hp is not None else binding.make_hparams()
        B = self.hp.block_size
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.params = [torch.zeros(s, dtype=torch.float32, device=device) for s in self.shapes]
        self.grads = [torch.zeros(s, dtype=torch.float32, device=device) for s in self.shapes]
        self.groups = parameter_groups(self.shapes, B, groups)
        self.opts = [binding.Shampoo([self.params[i] for i in g], [self.grads[i] for i in g], hp=self.hp, v0=v0)
                     for g in self.groups]
        dev = self.params[0].device
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.n_factors = sum(o.n_factors for o in self.opts)

    def load_params(self, host_params):
        for p, h in zip(self.params, host_params):
            p.copy_(h)

    def step(self, host_grads, host_params, stream=None):
        """One step: ``host_grads`` (pinned fp32, the parameters' shapes) in,
        the updated parameters out into ``host_params`` (pinned fp32).  The
        work is queued on ``stream`` (default: the current stream) and two
        copy streams; everything is ordered before later work on ``stream``,
        so synchronising it makes ``host_params`` valid."""
        import torch
        comp = stream if stream is not None else torch.cuda.current_stream(self.params[0].device)
        # the previous step's use of the device gradients and parameters is done
        self.h2d.wait_stream(comp)
        self.d2h.wait_stream(comp)
        landed = []
        with torch.cuda.stream(self.h2d):
            for g in self.groups:
                for i in g:
                    self.grads[i].copy_(host_grads[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.h2d)
                landed.append(ev)
        for g, opt, ev in zip(self.groups, self.opts, landed):
            comp.wait_event(ev)
            opt.step(stream=comp)
            done = torch.cuda.Event()
            done.record(comp)
            self.d2h.wait_event(done)
            with torch.cuda.stream(self.d2h):
                for i in g:
                    host_params[i].copy_(self.params[i], non_blocking=True)
        comp.wait_stream(self.d2h)
        comp.wait_stream(self.h2d)

    def status(self):
        """First non-zero status over the groups, with its device flags."""
        for o in self.opts:
            rc, flags = o.status()
            if rc != 0:
                return rc, flags
        return 0, 0
