"""Helpers shared by the GPU parity tests."""

import numpy as np


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def cuda_or_skip():
    import pytest
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_inverse_roots_stack_b200 import build
    build.build()
    return torch


def assert_mirrored_blocks(torch, F, tile=128, chunk=256):
    """Off-diagonal 128-column blocks of a symmetric launch's output.

    A symmetric launch computes the tiles that reach the upper triangle and
    writes each block above the diagonal twice, directly and transposed, so
    block (j, i) is block (i, j) transposed bit for bit.  Diagonal blocks are
    computed in full and are not compared.  F: an (n, B, B) tensor.
    """
    n, B, _ = F.shape
    blk = torch.arange(B, device=F.device) // tile
    off = blk[:, None] != blk[None, :]
    for s in range(0, n, chunk):
        Fc = F[s:s + chunk]
        assert torch.equal(Fc[:, off], Fc.transpose(1, 2)[:, off]), f"factors {s}..{s + Fc.shape[0]}"
