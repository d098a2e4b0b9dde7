"""Host-side checks of the C ABI (no GPU needed, no compute calls).

The library must load, export every entry point that include/dash_b200.h
declares, reject bad arguments with the documented codes before touching the
device, and build the same block table as the oracle's blocking.
"""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from matrix_inverse_roots_stack_b200 import binding as bd
from oracle import step as ostep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def declared_names():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if fn.endswith(".h"):
            with open(os.path.join(HEADER_DIR, fn)) as f:
                names |= set(re.findall(r"SHAMPOO_API\s+[\w\s\*]+?\b(shampoo_\w+)\s*\(", f.read()))
    return names


@pytest.fixture(scope="module")
def lib():
    from matrix_inverse_roots_stack_b200 import build
    build.build()
    return bd.load()


def test_exports_every_declared_symbol(lib):
    names = declared_names()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (shampoo_\w+)", out))
    assert names <= exported, names - exported
    assert exported == names, exported - names  # nothing beyond the header is exported
    assert set(bd.exported_names()) == names
    for n in names:
        assert hasattr(lib, n)


def test_no_driver_or_runtime_dependency(lib):
    out = subprocess.run(["ldd", bd.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_strerror(lib):
    assert bd.strerror(0) == "success"
    for code in range(-6, 0):
        assert bd.strerror(code) not in ("", "unknown status code")
    assert bd.strerror(-99) == "unknown status code"


def fake_params(shapes):
    arr = (bd.ShampooParam * len(shapes))()
    for i, (r, c) in enumerate(shapes):
        base = 0x10000000 * (i + 1)  # never dereferenced by the host-only calls
        arr[i] = bd.ShampooParam(r, c, base, base + 0x1000000, base + 0x2000000, base + 0x3000000)
    return arr


def init(lib, shapes, **hp):
    ctx = ctypes.c_void_p()
    nbytes = ctypes.c_size_t()
    h = bd.make_hparams(**hp)
    rc = lib.shampoo_init_blocks(ctypes.byref(ctx), fake_params(shapes), len(shapes), ctypes.byref(h),
                                 ctypes.byref(nbytes))
    return rc, ctx, nbytes.value


@pytest.mark.parametrize("shapes,B", [([(512, 512)], 128), ([(768, 2304), (50257, 768)], 512),
                                      ([(300, 200), (128, 520), (1, 1)], 128)])
def test_block_table_matches_oracle_blocking(lib, shapes, B):
    rc, ctx, nbytes = init(lib, shapes, block_size=B)
    assert rc == 0 and nbytes > 0
    nb, nf, bs = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    assert lib.shampoo_ctx_info(ctx, ctypes.byref(nb), ctypes.byref(nf), ctypes.byref(bs)) == 0
    expect = []
    for p, (r, c) in enumerate(shapes):
        for (r0, r1, c0, c1) in ostep.block_grid(r, c, B):
            expect.append((p, r0, c0, r1 - r0, c1 - c0))
    assert nb.value == len(expect) and nf.value == 2 * len(expect) and bs.value == B
    tab = np.zeros((nb.value, 7), dtype=np.int64)
    assert lib.shampoo_block_table(ctx, tab.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))) == 0
    for k, e in enumerate(expect):
        assert tuple(tab[k, :5]) == e and tab[k, 5] == 2 * k and tab[k, 6] == 2 * k + 1
    lib.shampoo_destroy(ctx)


def test_init_blocks_rejects_bad_arguments(lib):
    assert init(lib, [(4, 4)], block_size=100)[0] == bd.SHAMPOO_EUNSUPPORTED
    assert init(lib, [(4, 4)], block_size=4096)[0] == bd.SHAMPOO_EUNSUPPORTED
    assert init(lib, [(4, 4)], pi_starts=16)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], pi_iters=0)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], beta=1.0)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], ndb_iters1=0)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], cheb_degree=1)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], solver=7)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], root_every=-1)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], scaling=2)[0] == bd.SHAMPOO_EINVAL
    assert init(lib, [(4, 4)], root_every=5, scaling=bd.SCALING_FROBENIUS)[0] == bd.SHAMPOO_OK
    assert init(lib, [(0, 4)])[0] == bd.SHAMPOO_EINVAL
    ctx = ctypes.c_void_p()
    n = ctypes.c_size_t()
    h = bd.make_hparams()
    assert lib.shampoo_init_blocks(None, fake_params([(4, 4)]), 1, ctypes.byref(h), ctypes.byref(n)) == -1
    assert lib.shampoo_init_blocks(ctypes.byref(ctx), fake_params([(4, 4)]), 0, ctypes.byref(h),
                                   ctypes.byref(n)) == -1
    arr = fake_params([(4, 4)])
    arr[0].grad = None
    assert lib.shampoo_init_blocks(ctypes.byref(ctx), arr, 1, ctypes.byref(h), ctypes.byref(n)) == -1


def test_root_calls_validate_before_device_work(lib):
    p = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x100000)
    need = lib.shampoo_inv_root_workspace_bytes(4, 256, 0)
    assert need > 0
    assert lib.shampoo_inv_root_workspace_bytes(0, 256, 0) == 0
    assert lib.shampoo_inv_root_workspace_bytes(4, 200, 0) == 0
    ndb = lib.shampoo_inv_root_newton_db
    assert ndb(None, p, 4, 256, 8, 8, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert ndb(p, p, 4, 200, 8, 8, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EUNSUPPORTED
    assert ndb(p, p, 0, 256, 8, 8, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EUNSUPPORTED
    assert ndb(p, p, 4, 256, 0, 8, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert ndb(p, p, 4, 256, 8, 8, -1.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert ndb(p, p, 4, 256, 8, 8, 0.0, p, -1, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert ndb(p, p, 4, 256, 8, 8, 0.0, p, 101, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert ndb(p, p, 4, 256, 8, 8, 0.0, p, 10, None, None, need, None) == bd.SHAMPOO_EWORKSPACE
    assert ndb(p, p, 4, 256, 8, 8, 0.0, p, 10, None, ws, need - 1, None) == bd.SHAMPOO_EWORKSPACE
    assert ndb(p, p, 4, 256, 8, 8, 0.0, p, 10, None, ctypes.c_void_p(0x100010), need,
               None) == bd.SHAMPOO_EWORKSPACE
    cheb = lib.shampoo_inv_root_chebyshev
    assert cheb(p, p, 4, 256, 1, 1e-3, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert cheb(p, p, 4, 256, 16, 0.0, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EINVAL
    assert cheb(p, p, 4, 384 + 1, 16, 1e-3, 0.0, p, 10, None, ws, need, None) == bd.SHAMPOO_EUNSUPPORTED


def test_step_calls_validate_workspace(lib):
    rc, ctx, nbytes = init(lib, [(256, 256)], block_size=128)
    assert rc == 0
    p = ctypes.c_void_p(0x1000)
    assert lib.shampoo_accumulate(ctx, p, None, nbytes, None) == bd.SHAMPOO_EWORKSPACE
    assert lib.shampoo_accumulate(ctx, p, ctypes.c_void_p(0x100000), nbytes - 1, None) == bd.SHAMPOO_EWORKSPACE
    assert lib.shampoo_accumulate(None, p, ctypes.c_void_p(0x100000), nbytes, None) == bd.SHAMPOO_EINVAL
    assert lib.shampoo_precondition_step(ctx, p, p, 0, None, None, ctypes.c_void_p(0x100000), nbytes,
                                         None) == bd.SHAMPOO_EINVAL
    assert lib.shampoo_precondition_step(ctx, p, None, 1, None, None, ctypes.c_void_p(0x100000), nbytes,
                                         None) == bd.SHAMPOO_EINVAL
    # step 0 continues the device step counter: not before an explicit step on
    # this workspace (the call above returned before setting it), never below 0
    assert lib.shampoo_precondition_step(ctx, p, p, -1, None, None, ctypes.c_void_p(0x100000), nbytes,
                                         None) == bd.SHAMPOO_EINVAL
    lib.shampoo_destroy(ctx)
    lib.shampoo_destroy(None)


def test_header_static_capacity_matches_layout(lib):
    """The capacities the header states for the static scratch are the
    largest stacks whose workspace fits SHAMPOO_STATIC_SCRATCH_BYTES."""
    text = open(os.path.join(HEADER_DIR, "dash_b200.h")).read()
    flat = " ".join(text.split()).replace(" * ", " ")
    m = re.search(r"holds up to (\d+) matrices of 128, (\d+) of 256, (\d+) of 512, (\d+) of 1024", flat)
    assert m, "capacity sentence missing from the header"
    cap = re.search(r"#define SHAMPOO_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    scratch = int(cap.group(1)) << int(cap.group(2))
    assert scratch == bd.STATIC_SCRATCH_BYTES
    for B, stated in zip((128, 256, 512, 1024), map(int, m.groups())):
        fits = lambda n: lib.shampoo_inv_root_workspace_bytes(n, B, bd.SOLVER_NEWTON_DB) <= scratch
        assert fits(stated) and not fits(stated + 1), (B, stated)


def test_header_codes_and_chebyshev_contract():
    text = open(os.path.join(HEADER_DIR, "dash_b200.h")).read()
    codes = dict(re.findall(r"#define (SHAMPOO_E\w+|SHAMPOO_OK) \(?(-?\d+)\)?", text))
    assert {k: int(v) for k, v in codes.items()} == {
        "SHAMPOO_OK": bd.SHAMPOO_OK, "SHAMPOO_EINVAL": bd.SHAMPOO_EINVAL,
        "SHAMPOO_EUNSUPPORTED": bd.SHAMPOO_EUNSUPPORTED, "SHAMPOO_EWORKSPACE": bd.SHAMPOO_EWORKSPACE,
        "SHAMPOO_ECUDA": bd.SHAMPOO_ECUDA, "SHAMPOO_ENONFINITE": bd.SHAMPOO_ENONFINITE,
        "SHAMPOO_ETIMEOUT": bd.SHAMPOO_ETIMEOUT}
    flat = " ".join(text.split()).replace(" * ", " ")
    # the Chebyshev map the kernels and the oracle run: c = 1/(2 lambda),
    # x = c A' + delta I, X = c^(1/4) p(x) ~ (A' + 2 delta lambda I)^(-1/4)
    assert "c = 1/(2 lambda_i)" in flat and "x = c A_i' + delta I" in flat
    assert "X_i = c^(1/4) p(x) ~ (A_i' + 2 delta lambda_i I)^(-1/4)" in flat


def test_get_status_before_any_step(lib):
    rc, ctx, _ = init(lib, [(256, 256)], block_size=128)
    assert rc == 0
    flags = ctypes.c_int(7)
    assert lib.shampoo_get_status(ctx, ctypes.byref(flags)) == bd.SHAMPOO_OK and flags.value == 0
    assert lib.shampoo_get_status(None, ctypes.byref(flags)) == bd.SHAMPOO_EINVAL
    lib.shampoo_destroy(ctx)


def test_profile_read_size(lib):
    # eight timed stages of (ms, count, flops) and three counters: the header,
    # the library and the binding agree on 27 values
    n = 3 * len(bd.PROFILE_STAGES) + 3
    assert n == 27
    text = " ".join(open(os.path.join(HEADER_DIR, "dash_b200.h")).read().split()).replace(" * ", " ")
    assert f"out[0 .. {n - 1}]" in text and f"n >= {n}." in text
    buf = (ctypes.c_double * n)()
    assert lib.shampoo_profile_read(buf, n - 1) == bd.SHAMPOO_EINVAL
    assert lib.shampoo_profile_reset() == 0
    assert lib.shampoo_profile_read(buf, n) == 0
    assert list(buf)[:3 * len(bd.PROFILE_STAGES)] == [0.0] * (3 * len(bd.PROFILE_STAGES))
