"""ctypes binding of libdash_b200.so (argument marshalling only).

Every function named ``shampoo_*`` here forwards to the C entry point of the
same name declared in ``include/dash_b200.h``.  The torch helpers at the end
only allocate device buffers with PyTorch and pass their pointers; all of the
step's arithmetic runs in the library's CUDA kernels.  There is no fallback:
if the shared library is missing the import of this module's users fails.
"""

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdash_b200.so")

SHAMPOO_OK = 0
SHAMPOO_EINVAL = -1
SHAMPOO_EUNSUPPORTED = -2
SHAMPOO_EWORKSPACE = -3
SHAMPOO_ECUDA = -4
SHAMPOO_ENONFINITE = -5
SHAMPOO_ETIMEOUT = -6
SOLVER_NEWTON_DB = 0
SOLVER_CHEBYSHEV = 1
SOLVER_COUPLED_NEWTON = 2
SCALING_SPECTRAL = 0
SCALING_FROBENIUS = 1
PI_STARTS = 32


class ShampooError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {strerror(code)} ({code})")
        self.code = code


class ShampooParam(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("param", ctypes.c_void_p),
                ("grad", ctypes.c_void_p), ("m", ctypes.c_void_p), ("v", ctypes.c_void_p)]


class ShampooHParams(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int), ("beta", ctypes.c_float), ("eps", ctypes.c_float),
                ("init_scale", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("adam_eps", ctypes.c_float), ("lr", ctypes.c_float), ("solver", ctypes.c_int),
                ("ndb_iters1", ctypes.c_int), ("ndb_iters2", ctypes.c_int), ("cheb_degree", ctypes.c_int),
                ("cheb_delta", ctypes.c_float), ("pi_starts", ctypes.c_int), ("pi_iters", ctypes.c_int),
                ("root_every", ctypes.c_int), ("scaling", ctypes.c_int), ("cn_iters", ctypes.c_int),
                ("cn_fp16", ctypes.c_int)]


def make_hparams(block_size=1024, beta=0.95, eps=1e-6, init_scale=1e-6, beta1=0.9, beta2=0.999,
                 adam_eps=1e-8, lr=1e-3, solver=SOLVER_NEWTON_DB, ndb_iters1=14, ndb_iters2=14,
                 cheb_degree=16, cheb_delta=1e-3, pi_starts=PI_STARTS, pi_iters=10, root_every=1,
                 scaling=SCALING_SPECTRAL, cn_iters=16, cn_fp16=0):
    return ShampooHParams(block_size, beta, eps, init_scale, beta1, beta2, adam_eps, lr, solver,
                          ndb_iters1, ndb_iters2, cheb_degree, cheb_delta, pi_starts, pi_iters, root_every,
                          scaling, cn_iters, cn_fp16)


_lib = None

_VP, _SZ, _I, _F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_PROTOS = {
    "shampoo_init_blocks": (_I, [ctypes.POINTER(_VP), ctypes.POINTER(ShampooParam), _I,
                                 ctypes.POINTER(ShampooHParams), ctypes.POINTER(_SZ)]),
    "shampoo_ctx_info": (_I, [_VP, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "shampoo_block_table": (_I, [_VP, ctypes.POINTER(ctypes.c_int64)]),
    "shampoo_init_factors": (_I, [_VP, _VP, _VP]),
    "shampoo_accumulate": (_I, [_VP, _VP, _VP, _SZ, _VP]),
    "shampoo_precondition_step": (_I, [_VP, _VP, _VP, _I, _VP, _VP, _VP, _SZ, _VP]),
    "shampoo_inv_root_newton_db": (_I, [_VP, _VP, _I, _I, _I, _I, _F, _VP, _I, _VP, _VP, _SZ, _VP]),
    "shampoo_inv_root_chebyshev": (_I, [_VP, _VP, _I, _I, _I, _F, _F, _VP, _I, _VP, _VP, _SZ, _VP]),
    "shampoo_inv_root_coupled_newton": (_I, [_VP, _VP, _I, _I, _I, _I, _F, _VP, _I, _VP, _VP, _SZ, _VP]),
    "shampoo_inv_root_workspace_bytes": (_SZ, [_I, _I, _I]),
    "shampoo_read_status": (_I, [_VP, _VP, ctypes.POINTER(ctypes.c_uint)]),
    "shampoo_read_static_status": (_I, [_VP, ctypes.POINTER(ctypes.c_uint)]),
    "shampoo_get_status": (_I, [_VP, ctypes.POINTER(ctypes.c_int)]),
    "shampoo_strerror": (ctypes.c_char_p, [_I]),
    "shampoo_destroy": (None, [_VP]),
    "shampoo_inv_root_newton_db_static": (_I, [_VP, _VP, _I, _I, _I, _I, _F, _VP, _I, _VP, _VP]),
    "shampoo_debug_inject_timeout": (_I, []),
    "shampoo_profile_enable": (_I, [_I]),
    "shampoo_profile_reset": (_I, []),
    "shampoo_profile_read": (_I, [ctypes.POINTER(ctypes.c_double), _I]),
}


def load():
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m matrix_inverse_roots_stack_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def exported_names():
    return sorted(_PROTOS)


def strerror(code):
    return load().shampoo_strerror(int(code)).decode()


def _check(code, where):
    if code != SHAMPOO_OK:
        raise ShampooError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# --------------------------------------------------------------------------
# torch helpers (device memory and streams only)
# --------------------------------------------------------------------------

def _workspace(nbytes, device):
    import torch
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def inv_root_workspace_bytes(n, B, solver=SOLVER_NEWTON_DB):
    return int(load().shampoo_inv_root_workspace_bytes(n, B, solver))


def inv_root_newton_db(A, v0, iters1=14, iters2=14, eps=0.0, pi_iters=10, X=None, lam=None, ws=None,
                       stream=None):
    """X = (A + eps I)^(-1/4) for a (n, B, B) fp32 CUDA stack via the library's
    Newton-DB path.  Returns (X, lambda, ws)."""
    import torch
    n, B = A.shape[0], A.shape[1]
    X = torch.empty_like(A) if X is None else X
    lam = torch.empty(n, dtype=torch.float32, device=A.device) if lam is None else lam
    need = inv_root_workspace_bytes(n, B, SOLVER_NEWTON_DB)
    ws = _workspace(need, A.device) if ws is None else ws
    rc = load().shampoo_inv_root_newton_db(_ptr(A), _ptr(X), n, B, iters1, iters2, eps, _ptr(v0), pi_iters,
                                           _ptr(lam), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "shampoo_inv_root_newton_db")
    return X, lam, ws


def inv_root_chebyshev(A, v0, degree=16, delta=1e-3, eps=0.0, pi_iters=10, X=None, lam=None, ws=None,
                       stream=None):
    """Chebyshev/Clenshaw variant of :func:`inv_root_newton_db`."""
    import torch
    n, B = A.shape[0], A.shape[1]
    X = torch.empty_like(A) if X is None else X
    lam = torch.empty(n, dtype=torch.float32, device=A.device) if lam is None else lam
    need = inv_root_workspace_bytes(n, B, SOLVER_CHEBYSHEV)
    ws = _workspace(need, A.device) if ws is None else ws
    rc = load().shampoo_inv_root_chebyshev(_ptr(A), _ptr(X), n, B, degree, delta, eps, _ptr(v0), pi_iters,
                                           _ptr(lam), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "shampoo_inv_root_chebyshev")
    return X, lam, ws


STATIC_SCRATCH_BYTES = 64 << 20


def inv_root_coupled_newton(A, v0, iters=16, fp16=False, eps=0.0, pi_iters=10, X=None, lam=None, ws=None,
                            stream=None):
    """Coupled-Newton variant of :func:`inv_root_newton_db` (fp16: single-pass
    fp16 products)."""
    import torch
    n, B = A.shape[0], A.shape[1]
    X = torch.empty_like(A) if X is None else X
    lam = torch.empty(n, dtype=torch.float32, device=A.device) if lam is None else lam
    need = inv_root_workspace_bytes(n, B, SOLVER_COUPLED_NEWTON)
    ws = _workspace(need, A.device) if ws is None else ws
    rc = load().shampoo_inv_root_coupled_newton(_ptr(A), _ptr(X), n, B, iters, 1 if fp16 else 0, eps, _ptr(v0),
                                                pi_iters, _ptr(lam), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "shampoo_inv_root_coupled_newton")
    return X, lam, ws


def inv_root_newton_db_static(A, v0, iters1=14, iters2=14, eps=0.0, pi_iters=10, X=None, lam=None, stream=None):
    """:func:`inv_root_newton_db` through the entry point that uses the
    library's fixed scratch instead of a workspace (nothing is allocated by
    the library; X and lambda are allocated here only if not given)."""
    import torch
    n, B = A.shape[0], A.shape[1]
    X = torch.empty_like(A) if X is None else X
    lam = torch.empty(n, dtype=torch.float32, device=A.device) if lam is None else lam
    rc = load().shampoo_inv_root_newton_db_static(_ptr(A), _ptr(X), n, B, iters1, iters2, eps, _ptr(v0), pi_iters,
                                                  _ptr(lam), _stream(stream))
    _check(rc, "shampoo_inv_root_newton_db_static")
    return X, lam


def read_status(ws, stream=None):
    """Synchronise and return (code, flags) of a workspace's status word."""
    flags = ctypes.c_uint(0)
    rc = load().shampoo_read_status(_ptr(ws), _stream(stream), ctypes.byref(flags))
    return rc, flags.value


def read_static_status(stream=None):
    """(code, flags) of the static scratch's status word (after
    :func:`inv_root_newton_db_static`)."""
    flags = ctypes.c_uint(0)
    rc = load().shampoo_read_static_status(_stream(stream), ctypes.byref(flags))
    return rc, flags.value


PROFILE_STAGES = ("gemm", "accumulate", "power_iteration", "solver", "precondition", "adam_update", "gemm_wide",
                  "ndb_fused")


def profile_enable(on=True):
    _check(load().shampoo_profile_enable(1 if on else 0), "shampoo_profile_enable")


def profile_reset():
    _check(load().shampoo_profile_reset(), "shampoo_profile_reset")


def profile_read():
    """Return {stage: (ms, count, flops)}, plus "launches" and "dropped"."""
    n = 3 * len(PROFILE_STAGES) + 3
    buf = (ctypes.c_double * n)()
    _check(load().shampoo_profile_read(buf, n), "shampoo_profile_read")
    out = {s: (buf[3 * i], int(buf[3 * i + 1]), buf[3 * i + 2]) for i, s in enumerate(PROFILE_STAGES)}
    out["launches"] = int(buf[n - 3])
    out["dropped"] = int(buf[n - 2])
    out["wide_regs"] = int(buf[n - 1])
    return out


class Shampoo:
    """Batched block-Shampoo optimizer state over a list of CUDA fp32
    parameter/gradient tensors.  The factor stack, Adam moments and
    workspace are torch allocations; every step runs in the library."""

    def __init__(self, params, grads, hp=None, v0=None, m=None, v=None):
        import torch
        self.hp = hp if hp is not None else make_hparams()
        self.params, self.grads = list(params), list(grads)
        dev = self.params[0].device
        self.m = m if m is not None else [torch.zeros_like(p) for p in self.params]
        self.v = v if v is not None else [torch.zeros_like(p) for p in self.params]
        for t in self.params + self.grads + self.m + self.v:
            if t.dtype != torch.float32 or not t.is_contiguous() or t.dim() != 2 or not t.is_cuda:
                raise ValueError("parameters, gradients and moments must be contiguous 2-D fp32 CUDA tensors")
        arr = (ShampooParam * len(self.params))()
        for i, (p, g, m_, v_) in enumerate(zip(self.params, self.grads, self.m, self.v)):
            arr[i] = ShampooParam(p.shape[0], p.shape[1], p.data_ptr(), g.data_ptr(), m_.data_ptr(),
                                  v_.data_ptr())
        ctx = ctypes.c_void_p()
        nbytes = ctypes.c_size_t(0)
        _check(load().shampoo_init_blocks(ctypes.byref(ctx), arr, len(self.params), ctypes.byref(self.hp),
                                          ctypes.byref(nbytes)), "shampoo_init_blocks")
        self._ctx = ctx
        nb, nf, B = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        load().shampoo_ctx_info(ctx, ctypes.byref(nb), ctypes.byref(nf), ctypes.byref(B))
        self.n_blocks, self.n_factors, self.B = nb.value, nf.value, B.value
        self.ws = _workspace(nbytes.value, dev)
        self.factors = torch.empty((self.n_factors, self.B, self.B), dtype=torch.float32, device=dev)
        if v0 is None:
            from .workloads import pi_start_vectors
            v0 = torch.from_numpy(pi_start_vectors(self.B, PI_STARTS, seed=0)).to(dev)
        self.v0 = v0
        self.lam = torch.empty(self.n_factors, dtype=torch.float32, device=dev)
        self.t = 0
        _check(load().shampoo_init_factors(ctx, _ptr(self.factors), _stream(None)), "shampoo_init_factors")

    def block_table(self):
        import numpy as np
        out = np.zeros((self.n_blocks, 7), dtype=np.int64)
        _check(load().shampoo_block_table(self._ctx, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))),
               "shampoo_block_table")
        return out

    def accumulate(self, stream=None):
        _check(load().shampoo_accumulate(self._ctx, _ptr(self.factors), _ptr(self.ws), self.ws.numel(),
                                         _stream(stream)), "shampoo_accumulate")

    def precondition_step(self, roots_out=None, stream=None, device_step=False):
        """device_step: take the step number from the counter on the device
        (for steps captured into a CUDA graph; needs an earlier eager step)."""
        self.t += 1
        _check(load().shampoo_precondition_step(self._ctx, _ptr(self.factors), _ptr(self.v0),
                                                0 if device_step else self.t,
                                                _ptr(self.lam), _ptr(roots_out), _ptr(self.ws),
                                                self.ws.numel(), _stream(stream)),
               "shampoo_precondition_step")

    def step(self, roots_out=None, stream=None, device_step=False):
        """One full step: factor EMA, roots, precondition, Adam graft, update."""
        self.accumulate(stream)
        self.precondition_step(roots_out, stream, device_step)

    def status(self, stream=None):
        return read_status(self.ws, stream)

    def get_status(self):
        """(code, flags) of the last step call's workspace, on the stream it
        was given (the library remembers both)."""
        flags = ctypes.c_int(0)
        rc = load().shampoo_get_status(self._ctx, ctypes.byref(flags))
        return rc, flags.value

    def __del__(self):
        ctx = getattr(self, "_ctx", None)
        if ctx is not None and _lib is not None:
            _lib.shampoo_destroy(ctx)
            self._ctx = None
