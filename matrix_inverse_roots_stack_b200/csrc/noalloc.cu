// Newton-DB inverse fourth roots with library-owned scratch, for callers that
// cannot allocate device memory themselves (see shampoo_inv_root_newton_db_static
// in include/dash_b200.h).
#include <cuda_runtime.h>

#include "dash_b200.h"

namespace dash {
int inv_root_with_scratch(const float* A, float* X, int n, int B, float eps, const float* v0, int pi_iters, void* ws,
                          size_t ws_bytes, int solver, int it1, int it2, int degree, float delta, float* lambda_out,
                          void* stream);
int read_status_word(const void* ws, void* stream, unsigned* flags);
}

namespace {

// The scratch every call of the entry point works in.  It lives in the
// module's global memory, so each GPU that loads this library keeps it
// (SHAMPOO_STATIC_SCRATCH_BYTES) until the process exits.  In host code this
// name is only a host-side stand-in: kernels are given the device address
// obtained below.  The root layout puts the status word at offset 0.
__device__ __align__(256) unsigned char g_static_scratch[SHAMPOO_STATIC_SCRATCH_BYTES];

// Device address of the scratch on the current device.  It is looked up on
// every call, with the caller's device current: an address kept from an
// earlier call could be stale after the device's context was torn down and
// the module loaded again.  The first call on a device also loads the module.
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SHAMPOO_ECUDA;
  *out = p;
  return SHAMPOO_OK;
}

}  // namespace

extern "C" {

SHAMPOO_API int shampoo_inv_root_newton_db_static(const float* A, float* X, int n, int B, int iters1, int iters2,
                                                  float eps, const float* v0, int pi_iters, float* lambda_out,
                                                  void* stream) {
  if (!A || !X || !v0) return SHAMPOO_EINVAL;
  if (iters1 < 1 || iters2 < 1 || iters1 > 1000 || iters2 > 1000) return SHAMPOO_EINVAL;
  const size_t need = shampoo_inv_root_workspace_bytes(n, B, SHAMPOO_SOLVER_NEWTON_DB);
  if (need == 0) return SHAMPOO_EUNSUPPORTED;
  if (need > SHAMPOO_STATIC_SCRATCH_BYTES) return SHAMPOO_EWORKSPACE;  // problem larger than the scratch
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc) return rc;
  return dash::inv_root_with_scratch(A, X, n, B, eps, v0, pi_iters, ws, SHAMPOO_STATIC_SCRATCH_BYTES,
                                     SHAMPOO_SOLVER_NEWTON_DB, iters1, iters2, 0, 0.0f, lambda_out, stream);
}

SHAMPOO_API int shampoo_read_static_status(void* stream, unsigned* flags) {
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc) return rc;
  return dash::read_status_word(ws, stream, flags);
}

}  // extern "C"
