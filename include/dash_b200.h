/*
 * dash_b200.h -- C ABI of the batched block-Shampoo (DASH-style) step on one
 * NVIDIA B200 (sm_100a).
 *
 * Source of the method: "DASH: Faster Shampoo via Batched Block
 * Preconditioning and Efficient Inverse-Root Solvers" (howistudyai.com
 * explainer of arXiv 2602.02016), sections "Building blocks", "High-level
 * flow" and "Step-by-step".  Each entry point below names the passage that
 * defines the operation it performs.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers marked (device) are CUDA device pointers, (host) are host
 *    pointers.  All device buffers are owned by the caller; the library never
 *    allocates, frees or retains device memory.  A shampoo_ctx holds only
 *    host-side metadata.
 *  - Matrices are fp32, row-major.  A "stack" is n contiguous B x B matrices,
 *    layout (n, B, B).  Input matrices to the root solvers must be symmetric;
 *    symmetry is assumed, not checked.
 *  - B (the block size) must be a multiple of 128 in [128, 2048].
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Device work is enqueued on it asynchronously; no call
 *    synchronises except the three status readers (shampoo_read_status,
 *    shampoo_get_status, shampoo_read_static_status).
 *  - `ws` is a caller-owned device workspace of at least the size the
 *    matching *_workspace_bytes call reports, 256-byte aligned.  Its first
 *    word is a status word that every call clears when it starts and that the
 *    kernels set when they see a non-finite value or give up a bounded wait;
 *    read it with shampoo_read_status after the call.
 *  - Power iteration uses caller-supplied start vectors `v0` (device, fp32,
 *    B x 32 row-major: column j is start vector j).  A factor of true size
 *    b < B uses rows 0..b-1.  Its products run on the tensor cores with
 *    split-fp16 operands: each A + eps I is first scaled by the power of two
 *    2^-e with 2^(e-1) <= its largest diagonal entry < 2^e, which keeps every
 *    entry of a positive semi-definite matrix within [-1, 1] (exact scaling;
 *    lambda is returned unscaled).  A matrix with an entry beyond 65504 * 2^e
 *    (not positive semi-definite) sets the status word's non-finite bit.
 *  - Return value: 0 on success or a negative SHAMPOO_E* code.  No C++
 *    exception crosses this boundary.  On an error return nothing has been
 *    enqueued unless the code is SHAMPOO_ECUDA.
 *  - A ctx is not thread-safe; use one ctx per stream.
 *  - CUDA graphs: after a first call on a device (which sets the kernels'
 *    shared-memory limits), the standalone root calls make only stream-
 *    ordered CUDA calls, so a call can be captured and replayed with new
 *    inputs in the same buffers.  So can a full step (shampoo_accumulate +
 *    shampoo_precondition_step with step = 0, which takes its step number
 *    from a counter on the device), after one eager step on the same ws.
 */
#ifndef DASH_B200_H
#define DASH_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SHAMPOO_API __attribute__((visibility("default")))
#else
#define SHAMPOO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define SHAMPOO_OK 0
#define SHAMPOO_EINVAL (-1)       /* null pointer, bad count or hyper-parameter */
#define SHAMPOO_EUNSUPPORTED (-2) /* B not a multiple of 128, B > 2048, n < 1, ... */
#define SHAMPOO_EWORKSPACE (-3)   /* workspace missing, too small or misaligned */
#define SHAMPOO_ECUDA (-4)        /* a CUDA launch or runtime call failed */
#define SHAMPOO_ENONFINITE (-5)   /* (read_status) a kernel produced Inf/NaN */
#define SHAMPOO_ETIMEOUT (-6)     /* (read_status) a bounded device wait gave up */

#define SHAMPOO_SOLVER_NEWTON_DB 0
#define SHAMPOO_SOLVER_CHEBYSHEV 1
#define SHAMPOO_SOLVER_COUPLED_NEWTON 2

/* Scale estimate lambda each factor is divided by (c = 1 / (2 lambda)) before
 * the root solver ("Building blocks", scaling): the multi-start power
 * iteration's spectral estimate, or the Frobenius norm ||F + eps I||_F. */
#define SHAMPOO_SCALING_SPECTRAL 0
#define SHAMPOO_SCALING_FROBENIUS 1

/* Bits of the workspace status word. */
#define SHAMPOO_STATUS_NONFINITE 1u
#define SHAMPOO_STATUS_TIMEOUT 2u

typedef struct shampoo_ctx shampoo_ctx;

/* One parameter matrix of the model (all device pointers, rows x cols fp32
 * row-major, caller-owned).  `param`, `m`, `v` are updated in place by
 * shampoo_precondition_step; `grad` is read by shampoo_accumulate and
 * shampoo_precondition_step. */
typedef struct {
  int64_t rows, cols;
  float* param;
  const float* grad;
  float* m; /* Adam first moment */
  float* v; /* Adam second moment */
} shampoo_param;

/* Hyper-parameters (names follow the pages' notation). */
typedef struct {
  int block_size;   /* B */
  float beta;       /* factor EMA: L <- beta L + (1-beta) G G^T */
  float eps;        /* regulariser added at root time: L + eps I */
  float init_scale; /* initial factors init_scale * I (see shampoo_init_factors) */
  float beta1, beta2, adam_eps, lr; /* Adam graft and step size */
  int solver;       /* SHAMPOO_SOLVER_* */
  int ndb_iters1;   /* Newton-DB iterations, first stage (>= 1) */
  int ndb_iters2;   /* Newton-DB iterations, second stage on Y (>= 1) */
  int cheb_degree;  /* Chebyshev degree d, 2..256 */
  float cheb_delta; /* Chebyshev interval [delta, 1 + delta] */
  int pi_starts;    /* power-iteration start vectors K; must be 32 */
  int pi_iters;     /* power-iteration products, 1..100 */
  int root_every;   /* roots recomputed every root_every-th step (steps 1, 1 + f, ...);
                       other steps reuse the roots kept in the workspace (0 or 1: every step) */
  int scaling;      /* SHAMPOO_SCALING_* */
  int cn_iters;     /* coupled-Newton iterations, 0..1000 */
  int cn_fp16;      /* 1: coupled Newton with single-pass fp16 products (0: fp32-level split products) */
} shampoo_hparams;

/* Build the block table for a parameter set (host only; no device work).
 * Each rows x cols parameter is cut at multiples of B into blocks (edge
 * blocks smaller), as in "Step-by-step", step "Split into blocks and stack".
 * Block k (parameter order, row-major inside a parameter) owns factors 2k (L,
 * size b_r) and 2k+1 (R, size b_c); every factor is stored zero-padded to
 * B x B in the caller's factor stack (n_factors, B, B).
 * `params`: host array of n_params descriptors (copied).  `hp` (host, copied).
 * `workspace_bytes` (host out): bytes of `ws` the step calls need.
 * Errors: SHAMPOO_EINVAL (null pointer, n_params < 1, a dimension < 1, bad
 * hyper-parameter), SHAMPOO_EUNSUPPORTED (B). */
SHAMPOO_API int shampoo_init_blocks(shampoo_ctx** out, const shampoo_param* params, int n_params, const shampoo_hparams* hp,
                        size_t* workspace_bytes);

/* Counts of a ctx (host out pointers may be NULL). */
SHAMPOO_API int shampoo_ctx_info(const shampoo_ctx* ctx, int* n_blocks, int* n_factors, int* block_size);

/* Copy the block table to host memory: n_blocks rows of 7 int64 values
 * (param index, row0, col0, b_r, b_c, L factor index, R factor index). */
SHAMPOO_API int shampoo_block_table(const shampoo_ctx* ctx, int64_t* out_host);

/* Write init_scale * I into every factor of the (n_factors, B, B) device
 * stack (padding rows/columns included); the pages' initial state. */
SHAMPOO_API int shampoo_init_factors(shampoo_ctx* ctx, float* factors, void* stream);

/* Factor statistics ("Step-by-step", step "Build preconditioners"):
 * gathers every gradient block into the workspace (zero-padded to B) and
 * updates the factor stack in place,
 *     L_k <- beta L_k + (1-beta) G_k G_k^T,  R_k <- beta R_k + (1-beta) G_k^T G_k.
 * `factors` (device, (n_factors, B, B) fp32).  The gathered blocks stay in
 * `ws` for the following shampoo_precondition_step of the same step. */
SHAMPOO_API int shampoo_accumulate(shampoo_ctx* ctx, float* factors, void* ws, size_t ws_bytes, void* stream);

/* Root computation, preconditioning, Adam graft and update ("High-level
 * flow" after the EMA; "Step-by-step" steps "Scale each block",
 * "Compute inverse roots", "Grafting with Adam's magnitude", "Apply update"):
 *   for every factor F: A = F + eps I; lambda = power iteration on A from v0;
 *   X = A^(-1/4) by the configured solver (Newton-DB, Chebyshev or coupled Newton, as for the
 *   standalone calls below); then per block U = X_L G X_R; Adam moments
 *   m, v (bias-corrected with `step` >= 1); P = m_hat / (sqrt(v_hat) + adam_eps);
 *   s = ||P_b||_F / ||U_b||_F (0 when U_b = 0); param -= lr * s * U_b.
 * Requires shampoo_accumulate on the same ws earlier in the same step.
 * Roots are computed on root steps, (step - 1) % root_every == 0, and on any
 * step whose ws does not hold this ctx's roots yet; other steps precondition
 * with the roots kept in ws since the last root step (the factors, moments
 * and parameters are still updated every step), and leave lambda_out and
 * roots_out untouched.
 * `step` >= 1 is the step number; it also sets a step counter kept in ws.
 * `step` = 0 continues that counter on the device (t = previous t + 1), so
 * that a captured step can be replayed from a CUDA graph; it requires
 * root_every <= 1 (roots every step) and an earlier call with an explicit
 * step on the same ws, else SHAMPOO_EINVAL.  step < 0: SHAMPOO_EINVAL.
 * `lambda_out` (device, n_factors floats, or NULL) receives the estimates.
 * `roots_out` (device, (n_factors, B, B) fp32, or NULL) receives X. */
SHAMPOO_API int shampoo_precondition_step(shampoo_ctx* ctx, const float* factors, const float* v0, int step,
                              float* lambda_out, float* roots_out, void* ws, size_t ws_bytes, void* stream);

/* Standalone inverse fourth roots of a stack, Newton-DB solver
 * ("Building blocks", Newton-DB; "Building blocks", spectral scaling and
 * Multi-Power-Iteration):
 *   A_i' = A_i + eps I;  lambda_i = power iteration (pi_iters products, the
 *   32 starts of v0, max Rayleigh quotient);  c = 1/(2 lambda_i);
 *   stage 1: Y = c A_i', Z = I, iters1 times E = (3I - ZY)/2, Y <- YE, Z <- EZ;
 *   stage 2: the same from Y = Y(stage 1), Z = I, iters2 times;
 *   X_i = c^(1/4) Z  ~  (A_i + eps I)^(-1/4).
 * pi_iters = 0 selects Frobenius scaling instead: lambda_i = ||A_i'||_F (v0 is
 * then not read but must still be a valid pointer).
 * A (device, (n, B, B) fp32, symmetric, read only), X (device, (n, B, B) fp32,
 * written), lambda_out (device, n floats, or NULL).
 * Errors: SHAMPOO_EINVAL, SHAMPOO_EUNSUPPORTED, SHAMPOO_EWORKSPACE, SHAMPOO_ECUDA. */
SHAMPOO_API int shampoo_inv_root_newton_db(const float* A, float* X, int n, int B, int iters1, int iters2, float eps,
                               const float* v0, int pi_iters, float* lambda_out, void* ws, size_t ws_bytes,
                               void* stream);

/* Standalone inverse fourth roots of a stack, Chebyshev solver ("Building
 * blocks", Chebyshev; "Step-by-step", solver (d)): A_i' = A_i + eps I;
 * lambda_i as for the Newton-DB call; the common spectral scaling
 * c = 1/(2 lambda_i) of "Step-by-step" maps the spectrum of A_i' into
 * [delta, 1 + delta] by x = c A_i' + delta I (t = 2 c A_i' - I on [-1, 1]);
 * p of degree `degree` interpolates x^(-1/4) at the first-kind Chebyshev
 * nodes of [delta, 1 + delta] (fitted on the host in double precision); p is
 * evaluated with the matrix Clenshaw recurrence in t; X_i = c^(1/4) p(x)
 * ~ (A_i' + 2 delta lambda_i I)^(-1/4).  Arguments as for the Newton-DB call. */
SHAMPOO_API int shampoo_inv_root_chebyshev(const float* A, float* X, int n, int B, int degree, float delta, float eps,
                               const float* v0, int pi_iters, float* lambda_out, void* ws, size_t ws_bytes,
                               void* stream);

/* Standalone inverse fourth roots of a stack, coupled-Newton solver
 * ("Building blocks", Coupled-Newton; "Scoreboard": CN in FP16):
 *   A_i' = A_i + eps I;  lambda_i as for the Newton-DB call;  c = 1/(2 lambda_i);
 *   M = c A_i', X = I;  `iters` times: C = (5I - M)/4, X <- X C, M <- C^4 M;
 *   X_i = c^(1/4) X  ~  (A_i + eps I)^(-1/4).
 * fp16 = 1 computes every product in one pass of fp16 operands with fp32
 * accumulation (the pages' fast mode); fp16 = 0 uses the split-fp16 products
 * of the other solvers (about fp32 accuracy).  Other arguments as for the
 * Newton-DB call. */
SHAMPOO_API int shampoo_inv_root_coupled_newton(const float* A, float* X, int n, int B, int iters, int fp16,
                                                float eps, const float* v0, int pi_iters, float* lambda_out,
                                                void* ws, size_t ws_bytes, void* stream);

/* Variant of shampoo_inv_root_newton_db that allocates nothing and needs no
 * workspace from the caller.  The paper has no counterpart: this exists for
 * callers that cannot call cudaMalloc -- e.g. a plug-in running inside a host
 * framework that owns every device allocation, or a latency-critical path
 * where an allocation (which may synchronise the device) is not allowed.
 *
 * The scratch is a fixed array of SHAMPOO_STATIC_SCRATCH_BYTES in the
 * library's device global memory; every GPU that loads the library holds it
 * until the process exits.  Problems whose workspace
 * (shampoo_inv_root_workspace_bytes(n, B, SHAMPOO_SOLVER_NEWTON_DB)) exceeds it
 * are rejected with SHAMPOO_EWORKSPACE (it holds up to 161 matrices of 128,
 * 46 of 256, 12 of 512, 3 of 1024).  The caller still passes A, X, v0 and lambda_out (device
 * pointers, as for shampoo_inv_root_newton_db); the computation and the
 * results are the same.
 *
 * Every call looks up the scratch's device address with the caller's device
 * current (an address kept across calls could go stale if the device's
 * context were torn down); the first call on a device also loads the
 * library's device code there, so make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents (each call clears what must start at zero), so calls whose GPU work
 * overlaps -- on different streams, or from different threads -- race on it:
 * serialise them.  The status word (non-finite values, a bounded wait that
 * gave up) lives in the scratch too; each call clears it, and
 * shampoo_read_static_status reads it.
 * Errors: as shampoo_inv_root_newton_db, plus SHAMPOO_EWORKSPACE when the
 * problem does not fit the scratch. */
#define SHAMPOO_STATIC_SCRATCH_BYTES (64u << 20)
SHAMPOO_API int shampoo_inv_root_newton_db_static(const float* A, float* X, int n, int B, int iters1, int iters2,
                                                  float eps, const float* v0, int pi_iters, float* lambda_out,
                                                  void* stream);

/* Status word of the static scratch after shampoo_inv_root_newton_db_static
 * (no counterpart in the paper): synchronises `stream`, reads the word into
 * *flags (host, may be NULL) and returns as shampoo_read_status does.  It
 * reports the last static call whose work has finished on this device. */
SHAMPOO_API int shampoo_read_static_status(void* stream, unsigned* flags);

/* Workspace bytes for a standalone root call on n matrices of size B. */
SHAMPOO_API size_t shampoo_inv_root_workspace_bytes(int n, int B, int solver);

/* Synchronise `stream`, read the status word of `ws` into *flags (host, may
 * be NULL) and return SHAMPOO_OK, SHAMPOO_ETIMEOUT (checked first: a wait
 * that gave up leaves later results undefined) or SHAMPOO_ENONFINITE. */
SHAMPOO_API int shampoo_read_status(const void* ws, void* stream, unsigned* flags);

/* Status of a ctx's last step: synchronises the stream that the last
 * shampoo_accumulate or shampoo_precondition_step on `ctx` was given, reads
 * the status word of that call's workspace into *device_flags (host, may be
 * NULL; SHAMPOO_STATUS_* bits) and returns as shampoo_read_status does.
 * Before any step call it reports 0 and SHAMPOO_OK. */
SHAMPOO_API int shampoo_get_status(shampoo_ctx* ctx, int* device_flags);

/* Static description of a status code. */
SHAMPOO_API const char* shampoo_strerror(int code);

/* Kernel-time accounting for benchmarking (host side; off by default; not
 * part of the method).  While enabled the library records a CUDA event pair,
 * on the launching stream, around every launch of its tensor-core GEMM kernel
 * and around each stage of the calls above, and counts every kernel it
 * launches.  The events are created on first use and reused; no device
 * memory is allocated. */
SHAMPOO_API int shampoo_profile_enable(int enable);
/* Forget everything recorded so far. */
SHAMPOO_API int shampoo_profile_reset(void);
/* Synchronise the recorded events and fill out[0 .. 26]:
 * out[3s], out[3s+1], out[3s+2] = milliseconds, count and flops of stage s,
 * for s = 0 launches of the tensor-core GEMM with 128 x 128 tiles (executed
 * tensor-core flops: 3 * 2*128*128*B per computed tile, or 1 * ... for
 * single-pass fp16 launches), 1 gather + factor EMA, 2 power iteration,
 * 3 root solver, 4 preconditioner products, 5 Adam graft + update, 6 launches
 * of the tensor-core GEMM with 128 x 256 tiles (3 * 2*128*256*B per tile), 7
 * launches of the Newton-DB kernel on resident factors of 128 (9 * 2*128^3
 * per iteration and factor);
 * out[24] = kernel launches since the last reset; out[25] = records dropped;
 * out[26] = registers a thread of the 128 x 256 kernel was compiled with (it
 * is used only when that is 168, the count its register split assumes).
 * n >= 27. */
SHAMPOO_API int shampoo_profile_read(double* out, int n);

/* Test hook for the failure path (not part of the method): arms a one-shot
 * fault so that the next launch of a tensor-core product kernel (the GEMM,
 * or Newton-DB on resident factors of 128) withholds its operand loads.  Its bounded waits then expire (about 2 s), the kernel sets
 * SHAMPOO_STATUS_TIMEOUT in the workspace status word, releases its tensor
 * memory and returns; the context stays usable.  The results of that call
 * are undefined. */
SHAMPOO_API int shampoo_debug_inject_timeout(void);

/* Free a ctx (host memory only).  NULL is ignored. */
SHAMPOO_API void shampoo_destroy(shampoo_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* DASH_B200_H */
