// C ABI of the batched block-Shampoo step (declared in include/dash_b200.h).
//
// Host-side orchestration only: argument checks, the block table, workspace
// planning, Chebyshev coefficients, and the stream-ordered sequence of kernel
// launches.  All arithmetic of the step runs in the kernels of gemm.cu and
// kernels.cu.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "dash_b200.h"
#include "gemm.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "ptx.cuh"

using dash::BlockDesc;
using dash::GemmArgs;
using dash::ParamDev;

namespace dash {
int read_status_word(const void* ws, void* stream, unsigned* flags);
}

namespace {

constexpr float kZScale = 16.0f;  // Newton-DB Z is stored divided by this (fp16 range headroom)
constexpr size_t kSolverBudget = 32ull << 30;  // bytes of solver scratch per chunk of factors

size_t align256(size_t x) { return (x + 255u) & ~static_cast<size_t>(255u); }

size_t split_bytes(size_t nmat, int B) { return nmat * 2u * static_cast<size_t>(B) * B * sizeof(__half); }

struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  }
};

// Split matrices of solver scratch per factor: Newton-DB 5 (Y and Z
// ping-pong, D), Chebyshev 4 (T and the Clenshaw ring), coupled Newton 6 (M
// and X ping-pong, C^2, C^4).  Chunks of factors keep it within kSolverBudget.
int solver_mats(int solver) {
  return solver == SHAMPOO_SOLVER_COUPLED_NEWTON ? 6 : solver == SHAMPOO_SOLVER_CHEBYSHEV ? 4 : 5;
}
int solver_chunk(int nf, int B, int solver) {
  const size_t per = solver_mats(solver) * split_bytes(1, B);
  size_t m = kSolverBudget / per;
  if (m < 1) m = 1;
  return static_cast<int>(m < static_cast<size_t>(nf) ? m : nf);
}

// Workspace of the root solvers for nf factors of size B.
struct RootLayout {
  size_t status, lam, xscale, pscale, stats, w0, w1, vt, solver;
  int chunk;
};

void plan_roots(Bump& b, RootLayout& L, int nf, int B, int pi_iters, int extra_mats, int solver) {
  L.status = b.take(256);
  L.lam = b.take(sizeof(float) * nf);
  L.xscale = b.take(sizeof(float) * nf);
  L.stats = b.take(sizeof(float) * static_cast<size_t>(pi_iters) * nf * 3 * dash::kPiStarts);
  L.w0 = b.take(sizeof(float) * static_cast<size_t>(nf) * B * dash::kPiStarts);
  L.w1 = b.take(sizeof(float) * static_cast<size_t>(nf) * B * dash::kPiStarts);
  L.pscale = b.take(sizeof(float) * nf);
  L.vt = b.take(2 * sizeof(__half) * static_cast<size_t>(nf) * B * dash::kPiStarts);
  L.chunk = solver_chunk(nf, B, solver);
  const int per = solver_mats(solver);
  // the solver scratch also holds the split factors during the power iteration
  int mats = per * L.chunk > extra_mats ? per * L.chunk : extra_mats;
  if (mats < nf) mats = nf;
  L.solver = b.take(split_bytes(mats, B));
}

bool valid_B(int B) { return B >= 128 && B <= 2048 && B % 128 == 0; }

#define DASH_TRY(expr)                                  \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return SHAMPOO_ECUDA;        \
  } while (0)

#define DASH_LAUNCHED()                                 \
  do {                                                  \
    if (cudaGetLastError() != cudaSuccess) return SHAMPOO_ECUDA; \
  } while (0)

// Chebyshev interpolant of x^(-1/4) on [delta, 1 + delta] at the degree+1
// first-kind nodes, convention f ~ c0/2 + sum_k c_k T_k (double precision).
std::vector<double> cheb_coeffs(int degree, double delta) {
  const int n = degree + 1;
  const double pi = 3.14159265358979323846;
  std::vector<double> fx(n), c(n);
  for (int j = 0; j < n; ++j) {
    const double th = pi * (j + 0.5) / n;
    const double x = delta + 0.5 * (1.0 + std::cos(th));
    fx[j] = std::pow(x, -0.25);
  }
  for (int k = 0; k < n; ++k) {
    double s = 0.0;
    for (int j = 0; j < n; ++j) s += fx[j] * std::cos(pi * k * (j + 0.5) / n);
    c[k] = 2.0 * s / n;
  }
  return c;
}

__half* split_at(char* ws, size_t off, size_t mat, int B) {
  return reinterpret_cast<__half*>(ws + off) + mat * 2u * static_cast<size_t>(B) * B;
}

GemmArgs gemm_args(int B, int sym, unsigned* status) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.B = B;
  g.sym = sym;
  g.nops = 1;
  g.status = status;
  return g;
}

// Newton-DB on one chunk of n factors ("Building blocks", Newton-DB:
// Y0 = A, Z0 = I; E = (3I - ZY)/2; Y <- YE; Z <- EZ; chained twice).  The
// products keep the page's order (Y times E on the right, E times Z on the
// left): in finite precision that is the stable form of the coupled
// iteration, while symmetrising an iterate or moving Z's factor to the other
// side makes a perturbation mode grow once the condition number exceeds ~10.
// Every product is therefore a full (non-symmetric) product of the iterates in
// their natural layout (the GEMM reads the right factor MN-major).  E = I + D
// is applied in correction form Y + Y D, Z + D Z.  Z is stored divided by
// kZScale.  Scratch: Y x2, Z x2 (ping-pong), D: 5 split matrices per factor.
int run_ndb_chunk(const float* F, int n, int B, float eps, const int* fsize, const float* lam, float* xscale,
                  int it1, int it2, float* X_f32, __half* X_split, __half* S, unsigned* status,
                  cudaStream_t st) {
  const size_t m = static_cast<size_t>(n) * 2 * B * B;  // halves per buffer of n matrices
  __half* Yb[2] = {S, S + m};
  __half* Zb[2] = {S + 2 * m, S + 3 * m};
  __half* D = S + 4 * m;
  int yc = 0, zc = 0;
  dash::launch_ndb_init(F, n, B, eps, fsize, lam, kZScale, Yb[0], D, Zb[0], xscale, st);
  DASH_LAUNCHED();

  // Y <- Y + Y D  (A = Y, B = D)
  auto y_op = [&](GemmArgs& g, dash::OpBuffers* ob, int slot) {
    dash::GemmOp& o = g.op[slot];
    o.nprob = n;
    o.b_mn = 1;
    o.alpha = 1.0f;
    o.beta = 1.0f;
    o.cin_split = Yb[yc];
    o.out_split = Yb[yc ^ 1];
    ob[slot] = {Yb[yc], n, D, n};
  };
  // Z <- Z + D Z  (A = D, B = Z)
  auto z_op = [&](GemmArgs& g, dash::OpBuffers* ob, int slot) {
    dash::GemmOp& o = g.op[slot];
    o.nprob = n;
    o.b_mn = 1;
    o.alpha = 1.0f;
    o.beta = 1.0f;
    o.cin_split = Zb[zc];
    o.out_split = Zb[zc ^ 1];
    ob[slot] = {D, n, Zb[zc], n};
  };
  auto first_y = [&]() -> int {
    GemmArgs g = gemm_args(B, 0, status);
    dash::OpBuffers ob[2];
    y_op(g, ob, 0);
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
    yc ^= 1;
    return SHAMPOO_OK;
  };
  auto iterate = [&](int it0, int T, bool final_stage) -> int {
    for (int it = it0; it < T; ++it) {
      {  // D = (I - zs Zhat Y)/2   (A = Zhat, B = Y)
        GemmArgs g = gemm_args(B, 0, status);
        dash::GemmOp& o = g.op[0];
        o.nprob = n;
        o.b_mn = 1;
        o.alpha = -0.5f * kZScale;
        o.gamma = 0.5f;
        o.out_split = D;
        dash::OpBuffers ob[2] = {{Zb[zc], n, Yb[yc], n}, {Zb[zc], n, Yb[yc], n}};
        DASH_TRY(dash::launch_gemm_split(ob, g, st));
      }
      const bool last = (it == T - 1);
      GemmArgs g = gemm_args(B, 0, status);
      dash::OpBuffers ob[2];
      if (!last) {  // both updates in one launch
        y_op(g, ob, 0);
        z_op(g, ob, 1);
        g.nops = 2;
        DASH_TRY(dash::launch_gemm_split(ob, g, st));
        yc ^= 1;
        zc ^= 1;
      } else if (!final_stage) {  // only Y is carried into stage 2
        y_op(g, ob, 0);
        DASH_TRY(dash::launch_gemm_split(ob, g, st));
        yc ^= 1;
      } else {  // X = c^(1/4) zs (Zhat + D Zhat)
        z_op(g, ob, 0);
        dash::GemmOp& o = g.op[0];
        o.out_split = X_split;
        o.out_f32 = X_f32;
        o.scale = xscale;
        o.split_norm = 1;
        DASH_TRY(dash::launch_gemm_split(ob, g, st));
      }
    }
    return SHAMPOO_OK;
  };

  // at B = 128 a factor's iterates fit in one SM's shared memory: a stage's
  // iterations up to its last run there, in place on Y and Zhat
  const bool resident = B == 128;
  const float alpha_d = -0.5f * kZScale;
  int rc = SHAMPOO_OK;
  if (resident) {
    DASH_TRY(dash::launch_ndb_fused(Yb[yc], Zb[zc], D, n, B, alpha_d, 1, it1 >= 2 ? it1 - 2 : 0, it1 >= 2 ? 1 : 0,
                                    status, st));
  } else {
    rc = first_y();
    if (rc) return rc;
    rc = iterate(1, it1, false);
    if (rc) return rc;
  }
  // stage 2 on Y: D0 = (I - Y)/2, Zhat1 = (I + D0)/zs, Y1 = Y + Y D0
  dash::launch_ndb_stage2_init(Yb[yc], n, B, kZScale, D, Zb[zc], st);
  DASH_LAUNCHED();
  if (it2 == 1) {
    dash::launch_scale_split(Zb[zc], n, B, xscale, X_f32, X_split, st);
    DASH_LAUNCHED();
    return SHAMPOO_OK;
  }
  if (resident) {
    DASH_TRY(dash::launch_ndb_fused(Yb[yc], Zb[zc], D, n, B, alpha_d, 1, it2 - 2, 0, status, st));
    return iterate(it2 - 1, it2, true);
  }
  rc = first_y();
  if (rc) return rc;
  return iterate(1, it2, true);
}

// Chebyshev / Clenshaw on one chunk ("Building blocks", Chebyshev; the
// spectral scaling of "Step-by-step" precedes the solver): T = 2c A - I with
// c = 1/(2 lambda); b_k = c_k I + 2 T b_{k+1} - b_{k+2}; X = c^(1/4) (c0/2 I +
// T b1 - b2).  All iterates are polynomials in T; the Clenshaw recurrence is
// stable under symmetrisation, so only upper-triangle tiles are computed.
int run_cheb_chunk(const float* F, int n, int B, float eps, const int* fsize, const float* lam, float* xscale,
                   int d, const std::vector<double>& c, float* X_f32, __half* X_split, __half* S,
                   unsigned* status, cudaStream_t st) {
  const size_t m = static_cast<size_t>(n) * 2 * B * B;
  __half* T = S;
  __half* ring = S + m;  // 3 n matrices: b_k lives in slot k % 3
  auto slot = [&](int k) { return (k % 3) * n; };
  dash::launch_cheb_init(F, n, B, eps, fsize, lam, static_cast<float>(c[d - 1]), static_cast<float>(c[d]), T,
                         ring + static_cast<size_t>(slot(d - 1)) * 2 * B * B, xscale, st);
  DASH_LAUNCHED();
  dash::OpBuffers ob[2] = {{T, n, ring, 3 * n}, {T, n, ring, 3 * n}};
  auto base = [&]() {
    GemmArgs g = gemm_args(B, 1, status);
    g.op[0].nprob = n;
    return g;
  };
  if (d == 2) {
    GemmArgs g = base();
    dash::GemmOp& o = g.op[0];
    o.b.base = slot(1);
    o.alpha = 1.0f;
    o.gamma = static_cast<float>(0.5 * c[0] - c[2]);
    o.scale = xscale;
    o.split_norm = 1;
    o.out_f32 = X_f32;
    o.out_split = X_split;
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
    return SHAMPOO_OK;
  }
  {  // b_{d-2} = 2 T b_{d-1} + (c_{d-2} - c_d) I   (b_d = c_d I)
    GemmArgs g = base();
    dash::GemmOp& o = g.op[0];
    o.b.base = slot(d - 1);
    o.alpha = 2.0f;
    o.gamma = static_cast<float>(c[d - 2] - c[d]);
    o.out_split = ring;
    o.out_i.base = slot(d - 2);
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
  }
  for (int k = d - 3; k >= 1; --k) {  // b_k = c_k I + 2 T b_{k+1} - b_{k+2}
    GemmArgs g = base();
    dash::GemmOp& o = g.op[0];
    o.b.base = slot(k + 1);
    o.alpha = 2.0f;
    o.beta = -1.0f;
    o.cin_split = ring;
    o.cin_i.base = slot(k + 2);
    o.gamma = static_cast<float>(c[k]);
    o.out_split = ring;
    o.out_i.base = slot(k);
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
  }
  {  // X = c^(1/4) (c0/2 I + T b1 - b2)
    GemmArgs g = base();
    dash::GemmOp& o = g.op[0];
    o.b.base = slot(1);
    o.alpha = 1.0f;
    o.beta = -1.0f;
    o.cin_split = ring;
    o.cin_i.base = slot(2);
    o.gamma = static_cast<float>(0.5 * c[0]);
    o.scale = xscale;
    o.split_norm = 1;
    o.out_f32 = X_f32;
    o.out_split = X_split;
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
  }
  return SHAMPOO_OK;
}

// Coupled Newton on one chunk of n factors ("Building blocks", Coupled-Newton:
// C_k from M_k; X_{k+1} = X_k C_k; M_{k+1} = C_k^p M_k; C_k = (5I - M_k)/4 for
// p = 4).  Every iterate is a polynomial in A, so each product is symmetric
// and computed on upper-triangle tiles (mirrored); the iteration for M is a
// function of M alone, so symmetrising it is harmless.  Per iteration:
//   C^2 = (M M - 10 M + 25 I)/16;  C^4 = C^2 C^2;
//   M' = C^4 M  and  X' = (5 X - X M)/4  (one launch, both read the old M);
// the last iteration needs only X'.  fp16: single-pass fp16 products.
int run_cn_chunk(const float* F, int n, int B, float eps, const int* fsize, const float* lam, float* xscale,
                 int iters, int fp16, float* X_f32, __half* X_split, __half* S, unsigned* status,
                 cudaStream_t st) {
  const size_t m = static_cast<size_t>(n) * 2 * B * B;
  __half* Mb[2] = {S, S + m};
  __half* Xb[2] = {S + 2 * m, S + 3 * m};
  __half* C2 = S + 4 * m;
  __half* C4 = S + 5 * m;
  int mc = 0, xc = 0;
  dash::launch_cn_init(F, n, B, eps, fsize, lam, Mb[0], Xb[0], xscale, st);
  DASH_LAUNCHED();
  if (iters == 0) {
    dash::launch_scale_split(Xb[0], n, B, xscale, X_f32, X_split, st);
    DASH_LAUNCHED();
    return SHAMPOO_OK;
  }
  auto base = [&]() {
    GemmArgs g = gemm_args(B, 1, status);
    g.single_pass = fp16 ? 1 : 0;
    g.op[0].nprob = n;
    return g;
  };
  for (int it = 0; it < iters; ++it) {
    const bool last = it == iters - 1;
    if (!last) {
      {  // C^2 = M M / 16 - (10/16) M + (25/16) I
        GemmArgs g = base();
        dash::GemmOp& o = g.op[0];
        o.alpha = 1.0f / 16.0f;
        o.beta = -10.0f / 16.0f;
        o.cin_split = Mb[mc];
        o.gamma = 25.0f / 16.0f;
        o.out_split = C2;
        dash::OpBuffers ob[2] = {{Mb[mc], n, Mb[mc], n}, {Mb[mc], n, Mb[mc], n}};
        DASH_TRY(dash::launch_gemm_split(ob, g, st));
      }
      {  // C^4 = C^2 C^2
        GemmArgs g = base();
        dash::GemmOp& o = g.op[0];
        o.alpha = 1.0f;
        o.out_split = C4;
        dash::OpBuffers ob[2] = {{C2, n, C2, n}, {C2, n, C2, n}};
        DASH_TRY(dash::launch_gemm_split(ob, g, st));
      }
    }
    GemmArgs g = base();
    dash::OpBuffers ob[2];
    int xo = 0;
    if (!last) {  // M' = C^4 M
      dash::GemmOp& o = g.op[0];
      o.alpha = 1.0f;
      o.out_split = Mb[mc ^ 1];
      ob[0] = {C4, n, Mb[mc], n};
      g.op[1].nprob = n;
      g.nops = 2;
      xo = 1;
    }
    {  // X' = (5 X - X M)/4, scaled by c^(1/4) into the outputs on the last iteration
      dash::GemmOp& o = g.op[xo];
      o.alpha = -0.25f;
      o.beta = 1.25f;
      o.cin_split = Xb[xc];
      if (last) {
        o.out_split = X_split;
        o.out_f32 = X_f32;
        o.scale = xscale;
        o.split_norm = 1;
      } else {
        o.out_split = Xb[xc ^ 1];
      }
      ob[xo] = {Xb[xc], n, Mb[mc], n};
    }
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
    mc ^= 1;
    xc ^= 1;
  }
  return SHAMPOO_OK;
}

// Power iteration (pi_iters > 0) or Frobenius norm (pi_iters == 0) + solver
// on nf factors.  Writes X as fp32 (X_f32) and/or split (X_split).  fsize
// (device) gives each factor's true size or is null.  it1, it2: the Newton-DB
// stage iterations, or for the coupled Newton its iterations and fp16 flag.
int run_roots(const float* F, int nf, int B, float eps, const int* fsize, const float* v0, int pi_iters, int solver,
              int it1, int it2, int degree, float delta, float* lam_out, float* X_f32, __half* X_split, char* ws,
              const RootLayout& L, unsigned* status, cudaStream_t st) {
  float* lam = reinterpret_cast<float*>(ws + L.lam);
  float* xscale = reinterpret_cast<float*>(ws + L.xscale);
  float* stats = reinterpret_cast<float*>(ws + L.stats);
  float* W[2] = {reinterpret_cast<float*>(ws + L.w0), reinterpret_cast<float*>(ws + L.w1)};
  const size_t sstride = static_cast<size_t>(nf) * 3 * dash::kPiStarts;

  const int pslot = dash::prof_begin(dash::kProfPowerIter, st);
  if (pi_iters == 0) {  // Frobenius scaling: lambda = ||F + eps I||_F
    dash::launch_frob_norm(F, nf, B, eps, fsize, lam, lam_out, st);
    DASH_LAUNCHED();
  } else {  // multi-start power iteration ("Building blocks", Multi-Power-Iteration)
    // the split factors live in the solver scratch until the solver starts
    __half* As = reinterpret_cast<__half*>(ws + L.solver);
    __half* Vt = reinterpret_cast<__half*>(ws + L.vt);
    float* pscale = reinterpret_cast<float*>(ws + L.pscale);
    DASH_TRY(cudaMemsetAsync(stats, 0, sizeof(float) * sstride * pi_iters, st));
    dash::launch_pi_prepare(F, nf, B, eps, fsize, pscale, As, status, st);
    DASH_LAUNCHED();
    for (int t = 0; t < pi_iters; ++t) {
      const float* Wp = t ? W[(t - 1) & 1] : nullptr;
      const float* sp = t ? stats + (t - 1) * sstride : nullptr;
      dash::launch_pi_vectors(v0, Wp, sp, nf, B, fsize, Vt, st);
      DASH_LAUNCHED();
      DASH_TRY(dash::launch_pi_product(As, Vt, v0, Wp, sp, nf, B, fsize, W[t & 1], stats + t * sstride, status, st));
    }
    dash::launch_pi_finalize(stats + (pi_iters - 1) * sstride, nf, pscale, lam, lam_out, st);
    DASH_LAUNCHED();
  }
  dash::prof_end(pslot, st);

  const int sslot = dash::prof_begin(dash::kProfSolver, st);
  std::vector<double> c;
  if (solver == SHAMPOO_SOLVER_CHEBYSHEV) c = cheb_coeffs(degree, delta);
  __half* S = reinterpret_cast<__half*>(ws + L.solver);
  const size_t BB = static_cast<size_t>(B) * B;
  for (int f0 = 0; f0 < nf; f0 += L.chunk) {
    const int n = (nf - f0 < L.chunk) ? nf - f0 : L.chunk;
    const float* Fc = F + f0 * BB;
    const int* fs = fsize ? fsize + f0 : nullptr;
    float* Xf = X_f32 ? X_f32 + f0 * BB : nullptr;
    __half* Xs = X_split ? X_split + f0 * 2 * BB : nullptr;
    const int rc =
        (solver == SHAMPOO_SOLVER_NEWTON_DB)
            ? run_ndb_chunk(Fc, n, B, eps, fs, lam + f0, xscale + f0, it1, it2, Xf, Xs, S, status, st)
        : (solver == SHAMPOO_SOLVER_COUPLED_NEWTON)
            ? run_cn_chunk(Fc, n, B, eps, fs, lam + f0, xscale + f0, it1, it2, Xf, Xs, S, status, st)
            : run_cheb_chunk(Fc, n, B, eps, fs, lam + f0, xscale + f0, degree, c, Xf, Xs, S, status, st);
    if (rc) {
      dash::prof_end(sslot, st);
      return rc;
    }
  }
  dash::prof_end(sslot, st);
  return SHAMPOO_OK;
}

bool finite_nonneg(float x) { return std::isfinite(x) && x >= 0.0f; }

int check_ws(const void* ws, size_t have, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || have < need) return SHAMPOO_EWORKSPACE;
  return SHAMPOO_OK;
}

}  // namespace

// ============================================================ context

struct shampoo_ctx {
  int B = 0;
  shampoo_hparams hp{};
  std::vector<shampoo_param> params;
  std::vector<BlockDesc> blocks;
  std::vector<int> fsize;
  std::vector<ParamDev> pdev;
  std::vector<long long> prefix;
  long long n_items = 0, total_elems = 0;
  int n_blocks = 0, n_factors = 0;
  RootLayout roots{};
  size_t off_gs = 0, off_roots = 0, off_u = 0, off_pn = 0, off_un = 0, off_blocks = 0, off_params = 0,
         off_prefix = 0, off_fsize = 0, off_step = 0, off_gmax = 0, off_fscale2 = 0, off_bscale = 0, off_uscale = 0, total = 0;
  const void* tables_ws = nullptr;
  const void* roots_ws = nullptr;  // workspace holding the roots of the last root step
  const void* step_ws = nullptr;   // workspace whose step counter an explicit step has set
  const void* last_ws = nullptr;   // workspace and stream of the last step call (shampoo_get_status)
  void* last_stream = nullptr;
};

namespace {

int upload_tables(shampoo_ctx* c, char* ws, cudaStream_t st) {
  if (c->tables_ws == ws) return SHAMPOO_OK;
  DASH_TRY(cudaMemcpyAsync(ws + c->off_blocks, c->blocks.data(), sizeof(BlockDesc) * c->blocks.size(),
                           cudaMemcpyHostToDevice, st));
  DASH_TRY(cudaMemcpyAsync(ws + c->off_params, c->pdev.data(), sizeof(ParamDev) * c->pdev.size(),
                           cudaMemcpyHostToDevice, st));
  DASH_TRY(cudaMemcpyAsync(ws + c->off_prefix, c->prefix.data(), sizeof(long long) * c->prefix.size(),
                           cudaMemcpyHostToDevice, st));
  DASH_TRY(cudaMemcpyAsync(ws + c->off_fsize, c->fsize.data(), sizeof(int) * c->fsize.size(),
                           cudaMemcpyHostToDevice, st));
  c->tables_ws = ws;
  return SHAMPOO_OK;
}

int check_hparams(const shampoo_hparams* hp) {
  if (!hp) return SHAMPOO_EINVAL;
  if (!valid_B(hp->block_size)) return SHAMPOO_EUNSUPPORTED;
  if (!(hp->beta >= 0.0f && hp->beta < 1.0f) || !finite_nonneg(hp->eps) || !finite_nonneg(hp->init_scale))
    return SHAMPOO_EINVAL;
  if (!(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
      !finite_nonneg(hp->adam_eps) || !std::isfinite(hp->lr))
    return SHAMPOO_EINVAL;
  if (hp->solver != SHAMPOO_SOLVER_NEWTON_DB && hp->solver != SHAMPOO_SOLVER_CHEBYSHEV &&
      hp->solver != SHAMPOO_SOLVER_COUPLED_NEWTON)
    return SHAMPOO_EINVAL;
  if (hp->cn_iters < 0 || hp->cn_iters > 1000 || (hp->cn_fp16 != 0 && hp->cn_fp16 != 1)) return SHAMPOO_EINVAL;
  if (hp->ndb_iters1 < 1 || hp->ndb_iters2 < 1 || hp->ndb_iters1 > 1000 || hp->ndb_iters2 > 1000)
    return SHAMPOO_EINVAL;
  if (hp->cheb_degree < 2 || hp->cheb_degree > 256 || !(hp->cheb_delta > 0.0f) || !std::isfinite(hp->cheb_delta))
    return SHAMPOO_EINVAL;
  if (hp->pi_starts != dash::kPiStarts || hp->pi_iters < 1 || hp->pi_iters > 100) return SHAMPOO_EINVAL;
  if (hp->root_every < 0 || (hp->scaling != SHAMPOO_SCALING_SPECTRAL && hp->scaling != SHAMPOO_SCALING_FROBENIUS))
    return SHAMPOO_EINVAL;
  return SHAMPOO_OK;
}

}  // namespace

extern "C" {

int shampoo_init_blocks(shampoo_ctx** out, const shampoo_param* params, int n_params, const shampoo_hparams* hp,
                        size_t* workspace_bytes) {
  if (!out || !params || n_params < 1 || !workspace_bytes) return SHAMPOO_EINVAL;
  *out = nullptr;
  const int rc = check_hparams(hp);
  if (rc) return rc;
  const int B = hp->block_size;
  for (int p = 0; p < n_params; ++p) {
    const shampoo_param& q = params[p];
    if (q.rows < 1 || q.cols < 1 || q.rows > (1ll << 31) - 1 || q.cols > (1ll << 31) - 1) return SHAMPOO_EINVAL;
    if (!q.param || !q.grad || !q.m || !q.v) return SHAMPOO_EINVAL;
  }
  shampoo_ctx* c = new (std::nothrow) shampoo_ctx();
  if (!c) return SHAMPOO_EINVAL;
  c->B = B;
  c->hp = *hp;
  c->params.assign(params, params + n_params);
  long long uoff = 0, items = 0;
  for (int p = 0; p < n_params; ++p) {
    const shampoo_param& q = params[p];
    // each parameter's slice of the flat U buffer starts on 16 bytes, so the
    // float4 path of the update reads it aligned whatever the sizes before it
    uoff = (uoff + 3) & ~3ll;
    ParamDev d;
    d.grad = q.grad;
    d.param = q.param;
    d.m = q.m;
    d.v = q.v;
    d.uoff = uoff;
    d.item_base = items;
    d.rows = static_cast<int>(q.rows);
    d.cols = static_cast<int>(q.cols);
    d.blk_base = static_cast<int>(c->blocks.size());
    d.ncb = static_cast<int>((q.cols + B - 1) / B);
    d.chunks = static_cast<int>((q.cols + 1023) / 1024);
    const bool al = ((reinterpret_cast<uintptr_t>(q.grad) | reinterpret_cast<uintptr_t>(q.param) |
                      reinterpret_cast<uintptr_t>(q.m) | reinterpret_cast<uintptr_t>(q.v)) & 15u) == 0;
    d.vec = (q.cols % 4 == 0 && al) ? 1 : 0;
    for (long long r0 = 0; r0 < q.rows; r0 += B)
      for (long long c0 = 0; c0 < q.cols; c0 += B) {
        BlockDesc b;
        b.off = uoff;
        b.pitch = static_cast<int>(q.cols);
        b.r0 = static_cast<int>(r0);
        b.c0 = static_cast<int>(c0);
        b.br = static_cast<int>(std::min<long long>(B, q.rows - r0));
        b.bc = static_cast<int>(std::min<long long>(B, q.cols - c0));
        b.param = p;
        c->blocks.push_back(b);
        c->fsize.push_back(b.br);
        c->fsize.push_back(b.bc);
      }
    c->pdev.push_back(d);
    c->prefix.push_back(items);
    uoff += q.rows * q.cols;
    items += ((q.rows + dash::kUpdRows - 1) / dash::kUpdRows) * static_cast<long long>(d.chunks);
  }
  c->prefix.push_back(items);
  c->n_items = items;
  c->total_elems = uoff;
  c->n_blocks = static_cast<int>(c->blocks.size());
  c->n_factors = 2 * c->n_blocks;
  if (c->n_factors > 65535 || items > 0x7fffffffll) {
    delete c;
    return SHAMPOO_EUNSUPPORTED;
  }
  Bump b;
  plan_roots(b, c->roots, c->n_factors, B, hp->pi_iters, c->n_blocks, hp->solver);
  c->off_gs = b.take(split_bytes(c->n_factors, B));
  c->off_roots = b.take(split_bytes(c->n_factors, B));
  c->off_u = b.take(sizeof(float) * static_cast<size_t>(c->total_elems));
  c->off_pn = b.take(sizeof(float) * c->n_blocks);
  c->off_un = b.take(sizeof(float) * c->n_blocks);
  c->off_blocks = b.take(sizeof(BlockDesc) * c->n_blocks);
  c->off_params = b.take(sizeof(ParamDev) * n_params);
  c->off_prefix = b.take(sizeof(long long) * (n_params + 1));
  c->off_fsize = b.take(sizeof(int) * c->n_factors);
  c->off_step = b.take(4 * sizeof(int));  // step counter and the Adam bias corrections
  c->off_gmax = b.take(sizeof(unsigned) * c->n_blocks);  // gradient scaling: max |G_k| bits,
  c->off_fscale2 = b.take(sizeof(float) * c->n_factors);  // 2^(2 e_k) per factor,
  c->off_bscale = b.take(sizeof(float) * c->n_blocks);    // 2^(e_k) per block
  c->off_uscale = b.take(sizeof(float) * c->n_blocks);    // split roots: 2^(e_L + e_R) per block
  c->total = b.off;
  *workspace_bytes = c->total;
  *out = c;
  return SHAMPOO_OK;
}

int shampoo_ctx_info(const shampoo_ctx* ctx, int* n_blocks, int* n_factors, int* block_size) {
  if (!ctx) return SHAMPOO_EINVAL;
  if (n_blocks) *n_blocks = ctx->n_blocks;
  if (n_factors) *n_factors = ctx->n_factors;
  if (block_size) *block_size = ctx->B;
  return SHAMPOO_OK;
}

int shampoo_block_table(const shampoo_ctx* ctx, int64_t* out) {
  if (!ctx || !out) return SHAMPOO_EINVAL;
  for (int k = 0; k < ctx->n_blocks; ++k) {
    const BlockDesc& b = ctx->blocks[k];
    int64_t* r = out + 7 * k;
    r[0] = b.param;
    r[1] = b.r0;
    r[2] = b.c0;
    r[3] = b.br;
    r[4] = b.bc;
    r[5] = 2 * k;
    r[6] = 2 * k + 1;
  }
  return SHAMPOO_OK;
}

int shampoo_init_factors(shampoo_ctx* ctx, float* factors, void* stream) {
  if (!ctx || !factors) return SHAMPOO_EINVAL;
  dash::launch_init_factors(factors, ctx->n_factors, ctx->B, ctx->hp.init_scale,
                            static_cast<cudaStream_t>(stream));
  DASH_LAUNCHED();
  return SHAMPOO_OK;
}

int shampoo_accumulate(shampoo_ctx* ctx, float* factors, void* ws_v, size_t ws_bytes, void* stream) {
  if (!ctx || !factors) return SHAMPOO_EINVAL;
  int rc = check_ws(ws_v, ws_bytes, ctx->total);
  if (rc) return rc;
  char* ws = static_cast<char*>(ws_v);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_ws = ws_v;
  ctx->last_stream = stream;
  rc = upload_tables(ctx, ws, st);
  if (rc) return rc;
  unsigned* status = reinterpret_cast<unsigned*>(ws + ctx->roots.status);
  DASH_TRY(cudaMemsetAsync(status, 0, sizeof(unsigned), st));
  const int B = ctx->B;
  __half* Gs = split_at(ws, ctx->off_gs, 0, B);
  unsigned* gmax = reinterpret_cast<unsigned*>(ws + ctx->off_gmax);
  float* fscale2 = reinterpret_cast<float*>(ws + ctx->off_fscale2);
  const int aslot = dash::prof_begin(dash::kProfAccumulate, st);
  DASH_TRY(cudaMemsetAsync(gmax, 0, sizeof(unsigned) * ctx->n_blocks, st));
  // each block is gathered scaled by 2^-e (its entries then lie in (-1, 1), the
  // split-fp16 operand range), and the products undo it exactly
  dash::launch_gather(reinterpret_cast<const BlockDesc*>(ws + ctx->off_blocks),
                      reinterpret_cast<const ParamDev*>(ws + ctx->off_params), ctx->n_blocks, B, gmax, fscale2,
                      reinterpret_cast<float*>(ws + ctx->off_bscale), Gs, st);
  DASH_LAUNCHED();
  // L <- beta L + (1-beta) G G^T ; R <- beta R + (1-beta) G^T G   (factor f uses Gs[f] twice)
  GemmArgs g = gemm_args(B, 1, status);
  dash::GemmOp& o = g.op[0];
  o.nprob = ctx->n_factors;
  o.alpha = 1.0f - ctx->hp.beta;
  o.acc_scale = fscale2;  // 2^(2e): (2^-e G)(2^-e G)^T = 2^-2e G G^T
  o.beta = ctx->hp.beta;
  o.cin_f32 = factors;
  o.out_f32 = factors;
  dash::OpBuffers ob[2] = {{Gs, ctx->n_factors, Gs, ctx->n_factors}, {Gs, ctx->n_factors, Gs, ctx->n_factors}};
  DASH_TRY(dash::launch_gemm_split(ob, g, st));
  dash::prof_end(aslot, st);
  return SHAMPOO_OK;
}

int shampoo_precondition_step(shampoo_ctx* ctx, const float* factors, const float* v0, int step, float* lambda_out,
                              float* roots_out, void* ws_v, size_t ws_bytes, void* stream) {
  if (!ctx || !factors || !v0 || step < 0) return SHAMPOO_EINVAL;
  int rc = check_ws(ws_v, ws_bytes, ctx->total);
  if (rc) return rc;
  // step 0 continues the device step counter: the roots are then recomputed
  // every step, and an explicit step must have set the counter first
  if (step == 0 && ((ctx->hp.root_every > 1) || ctx->step_ws != ws_v)) return SHAMPOO_EINVAL;
  char* ws = static_cast<char*>(ws_v);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->last_ws = ws_v;
  ctx->last_stream = stream;
  rc = upload_tables(ctx, ws, st);
  if (rc) return rc;
  const shampoo_hparams& hp = ctx->hp;
  const int B = ctx->B, nf = ctx->n_factors, nb = ctx->n_blocks;
  unsigned* status = reinterpret_cast<unsigned*>(ws + ctx->roots.status);
  const int* fsize = reinterpret_cast<const int*>(ws + ctx->off_fsize);
  __half* roots = split_at(ws, ctx->off_roots, 0, B);
  const int every = hp.root_every > 0 ? hp.root_every : 1;
  if (step == 0 || (step - 1) % every == 0 || ctx->roots_ws != ws_v) {  // root step (or no roots kept yet)
    const int pi = hp.scaling == SHAMPOO_SCALING_FROBENIUS ? 0 : hp.pi_iters;
    const bool cn = hp.solver == SHAMPOO_SOLVER_COUPLED_NEWTON;
    rc = run_roots(factors, nf, B, hp.eps, fsize, v0, pi, hp.solver, cn ? hp.cn_iters : hp.ndb_iters1,
                   cn ? hp.cn_fp16 : hp.ndb_iters2, hp.cheb_degree, hp.cheb_delta, lambda_out, roots_out, roots, ws,
                   ctx->roots, status, st);
    if (rc) return rc;
    ctx->roots_ws = ws_v;
  }

  float* pn = reinterpret_cast<float*>(ws + ctx->off_pn);
  float* un = reinterpret_cast<float*>(ws + ctx->off_un);
  float* U = reinterpret_cast<float*>(ws + ctx->off_u);
  DASH_TRY(cudaMemsetAsync(pn, 0, sizeof(float) * nb, st));
  DASH_TRY(cudaMemsetAsync(un, 0, sizeof(float) * nb, st));
  __half* Gs = split_at(ws, ctx->off_gs, 0, B);
  __half* T1 = split_at(ws, ctx->roots.solver, 0, B);  // the solver scratch is free now
  const int uslot = dash::prof_begin(dash::kProfPrecond, st);
  {  // T1_k = G_k X_R   (A = G_k, B = X_R)
    GemmArgs g = gemm_args(B, 0, status);
    dash::GemmOp& o = g.op[0];
    o.nprob = nb;
    o.a.stride = 2;
    o.b.base = 1;
    o.b.stride = 2;
    o.b_mn = 1;
    o.alpha = 1.0f;
    o.out_split = T1;
    dash::OpBuffers ob[2] = {{Gs, nf, roots, nf}, {Gs, nf, roots, nf}};
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
  }
  {  // U_k = X_L T1_k, scattered into parameter layout with ||U_k||^2   (A = X_L, B = T1_k);
     // T1 was formed from the gathered 2^-e G and both split roots were stored
     // without their scales' powers of two, so U_k is multiplied back by them
    float* uscale = reinterpret_cast<float*>(ws + ctx->off_uscale);
    dash::launch_root_pair_scale(reinterpret_cast<const float*>(ws + ctx->roots.xscale), nb, uscale, st);
    DASH_LAUNCHED();
    GemmArgs g = gemm_args(B, 0, status);
    dash::GemmOp& o = g.op[0];
    o.nprob = nb;
    o.a.stride = 2;
    o.b_mn = 1;
    o.alpha = 1.0f;
    o.acc_scale = uscale;
    o.scale = reinterpret_cast<const float*>(ws + ctx->off_bscale);
    o.blocks = reinterpret_cast<const BlockDesc*>(ws + ctx->off_blocks);
    o.u_out = U;
    o.unorm = un;
    dash::OpBuffers ob[2] = {{roots, nf, T1, nb}, {roots, nf, T1, nb}};
    DASH_TRY(dash::launch_gemm_split(ob, g, st));
  }
  dash::prof_end(uslot, st);
  const int dslot = dash::prof_begin(dash::kProfAdam, st);
  const ParamDev* pd = reinterpret_cast<const ParamDev*>(ws + ctx->off_params);
  const long long* prefix = reinterpret_cast<const long long*>(ws + ctx->off_prefix);
  const int np = static_cast<int>(ctx->params.size());
  int* info = reinterpret_cast<int*>(ws + ctx->off_step);
  dash::launch_step_info(info, step, hp.beta1, hp.beta2, st);
  DASH_LAUNCHED();
  dash::launch_adam(pd, prefix, np, ctx->n_items, B, hp.beta1, hp.beta2, hp.adam_eps, info, pn, st);
  DASH_LAUNCHED();
  dash::launch_update(pd, prefix, np, ctx->n_items, B, hp.lr, U, pn, un, st);
  DASH_LAUNCHED();
  // only a step whose launches were all queued may be continued by step 0
  if (step > 0) ctx->step_ws = ws_v;
  dash::prof_end(dslot, st);
  return SHAMPOO_OK;
}

size_t shampoo_inv_root_workspace_bytes(int n, int B, int solver) {
  (void)solver;
  if (n < 1 || !valid_B(B)) return 0;
  Bump b;
  RootLayout L;
  plan_roots(b, L, n, B, 100, 0, solver);
  return b.off;
}

static int inv_root_common(const float* A, float* X, int n, int B, float eps, const float* v0, int pi_iters,
                           void* ws, size_t ws_bytes, int solver, int it1, int it2, int degree, float delta,
                           float* lambda_out, void* stream) {
  if (!A || !X || !v0) return SHAMPOO_EINVAL;
  if (n < 1 || !valid_B(B)) return SHAMPOO_EUNSUPPORTED;
  if (n > 32767) return SHAMPOO_EUNSUPPORTED;
  if (!finite_nonneg(eps) || pi_iters < 0 || pi_iters > 100) return SHAMPOO_EINVAL;
  const int rc = check_ws(ws, ws_bytes, shampoo_inv_root_workspace_bytes(n, B, solver));
  if (rc) return rc;
  Bump b;
  RootLayout L;
  plan_roots(b, L, n, B, 100, 0, solver);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = reinterpret_cast<unsigned*>(w + L.status);
  DASH_TRY(cudaMemsetAsync(status, 0, sizeof(unsigned), st));
  return run_roots(A, n, B, eps, nullptr, v0, pi_iters, solver, it1, it2, degree, delta, lambda_out, X, nullptr, w,
                   L, status, st);
}

int shampoo_inv_root_newton_db(const float* A, float* X, int n, int B, int iters1, int iters2, float eps,
                               const float* v0, int pi_iters, float* lambda_out, void* ws, size_t ws_bytes,
                               void* stream) {
  if (iters1 < 1 || iters2 < 1 || iters1 > 1000 || iters2 > 1000) return SHAMPOO_EINVAL;
  return inv_root_common(A, X, n, B, eps, v0, pi_iters, ws, ws_bytes, SHAMPOO_SOLVER_NEWTON_DB, iters1, iters2, 0,
                         0.0f, lambda_out, stream);
}

int shampoo_inv_root_chebyshev(const float* A, float* X, int n, int B, int degree, float delta, float eps,
                               const float* v0, int pi_iters, float* lambda_out, void* ws, size_t ws_bytes,
                               void* stream) {
  if (degree < 2 || degree > 256 || !(delta > 0.0f) || !std::isfinite(delta)) return SHAMPOO_EINVAL;
  return inv_root_common(A, X, n, B, eps, v0, pi_iters, ws, ws_bytes, SHAMPOO_SOLVER_CHEBYSHEV, 0, 0, degree, delta,
                         lambda_out, stream);
}

int shampoo_inv_root_coupled_newton(const float* A, float* X, int n, int B, int iters, int fp16, float eps,
                                    const float* v0, int pi_iters, float* lambda_out, void* ws, size_t ws_bytes,
                                    void* stream) {
  if (iters < 0 || iters > 1000 || (fp16 != 0 && fp16 != 1)) return SHAMPOO_EINVAL;
  return inv_root_common(A, X, n, B, eps, v0, pi_iters, ws, ws_bytes, SHAMPOO_SOLVER_COUPLED_NEWTON, iters, fp16, 0,
                         0.0f, lambda_out, stream);
}

int shampoo_read_status(const void* ws, void* stream, unsigned* flags) {
  return dash::read_status_word(ws, stream, flags);
}

int shampoo_get_status(shampoo_ctx* ctx, int* device_flags) {
  if (!ctx) return SHAMPOO_EINVAL;
  if (!ctx->last_ws) {  // no step call has run on this ctx yet: nothing to report
    if (device_flags) *device_flags = 0;
    return SHAMPOO_OK;
  }
  unsigned w = 0;
  const int rc = dash::read_status_word(static_cast<const char*>(ctx->last_ws) + ctx->roots.status,
                                        ctx->last_stream, &w);
  if (device_flags) *device_flags = static_cast<int>(w);
  return rc;
}

const char* shampoo_strerror(int code) {
  switch (code) {
    case SHAMPOO_OK: return "success";
    case SHAMPOO_EINVAL: return "invalid argument";
    case SHAMPOO_EUNSUPPORTED: return "unsupported shape (B must be a multiple of 128 in [128, 2048], n >= 1)";
    case SHAMPOO_EWORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case SHAMPOO_ECUDA: return "CUDA launch or runtime error";
    case SHAMPOO_ENONFINITE: return "a kernel produced a non-finite value";
    case SHAMPOO_ETIMEOUT: return "a bounded device wait gave up";
    default: return "unknown status code";
  }
}

void shampoo_destroy(shampoo_ctx* ctx) { delete ctx; }

int shampoo_debug_inject_timeout(void) {
  dash::arm_load_fault();
  return SHAMPOO_OK;
}

}  // extern "C"

namespace dash {

// Synchronise the stream and read a status word (shared by the status calls).
int read_status_word(const void* ws, void* stream, unsigned* flags) {
  if (!ws) return SHAMPOO_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DASH_TRY(cudaStreamSynchronize(st));
  unsigned w = 0;
  DASH_TRY(cudaMemcpy(&w, ws, sizeof(unsigned), cudaMemcpyDeviceToHost));
  if (flags) *flags = w;
  if (w & dash::kStatusTimeout) return SHAMPOO_ETIMEOUT;  // the root cause when both are set
  if (w & dash::kStatusNonFinite) return SHAMPOO_ENONFINITE;
  return SHAMPOO_OK;
}

// Standalone root computation on a caller-provided scratch region (used by
// the static-scratch entry point in noalloc.cu).
int inv_root_with_scratch(const float* A, float* X, int n, int B, float eps, const float* v0, int pi_iters, void* ws,
                          size_t ws_bytes, int solver, int it1, int it2, int degree, float delta, float* lambda_out,
                          void* stream) {
  return inv_root_common(A, X, n, B, eps, v0, pi_iters, ws, ws_bytes, solver, it1, it2, degree, delta, lambda_out,
                         stream);
}

}  // namespace dash
