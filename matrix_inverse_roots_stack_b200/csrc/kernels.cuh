// Memory-bound kernels of the batched block-Shampoo step: power iteration,
// solver prologues, gradient gather, Adam graft and update.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gemm.cuh"

namespace dash {

constexpr int kPiStarts = 32;  // power-iteration start vectors per factor

// Per-parameter metadata used by the Adam / update kernels.
// Rows per Adam / update work item (one item = kUpdRows rows x up to 1024
// columns of one parameter).
constexpr int kUpdRows = 8;

struct ParamDev {
  const float* grad;
  float* param;
  float* m;
  float* v;
  long long uoff;       // offset of this parameter in the flat U buffer
  long long item_base;  // first work item (kUpdRows rows x 1024 columns)
  int rows, cols;
  int blk_base;         // index of the parameter's first block
  int ncb;              // column blocks
  int chunks;           // 1024-column chunks per row
  int vec;              // 1: float4 path (cols % 4 == 0, 16-byte aligned)
};

// Power iteration on the tensor cores (power.cu).
// pi_prepare: pscale[f] = 2^-e with 2^(e-1) <= max_i (F_ii + eps) < 2^e, and
// As (a split stack of nf matrices) = (F + eps I) pscale on each factor's
// real part, 0 on the padding.
void launch_pi_prepare(const float* F, int nf, int B, float eps, const int* fsize, float* pscale, __half* As,
                       unsigned* status, cudaStream_t st);

// pi_vectors: Vt ((nf, 2, 32, B) fp16, hi/lo planes) = the next product's
// input vectors, transposed: v0 ((B, 32) fp32, shared by all factors) when
// W_prev is null, else W_prev ((nf, B, 32) fp32) with unit columns (norms
// from stats_prev).  Rows at or beyond a factor's true size are 0.
void launch_pi_vectors(const float* v0, const float* W_prev, const float* stats_prev, int nf, int B,
                       const int* fsize, __half* Vt, cudaStream_t st);

// pi_product: W_next = As V (V the split operand of pi_vectors; W_next is
// scaled by pscale like As) and, per column, |W_next|^2, V.W_next and V.V
// accumulated into stats_next ((nf, 3, 32), zeroed beforehand).
cudaError_t launch_pi_product(const __half* As, const __half* Vt, const float* v0, const float* W_prev,
                              const float* stats_prev, int nf, int B, const int* fsize, float* W_next,
                              float* stats_next, unsigned* status, cudaStream_t st);

// lambda[f] = max_j (V.W)_j / (V.V)_j / pscale[f] from the last product's
// statistics (pscale may be null: 1).
void launch_pi_finalize(const float* stats_last, int nf, const float* pscale, float* lambda, float* lambda_out,
                        cudaStream_t st);

// lambda_f = ||F_f + eps I||_F over the real fsize[f] x fsize[f] part (the
// Frobenius scale estimate, in place of the power iteration).
void launch_frob_norm(const float* F, int nf, int B, float eps, const int* fsize, float* lambda, float* lambda_out,
                      cudaStream_t st);

// Newton-DB stage-1 prologue: c = 1/(2 lambda); Y0 = c (F + eps I) (padding:
// identity); D0 = (I - Y0)/2; Zhat1 = (I + D0)/zs; xscale = c^(1/4) zs.
void launch_ndb_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda, float zs,
                     __half* Y0, __half* D0, __half* Z1, float* xscale, cudaStream_t st);

// Newton-DB stage-2 prologue from the split Y of stage 1:
// D0 = (I - Y)/2; Zhat1 = (I + D0)/zs.
void launch_ndb_stage2_init(const __half* Y, int nf, int B, float zs, __half* D0, __half* Z1, cudaStream_t st);

// out = xscale_f * Zhat (split in; fp32 and/or split out, the split output
// times 2^-e with 2^(e-1) <= xscale_f < 2^e); used when a stage has a single
// iteration.
// uscale[k] = 2^(e_2k + e_2k+1) with 2^(e_f - 1) <= xscale_f < 2^e_f: undoes
// the split roots' scaling in the preconditioner (nb blocks, factors 2k, 2k+1).
void launch_root_pair_scale(const float* xscale, int nb, float* uscale, cudaStream_t st);
void launch_scale_split(const __half* Z, int nf, int B, const float* xscale, float* out_f32, __half* out_split,
                        cudaStream_t st);

// Chebyshev prologue with the spectral scaling c = 1/(2 lambda):
// T = 2c (F + eps I) - I (padding: 0); b_{d-1} = c_{d-1} I + 2 c_d T;
// xscale = c^(1/4).
void launch_cheb_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda,
                      float c_dm1, float c_d, __half* T, __half* bdm1, float* xscale, cudaStream_t st);

// Coupled-Newton prologue: M0 = c (F + eps I) (I on padding), X0 = I, split;
// xscale = c^(1/4) with c = 1/(2 lambda).
void launch_cn_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda, __half* M0,
                    __half* X0, float* xscale, cudaStream_t st);

// Gather gradient blocks into padded split matrices scaled by a power of two
// per block, 2^-e_k with 2^(e_k - 1) <= max |G_k| < 2^e_k (exact):
// Gs[2k] = G_k 2^-e_k, Gs[2k+1] = its transpose; fscale2[2k] = fscale2[2k+1]
// = 2^(2 e_k) and bscale[k] = 2^(e_k) undo it in the products.  gmax (nb
// words) must be zero on entry; it receives each block's max |G| bits.
void launch_gather(const BlockDesc* blocks, const ParamDev* params, int nb, int B, unsigned* gmax, float* fscale2,
                   float* bscale, __half* Gs, cudaStream_t st);

// factors[f] = init_scale * I.
void launch_init_factors(float* F, int nf, int B, float init_scale, cudaStream_t st);

// Step counter and Adam bias corrections on the device: info[0] = step if
// step > 0, else info[0] + 1; info[1], info[2] = 1 / (1 - beta1^t),
// 1 / (1 - beta2^t) (float bits).
void launch_step_info(int* info, int step, float beta1, float beta2, cudaStream_t st);

// Adam moments and per-block sum of squares of the Adam direction P, with
// the bias corrections of launch_step_info's info.
void launch_adam(const ParamDev* params, const long long* item_prefix, int n_params, long long n_items, int B,
                 float beta1, float beta2, float adam_eps, const int* info, float* pnorm, cudaStream_t st);

// param -= lr * sqrt(pnorm_k / unorm_k) * U (0 where unorm_k == 0).
void launch_update(const ParamDev* params, const long long* item_prefix, int n_params, long long n_items, int B,
                   float lr, const float* U, const float* pnorm, const float* unorm, cudaStream_t st);

}  // namespace dash
