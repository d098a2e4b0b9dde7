// Multi-start power iteration on tcgen05 tensor cores (sm_100a).
//
// DASH explainer, "Building blocks" (Multi-Power-Iteration): the top
// eigenvalue of each factor is estimated from 32 random start vectors by
// repeated products with the factor and the largest Rayleigh quotient of the
// last product.  Each product W = (F + eps I) V is a 128-row by 32-column
// contraction per CTA, run on the tensor cores with split-fp16 operands
// (hi*hi + hi*lo + lo*hi, fp32 accumulation) so that the estimate keeps
// fp32 accuracy:
//   pi_prepare   scales each factor by a power of two 2^-e taken from its
//                largest diagonal entry (every entry of a positive
//                semi-definite factor then has magnitude at most 1, far
//                inside the fp16 range; the scaling is exact) and stores
//                (F + eps I) 2^-e once as split fp16 planes;
//   pi_vectors   writes the product's input vectors (the previous product
//                with unit columns) as split fp16, transposed, so that they
//                are a K-major MMA operand;
//   pi_product   one CTA per 128 rows of one factor: TMA streams 64-wide K
//                slabs of the factor and of the vectors through a two-stage
//                shared-memory ring, one thread issues the MMAs (M = 128,
//                N = 32, K = 16) into two tensor-memory accumulators (hi*hi,
//                and the cross terms), and the four warps write W and reduce
//                the column statistics |W|^2, V.W and V.V;
//   pi_finalize  lambda = max over starts of V.W / V.V, times 2^e.
// The step is bound by HBM: each product reads the split factor once (4
// bytes per element); the tensor work per byte is small.
#include "kernels.cuh"
#include "launch_util.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace dash {
namespace {

constexpr int kPRows = 128;                             // rows of W per CTA (MMA M)
constexpr int kPKBlk = 64;                              // K per stage: one 128-byte fp16 row
constexpr int kPStages = 2;
constexpr int kPATile = kPRows * kPKBlk * 2;            // 16 KB per plane of the factor
constexpr int kPVTile = kPiStarts * kPKBlk * 2;         // 4 KB per plane of the vectors
constexpr int kPStageBytes = 2 * kPATile + 2 * kPVTile;  // A hi, A lo, V hi, V lo
constexpr uint32_t kPTmemCols = 64;                     // hi*hi at column 0, cross terms at 32
constexpr int kPThreads = 128;
constexpr int kVRows = 64;                              // rows per CTA of pi_vectors

struct PiBars {
  uint64_t full[kPStages], empty[kPStages];
  uint64_t done;
  uint32_t tmem_slot;
  int abort;
  float inv[kPiStarts];
  float red[3][kPThreads / 32][kPiStarts];
};
constexpr int kPSmemBytes = kPStages * kPStageBytes + 1024 + static_cast<int>(sizeof(PiBars));

// 1 / |column j of the previous product| (1 for the start vectors).
__device__ __forceinline__ float pi_inv(const float* Wprev, const float* sprev, int f, int j) {
  if (!Wprev) return 1.0f;
  const float n2 = sprev[static_cast<size_t>(f) * 3 * kPiStarts + j];
  return n2 > 0.0f ? rsqrtf(n2) : 0.0f;
}

// pscale[f] = 2^-e with 2^(e-1) <= max_i (F_ii + eps) < 2^e over the
// factor's real part.  One warp per factor.
__global__ void pi_scale_kernel(const float* __restrict__ F, int nf, int B, float eps, const int* __restrict__ fsize,
                                float* __restrict__ pscale) {
  const int f = static_cast<int>((static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (f >= nf) return;
  const int b = fsize ? fsize[f] : B;
  const float* A = F + static_cast<size_t>(f) * B * B;
  float m = 0.0f;
  for (int i = lane; i < b; i += 32) m = fmaxf(m, A[static_cast<size_t>(i) * B + i] + eps);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) {
    float s = 1.0f;
    if (m > 0.0f && isfinite(m)) {
      int e = 0;
      frexpf(m, &e);
      s = ldexpf(1.0f, -e);
    }
    pscale[f] = s;
  }
}

// As[2f] / As[2f+1] = hi / lo planes of (F_f + eps I) pscale_f on the real
// b x b part, 0 on the padding.  Each thread converts 8 consecutive elements.
__global__ void __launch_bounds__(256) pi_split_kernel(const float* __restrict__ F, int B, float eps,
                                                       const int* __restrict__ fsize,
                                                       const float* __restrict__ pscale, __half* __restrict__ As,
                                                       unsigned* status) {
  const int f = blockIdx.y;
  const int b = fsize ? fsize[f] : B;
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t e0 = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (e0 >= BB) return;
  const int r = static_cast<int>(e0 / B), c0 = static_cast<int>(e0 % B);
  const float s = pscale[f];
  float v[8];
  if (r < b && c0 < b) {
    const float4* src = reinterpret_cast<const float4*>(F + static_cast<size_t>(f) * BB + e0);
    const float4 x = src[0], y = src[1];
    v[0] = x.x, v[1] = x.y, v[2] = x.z, v[3] = x.w, v[4] = y.x, v[5] = y.y, v[6] = y.z, v[7] = y.w;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = c0 + j;
      if (c >= b) v[j] = 0.0f;
      if (c == r) v[j] += eps;
      v[j] *= s;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.0f;
  }
  __align__(16) __half hi[8];
  __align__(16) __half lo[8];
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    split_f16(v[j], hi[j], lo[j]);
    bad |= (__hisinf(hi[j]) != 0) || !isfinite(v[j]);
  }
  *reinterpret_cast<uint4*>(As + 2 * static_cast<size_t>(f) * BB + e0) = *reinterpret_cast<const uint4*>(hi);
  *reinterpret_cast<uint4*>(As + (2 * static_cast<size_t>(f) + 1) * BB + e0) = *reinterpret_cast<const uint4*>(lo);
  if (bad && status) atomicOr(status, kStatusNonFinite);
}

// Vt[2f + p] (p = 0 hi, 1 lo) is 32 x B: row j holds start j's vector
// (v0 for the first product, else the previous product with unit columns),
// 0 at rows of the factor at or beyond its size.  64 rows per CTA,
// transposed through shared memory.
__global__ void __launch_bounds__(256) pi_vectors_kernel(const float* __restrict__ v0,
                                                         const float* __restrict__ Wprev,
                                                         const float* __restrict__ sprev, int B,
                                                         const int* __restrict__ fsize, __half* __restrict__ Vt) {
  __shared__ float tile[kPiStarts][kVRows + 1];
  __shared__ float inv[kPiStarts];
  const int f = blockIdx.y, r0 = blockIdx.x * kVRows, t = threadIdx.x;
  const int b = fsize ? fsize[f] : B;
  if (t < kPiStarts) inv[t] = pi_inv(Wprev, sprev, f, t);
  __syncthreads();
  const float* src = Wprev ? Wprev + static_cast<size_t>(f) * B * kPiStarts : v0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int i = t + 256 * q;  // float4 index in the 64 x 32 slab
    const int rr = i >> 3, c = 4 * (i & 7);
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + rr < b) x = *reinterpret_cast<const float4*>(src + static_cast<size_t>(r0 + rr) * kPiStarts + c);
    tile[c][rr] = x.x * inv[c];
    tile[c + 1][rr] = x.y * inv[c + 1];
    tile[c + 2][rr] = x.z * inv[c + 2];
    tile[c + 3][rr] = x.w * inv[c + 3];
  }
  __syncthreads();
  const int j = t >> 3, rr = 8 * (t & 7);
  __align__(16) __half hi[8];
  __align__(16) __half lo[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) split_f16(tile[j][rr + e], hi[e], lo[e]);
  const size_t plane = static_cast<size_t>(kPiStarts) * B;
  __half* dst = Vt + 2 * static_cast<size_t>(f) * plane + static_cast<size_t>(j) * B + r0 + rr;
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(hi);
  *reinterpret_cast<uint4*>(dst + plane) = *reinterpret_cast<const uint4*>(lo);
}

// On entry each lane holds one row's values of the 32 columns; on exit lane
// j holds in v[0] the sum of column j over the warp's 32 rows (each step
// halves the columns a lane carries and exchanges the other half).
__device__ __forceinline__ float warp_colsum32(float (&v)[kPiStarts], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

__device__ __forceinline__ void pi_fail(volatile int* abort_flag, unsigned* status) {
  *abort_flag = 1;
  if (status) atomicOr(status, kStatusTimeout);
}

// W_next[f] rows r0..r0+127 = As_f V (the split operands of pi_prepare and
// pi_vectors), plus the column statistics of these rows accumulated into
// snext[f] = (|W|^2, V.W, V.V), where V is the unit-column input in fp32.
__global__ void __launch_bounds__(kPThreads, 2)
    pi_product_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmV,
                      const float* __restrict__ v0, const float* __restrict__ Wprev,
                      const float* __restrict__ sprev, int B, const int* __restrict__ fsize,
                      float* __restrict__ Wnext, float* __restrict__ snext, unsigned* status) {
  const int ntile = B / kPRows;
  const int f = static_cast<int>(blockIdx.x / ntile), r0 = static_cast<int>(blockIdx.x % ntile) * kPRows;
  const int b = fsize ? fsize[f] : B;
  if (r0 >= b) return;  // no rows of the factor in this tile (uniform over the CTA)

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  PiBars* bars = reinterpret_cast<PiBars*>(smem + kPStages * kPStageBytes);
  volatile int* abort_flag = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (b + kPKBlk - 1) / kPKBlk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmV);
  }
  if (threadIdx.x < kPiStarts) bars->inv[threadIdx.x] = pi_inv(Wprev, sprev, f, threadIdx.x);
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, kPTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t s = 0, epar = 1;  // fresh barriers pass on parity 1
    int kb = 0;
    for (; kb < nk; ++kb) {
      if (!mbar_wait(&bars->empty[s], epar, abort_flag)) {
        pi_fail(abort_flag, status);
        break;
      }
      uint8_t* st = smem + s * kPStageBytes;
      mbar_arrive_expect_tx(&bars->full[s], kPStageBytes);
      tma_load_3d(st, &tmA, &bars->full[s], kb * kPKBlk, r0, 2 * f);
      tma_load_3d(st + kPATile, &tmA, &bars->full[s], kb * kPKBlk, r0, 2 * f + 1);
      tma_load_3d(st + 2 * kPATile, &tmV, &bars->full[s], kb * kPKBlk, 0, 2 * f);
      tma_load_3d(st + 2 * kPATile + kPVTile, &tmV, &bars->full[s], kb * kPKBlk, 0, 2 * f + 1);
      if (++s == kPStages) {
        s = 0;
        epar ^= 1u;
      }
    }
    if (*abort_flag) {  // let this CTA's own copies land before it can exit
      volatile int never = 0;
      for (int j = (kb > kPStages ? kb - kPStages : 0); j < kb; ++j)
        mbar_wait(&bars->full[j % kPStages], static_cast<uint32_t>(j / kPStages) & 1u, &never);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t d0 = sw128_kmajor_desc(smem_u32(smem));
    constexpr uint32_t kA = kPATile >> 4, kV = kPVTile >> 4, kS = kPStageBytes >> 4;  // descriptor units
    const uint32_t idesc = f16_idesc(kPRows, kPiStarts);
    const uint32_t dh = tbase, dx = tbase + 32u;
    uint32_t s = 0, fpar = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!mbar_wait(&bars->full[s], fpar, abort_flag)) {
        pi_fail(abort_flag, status);
        break;
      }
      tc_fence_after();
      const uint64_t ah = d0 + s * kS, al = ah + kA, vh = ah + 2 * kA, vl = vh + kV;
#pragma unroll
      for (int kk = 0; kk < kPKBlk / 16; ++kk) {
        const uint32_t acc = (kb | kk) ? 1u : 0u;
        mma_f16_ss(dh, ah + 2u * kk, vh + 2u * kk, idesc, acc);  // hi * hi
        mma_f16_ss(dx, ah + 2u * kk, vl + 2u * kk, idesc, acc);  // hi * lo
        mma_f16_ss(dx, al + 2u * kk, vh + 2u * kk, idesc, 1u);   // + lo * hi
      }
      mma_commit(&bars->empty[s]);
      if (++s == kPStages) {
        s = 0;
        fpar ^= 1u;
      }
    }
    // arrives once every MMA issued above has completed; tensor memory is
    // released only after that
    mma_commit(&bars->done);
    volatile int never = 0;
    mbar_wait(&bars->done, 0u, &never);
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  bool ok = mbar_wait_sleep(&bars->done, 0u, abort_flag) && !*abort_flag;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  const int row = r0 + 32 * warp + lane;
  if (ok) {
    float w[kPiStarts];
    {
      uint32_t h[32], x[32];
      const uint32_t ta = tbase + (static_cast<uint32_t>(32 * warp) << 16);
      tmem_ld_32x32b_x32(ta, h);
      tmem_ld_32x32b_x32(ta + 32u, x);
      tmem_ld_wait_regs<32>(h);
      tmem_ld_wait_regs<32>(x);
#pragma unroll
      for (int j = 0; j < kPiStarts; ++j) w[j] = __uint_as_float(h[j]) + __uint_as_float(x[j]) * kLoUnscale;
    }
    float4* wo = reinterpret_cast<float4*>(Wnext + (static_cast<size_t>(f) * B + row) * kPiStarts);
#pragma unroll
    for (int q = 0; q < kPiStarts / 4; ++q) wo[q] = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    float vn[kPiStarts];
    if (row < b) {
      const float* src = Wprev ? Wprev + (static_cast<size_t>(f) * B + row) * kPiStarts
                               : v0 + static_cast<size_t>(row) * kPiStarts;
#pragma unroll
      for (int q = 0; q < kPiStarts / 4; ++q) {
        const float4 x = reinterpret_cast<const float4*>(src)[q];
        vn[4 * q] = x.x * bars->inv[4 * q];
        vn[4 * q + 1] = x.y * bars->inv[4 * q + 1];
        vn[4 * q + 2] = x.z * bars->inv[4 * q + 2];
        vn[4 * q + 3] = x.w * bars->inv[4 * q + 3];
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPiStarts; ++j) vn[j] = 0.0f;
    }
    float a[kPiStarts];
#pragma unroll
    for (int j = 0; j < kPiStarts; ++j) a[j] = w[j] * w[j];
    bars->red[0][warp][lane] = warp_colsum32(a, lane);
#pragma unroll
    for (int j = 0; j < kPiStarts; ++j) a[j] = vn[j] * w[j];
    bars->red[1][warp][lane] = warp_colsum32(a, lane);
#pragma unroll
    for (int j = 0; j < kPiStarts; ++j) a[j] = vn[j] * vn[j];
    bars->red[2][warp][lane] = warp_colsum32(a, lane);
  }
  const bool all_ok = __syncthreads_and(ok) != 0;
  if (all_ok && threadIdx.x < 3 * kPiStarts) {
    const int q = threadIdx.x / kPiStarts, c = threadIdx.x % kPiStarts;
    float sum = 0.0f;
#pragma unroll
    for (int w4 = 0; w4 < kPThreads / 32; ++w4) sum += bars->red[q][w4][c];
    if (sum != 0.0f) atomicAdd(&snext[static_cast<size_t>(f) * 3 * kPiStarts + q * kPiStarts + c], sum);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kPTmemCols);
  }
}

__global__ void pi_finalize_kernel(const float* __restrict__ s, int nf, const float* __restrict__ pscale,
                                   float* __restrict__ lam, float* __restrict__ lam_out) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= nf) return;
  const float* sf = s + static_cast<size_t>(f) * 3 * kPiStarts;
  float best = 0.0f;
  bool any = false;
  for (int j = 0; j < kPiStarts; ++j) {
    const float den = sf[2 * kPiStarts + j];
    const float rq = den > 0.0f ? sf[kPiStarts + j] / den : 0.0f;
    if (!any || rq > best) best = rq;
    any = true;
  }
  if (pscale) best /= pscale[f];
  lam[f] = best;
  if (lam_out) lam_out[f] = best;
}

}  // namespace

void launch_pi_prepare(const float* F, int nf, int B, float eps, const int* fsize, float* pscale, __half* As,
                       unsigned* status, cudaStream_t st) {
  pi_scale_kernel<<<(nf + 7) / 8, 256, 0, st>>>(F, nf, B, eps, fsize, pscale);
  prof_count_launch();
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 2048), nf);
  pi_split_kernel<<<grid, 256, 0, st>>>(F, B, eps, fsize, pscale, As, status);
  prof_count_launch();
}

void launch_pi_vectors(const float* v0, const float* W_prev, const float* stats_prev, int nf, int B,
                       const int* fsize, __half* Vt, cudaStream_t st) {
  dim3 grid(B / kVRows, nf);
  pi_vectors_kernel<<<grid, 256, 0, st>>>(v0, W_prev, stats_prev, B, fsize, Vt);
  prof_count_launch();
}

cudaError_t launch_pi_product(const __half* As, const __half* Vt, const float* v0, const float* W_prev,
                              const float* stats_prev, int nf, int B, const int* fsize, float* W_next,
                              float* stats_next, unsigned* status, cudaStream_t st) {
  if (nf < 1 || B % kPRows != 0) return cudaErrorInvalidValue;
  CUtensorMap ma, mv;
  cudaError_t e = encode_split_stack_map(&ma, As, B, nf, kPRows);
  if (e != cudaSuccess) return e;
  e = encode_f16_3d_map(&mv, Vt, B, kPiStarts, 2ll * nf, kPiStarts);
  if (e != cudaSuccess) return e;
  static std::atomic<unsigned long long> attr_set;
  e = smem_limit_once(pi_product_kernel, kPSmemBytes, attr_set);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(nf) * static_cast<unsigned>(B / kPRows);
  pi_product_kernel<<<grid, kPThreads, kPSmemBytes, st>>>(ma, mv, v0, W_prev, stats_prev, B, fsize, W_next,
                                                          stats_next, status);
  prof_count_launch();
  return cudaGetLastError();
}

void launch_pi_finalize(const float* stats_last, int nf, const float* pscale, float* lambda, float* lambda_out,
                        cudaStream_t st) {
  pi_finalize_kernel<<<(nf + 127) / 128, 128, 0, st>>>(stats_last, nf, pscale, lambda, lambda_out);
  prof_count_launch();
}

}  // namespace dash
