// Memory-bound kernels of the batched block-Shampoo step (see kernels.cuh).
#include "kernels.cuh"
#include "profile.cuh"
#include "ptx.cuh"

namespace dash {
namespace {

// Frobenius-norm scale estimate ("Building blocks", scaling: the Frobenius
// alternative to spectral scaling): lambda_f = ||F_f + eps I||_F over the
// factor's real b x b part (padding excluded).  One CTA per factor, float64
// accumulation; sum of squares of F plus 2 eps tr(F) + b eps^2.
__global__ void frob_norm_kernel(const float* __restrict__ F, int B, float eps, const int* __restrict__ fsize,
                                 float* __restrict__ lam, float* __restrict__ lam_out) {
  const int f = blockIdx.x;
  const int b = fsize ? fsize[f] : B;
  const float* A = F + static_cast<size_t>(f) * B * B;
  double ss = 0.0, tr = 0.0;
  for (int i = threadIdx.y; i < b; i += blockDim.y) {
    const float* row = A + static_cast<size_t>(i) * B;
    for (int j = threadIdx.x; j < b; j += blockDim.x) {
      const double x = row[j];
      ss += x * x;
      if (j == i) tr += x;
    }
  }
  ss += 2.0 * static_cast<double>(eps) * tr;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  __shared__ double part[32];
  const int w = (threadIdx.y * blockDim.x + threadIdx.x) >> 5, nw = (blockDim.x * blockDim.y) >> 5;
  if ((threadIdx.x & 31) == 0) part[w] = ss;
  __syncthreads();
  if (threadIdx.x == 0 && threadIdx.y == 0) {
    double t = 0.0;
    for (int k = 0; k < nw; ++k) t += part[k];
    t += static_cast<double>(b) * static_cast<double>(eps) * static_cast<double>(eps);
    const float v = static_cast<float>(sqrt(t > 0.0 ? t : 0.0));
    lam[f] = v;
    if (lam_out) lam_out[f] = v;
  }
}

// ------------------------------------------------------------ solver prologues

__device__ __forceinline__ void store_split4(__half* base, size_t BB, size_t idx, const float* x) {
  __half2 h[2], l[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) split_f16x2(x[2 * e], x[2 * e + 1], h[e], l[e]);
  *reinterpret_cast<uint2*>(base + idx) = *reinterpret_cast<const uint2*>(h);
  *reinterpret_cast<uint2*>(base + BB + idx) = *reinterpret_cast<const uint2*>(l);
}

__device__ __forceinline__ void load_split4(const __half* base, size_t BB, size_t idx, float* x) {
  const uint2 a = *reinterpret_cast<const uint2*>(base + idx);
  const uint2 b = *reinterpret_cast<const uint2*>(base + BB + idx);
  const __half2* h = reinterpret_cast<const __half2*>(&a);
  const __half2* l = reinterpret_cast<const __half2*>(&b);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float2 fh = __half22float2(h[e]), fl = __half22float2(l[e]);
    x[2 * e] = fh.x + fl.x * kLoUnscale;
    x[2 * e + 1] = fh.y + fl.y * kLoUnscale;
  }
}

// Newton-DB prologues (element-wise; grid (B*B/1024, nf), 256 threads, 4
// consecutive elements per thread).

__global__ void __launch_bounds__(256) ndb_init_kernel(const float* __restrict__ F, int B, float eps,
                                                       const int* __restrict__ fsize,
                                                       const float* __restrict__ lam, float zs,
                                                       __half* __restrict__ Y0, __half* __restrict__ D0,
                                                       __half* __restrict__ Z1, float* __restrict__ xscale) {
  const int f = blockIdx.y;
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t idx = (static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  const int b = fsize ? fsize[f] : B;
  const float c = 0.5f / lam[f];
  if (idx == 0) xscale[f] = sqrtf(sqrtf(c)) * zs;
  const int r = static_cast<int>(idx / B), col = static_cast<int>(idx % B);
  const float4 a4 = *reinterpret_cast<const float4*>(F + f * BB + idx);
  const float av[4] = {a4.x, a4.y, a4.z, a4.w};
  float y[4], d[4], z[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int cc = col + e;
    const float id = (r == cc) ? 1.0f : 0.0f;
    const float a = (r < b && cc < b) ? c * (av[e] + id * eps) : id;
    y[e] = a;
    d[e] = 0.5f * (id - a);
    z[e] = (id + d[e]) / zs;
  }
  store_split4(Y0 + 2 * f * BB, BB, idx, y);
  store_split4(D0 + 2 * f * BB, BB, idx, d);
  store_split4(Z1 + 2 * f * BB, BB, idx, z);
}

__global__ void __launch_bounds__(256) ndb_stage2_init_kernel(const __half* __restrict__ Y, int B, float zs,
                                                              __half* __restrict__ D0, __half* __restrict__ Z1) {
  const int f = blockIdx.y;
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t idx = (static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  const int r = static_cast<int>(idx / B), col = static_cast<int>(idx % B);
  float y[4], d[4], z[4];
  load_split4(Y + 2 * f * BB, BB, idx, y);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float id = (r == col + e) ? 1.0f : 0.0f;
    d[e] = 0.5f * (id - y[e]);
    z[e] = (id + d[e]) / zs;
  }
  store_split4(D0 + 2 * f * BB, BB, idx, d);
  store_split4(Z1 + 2 * f * BB, BB, idx, z);
}

__global__ void __launch_bounds__(256) scale_split_kernel(const __half* __restrict__ Z, int B,
                                                          const float* __restrict__ xscale,
                                                          float* __restrict__ out_f32,
                                                          __half* __restrict__ out_split) {
  const int f = blockIdx.y;
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t idx = (static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  float z[4];
  load_split4(Z + 2 * f * BB, BB, idx, z);
  const float s = xscale[f];
#pragma unroll
  for (int e = 0; e < 4; ++e) z[e] *= s;
  if (out_f32) *reinterpret_cast<float4*>(out_f32 + f * BB + idx) = make_float4(z[0], z[1], z[2], z[3]);
  if (out_split) {  // split roots carry the power of two of their scale back out (fp16 range)
    int ex = 0;
    if (isfinite(s) && s != 0.0f) frexpf(s, &ex);
    const float ss = ldexpf(1.0f, -ex);
#pragma unroll
    for (int e = 0; e < 4; ++e) z[e] *= ss;
    store_split4(out_split + 2 * f * BB, BB, idx, z);
  }
}

// uscale[k] = 2^(e_L + e_R): the powers of two that the split roots of block
// k's factors (2k, 2k+1) were stored without, 2^(e-1) <= xscale < 2^e.
__global__ void root_pair_scale_kernel(const float* __restrict__ xscale, int nb, float* __restrict__ uscale) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= nb) return;
  int el = 0, er = 0;
  const float sl = xscale[2 * k], sr = xscale[2 * k + 1];
  if (isfinite(sl) && sl != 0.0f) frexpf(sl, &el);
  if (isfinite(sr) && sr != 0.0f) frexpf(sr, &er);
  uscale[k] = ldexpf(1.0f, el + er);
}

__global__ void __launch_bounds__(256) cheb_init_kernel(const float* __restrict__ F, int B, float eps,
                                                        const int* __restrict__ fsize,
                                                        const float* __restrict__ lam, float c_dm1, float c_d,
                                                        __half* __restrict__ T, __half* __restrict__ bdm1,
                                                        float* __restrict__ xscale) {
  const int f = blockIdx.y;
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t idx = (static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  const int b = fsize ? fsize[f] : B;
  const float c = 0.5f / lam[f];  // spectral scaling 1/(2 lambda), as for Newton-DB
  const float two_c = 2.0f * c;
  if (idx == 0) xscale[f] = sqrtf(sqrtf(c));
  const int r = static_cast<int>(idx / B), col = static_cast<int>(idx % B);
  const float4 a4 = *reinterpret_cast<const float4*>(F + f * BB + idx);
  const float av[4] = {a4.x, a4.y, a4.z, a4.w};
  float t[4], bb[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int cc = col + e;
    const float id = (r == cc) ? 1.0f : 0.0f;
    t[e] = (r < b && cc < b) ? two_c * (av[e] + id * eps) - id : 0.0f;
    bb[e] = c_dm1 * id + 2.0f * c_d * t[e];
  }
  store_split4(T + 2 * f * BB, BB, idx, t);
  store_split4(bdm1 + 2 * f * BB, BB, idx, bb);
}

// Coupled-Newton prologue ("Building blocks", Coupled-Newton): with the
// common scaling c = 1/(2 lambda), M0 = c (F + eps I) and X0 = I; padding rows
// and columns get M0 = I (a fixed point: C = I there).  xscale = c^(1/4).
__global__ void __launch_bounds__(256) cn_init_kernel(const float* __restrict__ F, int B, float eps,
                                                      const int* __restrict__ fsize, const float* __restrict__ lam,
                                                      __half* __restrict__ M0, __half* __restrict__ X0,
                                                      float* __restrict__ xscale) {
  const int f = blockIdx.y;
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t idx = (static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  const int b = fsize ? fsize[f] : B;
  const float c = 0.5f / lam[f];
  if (idx == 0) xscale[f] = sqrtf(sqrtf(c));
  const int r = static_cast<int>(idx / B), col = static_cast<int>(idx % B);
  const float4 a4 = *reinterpret_cast<const float4*>(F + f * BB + idx);
  const float av[4] = {a4.x, a4.y, a4.z, a4.w};
  float m[4], x[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int cc = col + e;
    const float id = (r == cc) ? 1.0f : 0.0f;
    m[e] = (r < b && cc < b) ? c * (av[e] + id * eps) : id;
    x[e] = id;
  }
  store_split4(M0 + 2 * f * BB, BB, idx, m);
  store_split4(X0 + 2 * f * BB, BB, idx, x);
}

// ------------------------------------------------------------ gather

// Largest |G| of every gradient block, as float bits (atomicMax on the bits
// orders non-negative floats; NaN sorts above +Inf).  grid (B/32, nb), 256
// threads: a CTA takes 32 rows of one block, a warp 4 rows.
__global__ void __launch_bounds__(256) block_absmax_kernel(const BlockDesc* __restrict__ blocks,
                                                           const ParamDev* __restrict__ params,
                                                           unsigned* __restrict__ gmax) {
  const int k = blockIdx.y;
  const BlockDesc bd = blocks[k];
  const float* G = params[bd.param].grad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned m = 0u;
  for (int i = 0; i < 4; ++i) {
    const int r = blockIdx.x * 32 + warp * 4 + i;
    if (r >= bd.br) break;
    const float* row = G + static_cast<long long>(bd.r0 + r) * bd.pitch + bd.c0;
    for (int c = lane; c < bd.bc; c += 32) m = max(m, __float_as_uint(fabsf(row[c])));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if (lane == 0 && m != 0u) atomicMax(&gmax[k], m);
}

// Power-of-two scale 2^-e of a gradient block with largest entry x:
// 2^(e-1) <= x < 2^e, so every scaled entry lies in (-1, 1) and its fp16
// split neither overflows nor (for entries within 2^-14 of the largest)
// loses bits to subnormals; 1 for an all-zero or non-finite block.
__device__ __forceinline__ int block_exponent(unsigned bits) {
  const float x = __uint_as_float(bits);
  if (bits == 0u || !isfinite(x)) return 0;
  int e;
  frexpf(x, &e);
  return e;
}

// grid (B/32, B/32, nb), block (32, 8).  Gs[2k] = G_k 2^-e_k, Gs[2k+1] its
// transpose; the CTA at tile (0, 0) also writes the exact factors that undo
// the scaling: fscale2[2k] = fscale2[2k+1] = 2^(2 e_k) (for G G^T, G^T G)
// and bscale[k] = 2^(e_k) (for X_L G X_R).
__global__ void gather_kernel(const BlockDesc* __restrict__ blocks, const ParamDev* __restrict__ params, int B,
                              const unsigned* __restrict__ gmax, float* __restrict__ fscale2,
                              float* __restrict__ bscale, __half* __restrict__ Gs) {
  __shared__ float tile[32][33];
  const int k = blockIdx.z;
  const BlockDesc bd = blocks[k];
  const float* G = params[bd.param].grad;
  const size_t BB = static_cast<size_t>(B) * B;
  __half* g0 = Gs + static_cast<size_t>(2 * k) * 2 * BB;
  __half* g1 = Gs + static_cast<size_t>(2 * k + 1) * 2 * BB;
  const int e = block_exponent(gmax[k]);
  const float sc = ldexpf(1.0f, -e);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && threadIdx.y == 0) {
    fscale2[2 * k] = fscale2[2 * k + 1] = ldexpf(1.0f, 2 * e);
    bscale[k] = ldexpf(1.0f, e);
  }
  const int tr = blockIdx.y * 32, tc = blockIdx.x * 32;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr + threadIdx.y + 8 * i, c = tc + threadIdx.x;
    float v = 0.0f;
    if (r < bd.br && c < bd.bc) v = sc * G[static_cast<long long>(bd.r0 + r) * bd.pitch + bd.c0 + c];
    tile[threadIdx.y + 8 * i][threadIdx.x] = v;
    __half h, l;
    split_f16(v, h, l);
    g0[static_cast<size_t>(r) * B + c] = h;
    g0[BB + static_cast<size_t>(r) * B + c] = l;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tc + threadIdx.y + 8 * i, c = tr + threadIdx.x;  // row of G^T
    const float v = tile[threadIdx.x][threadIdx.y + 8 * i];
    __half h, l;
    split_f16(v, h, l);
    g1[static_cast<size_t>(r) * B + c] = h;
    g1[BB + static_cast<size_t>(r) * B + c] = l;
  }
}

__global__ void init_factors_kernel(float* __restrict__ F, int B, float s) {
  const size_t BB = static_cast<size_t>(B) * B;
  const size_t idx = (static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  const int f = blockIdx.y;
  const int r = static_cast<int>(idx / B), c = static_cast<int>(idx % B);
  float4 v = make_float4(r == c ? s : 0.f, r == c + 1 ? s : 0.f, r == c + 2 ? s : 0.f, r == c + 3 ? s : 0.f);
  *reinterpret_cast<float4*>(F + f * BB + idx) = v;
}

// ------------------------------------------------------------ Adam + update
//
// DASH explainer, "Step-by-step" (grafting with Adam's magnitude): P is the
// Adam direction, s = ||P||_F / ||U||_F per block, theta -= lr * s * U.
// One CTA = one work item = kUpdRows rows x up to 1024 columns of one
// parameter; a warp covers 128 aligned columns, which lie in one block
// (B % 128 == 0), and the rows of an item lie in one block row (B % 8 == 0),
// so each warp's sum of P^2 belongs to one block.  Warps of the same block
// are combined in shared memory before the one atomic per block and item.

__device__ __forceinline__ int find_param(const long long* prefix, int n, long long item) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void adam4(const float* g, float* m, float* v, float b1, float b2, float eps, float ibc1,
                                      float ibc2, float& sq) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    m[e] = b1 * m[e] + (1.0f - b1) * g[e];
    v[e] = b2 * v[e] + (1.0f - b2) * g[e] * g[e];
    const float p = (m[e] * ibc1) / (sqrtf(v[e] * ibc2) + eps);
    sq += p * p;
  }
}

// The step's Adam bias corrections on the device: step > 0 sets the step
// counter info[0] to it; step == 0 advances the counter by one.  info[1],
// info[2] receive 1 / (1 - beta1^t) and 1 / (1 - beta2^t) as floats.
__global__ void step_info_kernel(int* __restrict__ info, int step, float beta1, float beta2) {
  const int t = step > 0 ? step : info[0] + 1;
  info[0] = t;
  float* f = reinterpret_cast<float*>(info + 1);
  f[0] = 1.0f / static_cast<float>(1.0 - pow(static_cast<double>(beta1), t));
  f[1] = 1.0f / static_cast<float>(1.0 - pow(static_cast<double>(beta2), t));
}

__global__ void __launch_bounds__(256) adam_kernel(const ParamDev* __restrict__ params,
                                                   const long long* __restrict__ prefix, int n_params, int B,
                                                   float b1, float b2, float eps, const int* __restrict__ info,
                                                   float* __restrict__ pnorm) {
  const float ibc1 = __int_as_float(info[1]), ibc2 = __int_as_float(info[2]);
  __shared__ float wsum[8];
  __shared__ int wblk[8];
  const long long item = blockIdx.x;
  const int pi = find_param(prefix, n_params, item);
  const ParamDev P = params[pi];
  const long long local = item - P.item_base;
  const int r0 = static_cast<int>(local / P.chunks) * kUpdRows;
  const int c0 = static_cast<int>(local % P.chunks) * 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = c0 + threadIdx.x * 4;
  const int r1 = min(r0 + kUpdRows, P.rows);
  float sq = 0.0f;
  for (int r = r0; r < r1; ++r) {
    const size_t base = static_cast<size_t>(r) * P.cols;
    if (P.vec) {
      if (c < P.cols) {
        const float4 g4 = *reinterpret_cast<const float4*>(P.grad + base + c);
        const float4 m4 = *reinterpret_cast<const float4*>(P.m + base + c);
        const float4 v4 = *reinterpret_cast<const float4*>(P.v + base + c);
        const float g[4] = {g4.x, g4.y, g4.z, g4.w};
        float m[4] = {m4.x, m4.y, m4.z, m4.w}, v[4] = {v4.x, v4.y, v4.z, v4.w};
        adam4(g, m, v, b1, b2, eps, ibc1, ibc2, sq);
        *reinterpret_cast<float4*>(P.m + base + c) = make_float4(m[0], m[1], m[2], m[3]);
        *reinterpret_cast<float4*>(P.v + base + c) = make_float4(v[0], v[1], v[2], v[3]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ce = c + e;
        if (ce < P.cols) {
          const float g = P.grad[base + ce];
          const float m = b1 * P.m[base + ce] + (1.0f - b1) * g;
          const float v = b2 * P.v[base + ce] + (1.0f - b2) * g * g;
          P.m[base + ce] = m;
          P.v[base + ce] = v;
          const float p = (m * ibc1) / (sqrtf(v * ibc2) + eps);
          sq += p * p;
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const int cw = c0 + warp * 128;
  if (lane == 0) {
    wsum[warp] = sq;
    wblk[warp] = cw < P.cols ? P.blk_base + (r0 / B) * P.ncb + cw / B : -1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // one atomic per block the item touches
    float acc = 0.0f;
    for (int w = 0; w < 8; ++w) {
      if (wblk[w] < 0) break;
      acc += wsum[w];
      if (w == 7 || wblk[w + 1] != wblk[w]) {
        if (acc != 0.0f) atomicAdd(&pnorm[wblk[w]], acc);
        acc = 0.0f;
      }
    }
  }
}

__global__ void __launch_bounds__(256) update_kernel(const ParamDev* __restrict__ params,
                                                     const long long* __restrict__ prefix, int n_params, int B,
                                                     float lr, const float* __restrict__ U,
                                                     const float* __restrict__ pnorm,
                                                     const float* __restrict__ unorm) {
  const long long item = blockIdx.x;
  const int pi = find_param(prefix, n_params, item);
  const ParamDev P = params[pi];
  const long long local = item - P.item_base;
  const int r0 = static_cast<int>(local / P.chunks) * kUpdRows;
  const int c0 = static_cast<int>(local % P.chunks) * 1024;
  const int c = c0 + threadIdx.x * 4;
  if (c >= P.cols) return;
  const int k = P.blk_base + (r0 / B) * P.ncb + c / B;
  const float un = unorm[k];
  const float s = un > 0.0f ? lr * sqrtf(pnorm[k] / un) : 0.0f;
  const int r1 = min(r0 + kUpdRows, P.rows);
  for (int r = r0; r < r1; ++r) {
    const size_t base = static_cast<size_t>(r) * P.cols;
    const float* u = U + P.uoff + base;
    if (P.vec) {
      float4 th = *reinterpret_cast<const float4*>(P.param + base + c);
      const float4 uu = *reinterpret_cast<const float4*>(u + c);
      th.x -= s * uu.x;
      th.y -= s * uu.y;
      th.z -= s * uu.z;
      th.w -= s * uu.w;
      *reinterpret_cast<float4*>(P.param + base + c) = th;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c + e < P.cols) P.param[base + c + e] -= s * u[c + e];
    }
  }
}

}  // namespace

// ------------------------------------------------------------ launchers

void launch_frob_norm(const float* F, int nf, int B, float eps, const int* fsize, float* lambda, float* lambda_out,
                      cudaStream_t st) {
  frob_norm_kernel<<<nf, dim3(128, 8), 0, st>>>(F, B, eps, fsize, lambda, lambda_out);
  prof_count_launch();
}

void launch_ndb_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda, float zs,
                     __half* Y0, __half* D0, __half* Z1, float* xscale, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  ndb_init_kernel<<<grid, 256, 0, st>>>(F, B, eps, fsize, lambda, zs, Y0, D0, Z1, xscale);
  prof_count_launch();
}

void launch_ndb_stage2_init(const __half* Y, int nf, int B, float zs, __half* D0, __half* Z1, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  ndb_stage2_init_kernel<<<grid, 256, 0, st>>>(Y, B, zs, D0, Z1);
  prof_count_launch();
}

void launch_scale_split(const __half* Z, int nf, int B, const float* xscale, float* out_f32, __half* out_split,
                        cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  scale_split_kernel<<<grid, 256, 0, st>>>(Z, B, xscale, out_f32, out_split);
  prof_count_launch();
}

void launch_cheb_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda,
                      float c_dm1, float c_d, __half* T, __half* bdm1, float* xscale, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  cheb_init_kernel<<<grid, 256, 0, st>>>(F, B, eps, fsize, lambda, c_dm1, c_d, T, bdm1, xscale);
  prof_count_launch();
}

void launch_cn_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda, __half* M0,
                    __half* X0, float* xscale, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  cn_init_kernel<<<grid, 256, 0, st>>>(F, B, eps, fsize, lambda, M0, X0, xscale);
  prof_count_launch();
}

void launch_gather(const BlockDesc* blocks, const ParamDev* params, int nb, int B, unsigned* gmax, float* fscale2,
                   float* bscale, __half* Gs, cudaStream_t st) {
  block_absmax_kernel<<<dim3(B / 32, nb), 256, 0, st>>>(blocks, params, gmax);
  prof_count_launch();
  dim3 grid(B / 32, B / 32, nb);
  gather_kernel<<<grid, dim3(32, 8), 0, st>>>(blocks, params, B, gmax, fscale2, bscale, Gs);
  prof_count_launch();
}

void launch_root_pair_scale(const float* xscale, int nb, float* uscale, cudaStream_t st) {
  root_pair_scale_kernel<<<(nb + 255) / 256, 256, 0, st>>>(xscale, nb, uscale);
  prof_count_launch();
}

void launch_init_factors(float* F, int nf, int B, float init_scale, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  init_factors_kernel<<<grid, 256, 0, st>>>(F, B, init_scale);
  prof_count_launch();
}

void launch_step_info(int* info, int step, float beta1, float beta2, cudaStream_t st) {
  step_info_kernel<<<1, 1, 0, st>>>(info, step, beta1, beta2);
  prof_count_launch();
}

void launch_adam(const ParamDev* params, const long long* item_prefix, int n_params, long long n_items, int B,
                 float beta1, float beta2, float adam_eps, const int* info, float* pnorm, cudaStream_t st) {
  adam_kernel<<<static_cast<unsigned>(n_items), 256, 0, st>>>(params, item_prefix, n_params, B, beta1, beta2,
                                                               adam_eps, info, pnorm);
  prof_count_launch();
}

void launch_update(const ParamDev* params, const long long* item_prefix, int n_params, long long n_items, int B,
                   float lr, const float* U, const float* pnorm, const float* unorm, cudaStream_t st) {
  update_kernel<<<static_cast<unsigned>(n_items), 256, 0, st>>>(params, item_prefix, n_params, B, lr, U, pnorm,
                                                                unorm);
  prof_count_launch();
}

}  // namespace dash
