// Memory-bound kernels of the batched block-Shampoo step (see kernels.cuh).
#include "kernels.cuh"
#include "profile.cuh"
#include "ptx.cuh"

namespace dash {
namespace {

// ------------------------------------------------------------ power iteration
//
// DASH explainer, "Building blocks" (Multi-Power-Iteration): K random starts,
// repeated products with the factor, largest Rayleigh quotient.  One CTA
// computes 128 rows of W = A V (32 columns) for one factor, streaming A in
// 128 x 32 slabs through shared memory.

constexpr int kPiRows = 128;
constexpr int kPiK = 32;

__global__ void __launch_bounds__(256) pi_iter_kernel(const float* __restrict__ F, int B, float eps,
                                                      const int* __restrict__ fsize, const float* __restrict__ v0,
                                                      const float* __restrict__ Wprev,
                                                      const float* __restrict__ sprev, float* __restrict__ Wnext,
                                                      float* __restrict__ snext) {
  __shared__ float As[kPiRows][kPiK + 1];
  __shared__ __align__(16) float Vs[kPiK][kPiStarts];
  __shared__ float inv[kPiStarts];
  __shared__ float red[8][3][kPiStarts];

  const int f = blockIdx.y;
  const int r0 = blockIdx.x * kPiRows;
  const int b = fsize ? fsize[f] : B;
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  if (t < kPiStarts) {
    float n2 = Wprev ? sprev[static_cast<size_t>(f) * 3 * kPiStarts + t] : 1.0f;
    inv[t] = Wprev ? (n2 > 0.0f ? rsqrtf(n2) : 0.0f) : 1.0f;
  }
  __syncthreads();

  const float* Fm = F + static_cast<size_t>(f) * B * B;
  const float* Vsrc = Wprev ? Wprev + static_cast<size_t>(f) * B * kPiStarts : v0;
  const int row = t >> 1;
  const int cb = (t & 1) * 16;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0f;

  if (r0 < b) {
    for (int k0 = 0; k0 < b; k0 += kPiK) {
#pragma unroll
      for (int i = 0; i < (kPiRows * kPiK) / 256; ++i) {
        const int idx = i * 256 + t;
        const int rr = idx / kPiK, kk = idx % kPiK;
        const int gr = r0 + rr, gk = k0 + kk;
        float a = 0.0f;
        if (gr < b && gk < b) a = Fm[static_cast<size_t>(gr) * B + gk] + (gr == gk ? eps : 0.0f);
        As[rr][kk] = a;
      }
#pragma unroll
      for (int i = 0; i < (kPiK * kPiStarts) / 256; ++i) {
        const int idx = i * 256 + t;
        const int kk = idx / kPiStarts, c = idx % kPiStarts;
        const int gk = k0 + kk;
        Vs[kk][c] = gk < b ? Vsrc[static_cast<size_t>(gk) * kPiStarts + c] * inv[c] : 0.0f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kPiK; ++kk) {
        const float a = As[row][kk];
        const float4* v4 = reinterpret_cast<const float4*>(&Vs[kk][cb]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v = v4[q];
          acc[4 * q] += a * v.x;
          acc[4 * q + 1] += a * v.y;
          acc[4 * q + 2] += a * v.z;
          acc[4 * q + 3] += a * v.w;
        }
      }
      __syncthreads();
    }
  }

  const int gr = r0 + row;
  float* Wo = Wnext + static_cast<size_t>(f) * B * kPiStarts + static_cast<size_t>(gr) * kPiStarts + cb;
#pragma unroll
  for (int j = 0; j < 16; ++j) Wo[j] = acc[j];

  // column statistics of this CTA's rows
  float w2[16], vw[16], v2[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float v = gr < b ? Vsrc[static_cast<size_t>(gr) * kPiStarts + cb + j] * inv[cb + j] : 0.0f;
    w2[j] = acc[j] * acc[j];
    vw[j] = v * acc[j];
    v2[j] = v * v;
  }
#pragma unroll
  for (int o = 2; o < 32; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      w2[j] += __shfl_xor_sync(0xffffffffu, w2[j], o);
      vw[j] += __shfl_xor_sync(0xffffffffu, vw[j], o);
      v2[j] += __shfl_xor_sync(0xffffffffu, v2[j], o);
    }
  }
  if (lane < 2) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      red[warp][0][cb + j] = w2[j];
      red[warp][1][cb + j] = vw[j];
      red[warp][2][cb + j] = v2[j];
    }
  }
  __syncthreads();
  if (t < 3 * kPiStarts) {
    const int q = t / kPiStarts, c = t % kPiStarts;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w][q][c];
    if (s != 0.0f) atomicAdd(&snext[static_cast<size_t>(f) * 3 * kPiStarts + q * kPiStarts + c], s);
  }
}

__global__ void pi_finalize_kernel(const float* __restrict__ s, int nf, float* __restrict__ lam,
                                   float* __restrict__ lam_out) {
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
  lam[f] = best;
  if (lam_out) lam_out[f] = best;
}

// ------------------------------------------------------------ solver prologues

__device__ __forceinline__ void store_split4(__half* base, size_t BB, size_t idx, const float* x) {
  __half h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) split_f16(x[e], h[e], l[e]);
  *reinterpret_cast<uint2*>(base + idx) = *reinterpret_cast<const uint2*>(h);
  *reinterpret_cast<uint2*>(base + BB + idx) = *reinterpret_cast<const uint2*>(l);
}

__device__ __forceinline__ void load_split4(const __half* base, size_t BB, size_t idx, float* x) {
  const uint2 a = *reinterpret_cast<const uint2*>(base + idx);
  const uint2 b = *reinterpret_cast<const uint2*>(base + BB + idx);
  const __half* h = reinterpret_cast<const __half*>(&a);
  const __half* l = reinterpret_cast<const __half*>(&b);
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = join_f16(h[e], l[e]);
}

// Newton-DB prologues.  grid (B/32, B/32, nf), block (32, 8): each CTA owns a
// 32 x 32 tile, writes its outputs in place and, through shared memory, the
// transposed copies the K-major GEMM needs (exact transposes, so the stage-2
// iterates, which are not exactly symmetric, keep consistent copies).

__device__ __forceinline__ void put_split(__half* base, size_t BB, size_t idx, float x) {
  __half h, l;
  split_f16(x, h, l);
  base[idx] = h;
  base[BB + idx] = l;
}

__global__ void ndb_init_kernel(const float* __restrict__ F, int B, float eps, const int* __restrict__ fsize,
                                const float* __restrict__ lam, float zs, __half* __restrict__ Y0,
                                __half* __restrict__ D0, __half* __restrict__ D0t, __half* __restrict__ Z1,
                                __half* __restrict__ Z1t, float* __restrict__ xscale) {
  __shared__ float td[32][33], tz[32][33];
  const int f = blockIdx.z;
  const size_t BB = static_cast<size_t>(B) * B;
  const int tr = blockIdx.y * 32, tc = blockIdx.x * 32;
  const int b = fsize ? fsize[f] : B;
  const float c = 0.5f / lam[f];
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && threadIdx.y == 0) xscale[f] = sqrtf(sqrtf(c)) * zs;
  const float* Fm = F + f * BB;
  const size_t off = static_cast<size_t>(f) * 2 * BB;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr + threadIdx.y + 8 * i, col = tc + threadIdx.x;
    const float id = (r == col) ? 1.0f : 0.0f;
    const float a = (r < b && col < b) ? c * (Fm[static_cast<size_t>(r) * B + col] + id * eps) : id;
    const float d = 0.5f * (id - a);
    const float z = (id + d) / zs;
    const size_t e = static_cast<size_t>(r) * B + col;
    put_split(Y0 + off, BB, e, a);
    put_split(D0 + off, BB, e, d);
    put_split(Z1 + off, BB, e, z);
    td[threadIdx.y + 8 * i][threadIdx.x] = d;
    tz[threadIdx.y + 8 * i][threadIdx.x] = z;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tc + threadIdx.y + 8 * i, col = tr + threadIdx.x;
    const size_t e = static_cast<size_t>(r) * B + col;
    put_split(D0t + off, BB, e, td[threadIdx.x][threadIdx.y + 8 * i]);
    put_split(Z1t + off, BB, e, tz[threadIdx.x][threadIdx.y + 8 * i]);
  }
}

__global__ void ndb_stage2_init_kernel(const __half* __restrict__ Y, int B, float zs, __half* __restrict__ D0,
                                       __half* __restrict__ D0t, __half* __restrict__ Z1,
                                       __half* __restrict__ Z1t) {
  __shared__ float td[32][33], tz[32][33];
  const int f = blockIdx.z;
  const size_t BB = static_cast<size_t>(B) * B;
  const int tr = blockIdx.y * 32, tc = blockIdx.x * 32;
  const size_t off = static_cast<size_t>(f) * 2 * BB;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr + threadIdx.y + 8 * i, col = tc + threadIdx.x;
    const size_t e = static_cast<size_t>(r) * B + col;
    const float id = (r == col) ? 1.0f : 0.0f;
    const float y = join_f16(Y[off + e], Y[off + BB + e]);
    const float d = 0.5f * (id - y);
    const float z = (id + d) / zs;
    put_split(D0 + off, BB, e, d);
    put_split(Z1 + off, BB, e, z);
    td[threadIdx.y + 8 * i][threadIdx.x] = d;
    tz[threadIdx.y + 8 * i][threadIdx.x] = z;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tc + threadIdx.y + 8 * i, col = tr + threadIdx.x;
    const size_t e = static_cast<size_t>(r) * B + col;
    put_split(D0t + off, BB, e, td[threadIdx.x][threadIdx.y + 8 * i]);
    put_split(Z1t + off, BB, e, tz[threadIdx.x][threadIdx.y + 8 * i]);
  }
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
  if (out_split) store_split4(out_split + 2 * f * BB, BB, idx, z);
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

// ------------------------------------------------------------ gather

// grid (B/32, B/32, nb), block (32, 8)
__global__ void gather_kernel(const BlockDesc* __restrict__ blocks, const ParamDev* __restrict__ params, int B,
                              __half* __restrict__ Gs) {
  __shared__ float tile[32][33];
  const int k = blockIdx.z;
  const BlockDesc bd = blocks[k];
  const float* G = params[bd.param].grad;
  const size_t BB = static_cast<size_t>(B) * B;
  __half* g0 = Gs + static_cast<size_t>(2 * k) * 2 * BB;
  __half* g1 = Gs + static_cast<size_t>(2 * k + 1) * 2 * BB;
  const int tr = blockIdx.y * 32, tc = blockIdx.x * 32;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr + threadIdx.y + 8 * i, c = tc + threadIdx.x;
    float v = 0.0f;
    if (r < bd.br && c < bd.bc) v = G[static_cast<long long>(bd.r0 + r) * bd.pitch + bd.c0 + c];
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
// One CTA = one work item = up to 1024 columns of one row of one parameter;
// a warp covers 128 aligned columns, which lie in one block (B % 128 == 0).

__device__ __forceinline__ int find_param(const long long* prefix, int n, long long item) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) adam_kernel(const ParamDev* __restrict__ params,
                                                   const long long* __restrict__ prefix, int n_params, int B,
                                                   float b1, float b2, float eps, float ibc1, float ibc2,
                                                   float* __restrict__ pnorm) {
  const long long item = blockIdx.x;
  const int pi = find_param(prefix, n_params, item);
  const ParamDev P = params[pi];
  const long long local = item - P.item_base;
  const int r = static_cast<int>(local / P.chunks);
  const int c0 = static_cast<int>(local % P.chunks) * 1024;
  const int warp = threadIdx.x >> 5;
  const int c = c0 + threadIdx.x * 4;
  const size_t base = static_cast<size_t>(r) * P.cols;
  float sq = 0.0f;
  if (P.vec) {
    if (c < P.cols) {
      const float4 g = *reinterpret_cast<const float4*>(P.grad + base + c);
      float4 m = *reinterpret_cast<const float4*>(P.m + base + c);
      float4 v = *reinterpret_cast<const float4*>(P.v + base + c);
      const float gv[4] = {g.x, g.y, g.z, g.w};
      float mv[4] = {m.x, m.y, m.z, m.w}, vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        mv[e] = b1 * mv[e] + (1.0f - b1) * gv[e];
        vv[e] = b2 * vv[e] + (1.0f - b2) * gv[e] * gv[e];
        const float p = (mv[e] * ibc1) / (sqrtf(vv[e] * ibc2) + eps);
        sq += p * p;
      }
      *reinterpret_cast<float4*>(P.m + base + c) = make_float4(mv[0], mv[1], mv[2], mv[3]);
      *reinterpret_cast<float4*>(P.v + base + c) = make_float4(vv[0], vv[1], vv[2], vv[3]);
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
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const int cw = c0 + warp * 128;
  if ((threadIdx.x & 31) == 0 && cw < P.cols && sq != 0.0f) {
    const int k = P.blk_base + (r / B) * P.ncb + cw / B;
    atomicAdd(&pnorm[k], sq);
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
  const int r = static_cast<int>(local / P.chunks);
  const int c0 = static_cast<int>(local % P.chunks) * 1024;
  const int c = c0 + threadIdx.x * 4;
  if (c >= P.cols) return;
  const int k = P.blk_base + (r / B) * P.ncb + c / B;
  const float un = unorm[k];
  const float s = un > 0.0f ? lr * sqrtf(pnorm[k] / un) : 0.0f;
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

}  // namespace

// ------------------------------------------------------------ launchers

void launch_pi_iter(const float* F, int nf, int B, float eps, const int* fsize, const float* v0,
                    const float* W_prev, const float* stats_prev, float* W_next, float* stats_next,
                    cudaStream_t st) {
  dim3 grid(B / kPiRows, nf);
  pi_iter_kernel<<<grid, 256, 0, st>>>(F, B, eps, fsize, v0, W_prev, stats_prev, W_next, stats_next);
  prof_count_launch();
}

void launch_pi_finalize(const float* stats_last, int nf, float* lambda, float* lambda_out, cudaStream_t st) {
  pi_finalize_kernel<<<(nf + 127) / 128, 128, 0, st>>>(stats_last, nf, lambda, lambda_out);
  prof_count_launch();
}

void launch_ndb_init(const float* F, int nf, int B, float eps, const int* fsize, const float* lambda, float zs,
                     __half* Y0, __half* D0, __half* D0t, __half* Z1, __half* Z1t, float* xscale,
                     cudaStream_t st) {
  dim3 grid(B / 32, B / 32, nf);
  ndb_init_kernel<<<grid, dim3(32, 8), 0, st>>>(F, B, eps, fsize, lambda, zs, Y0, D0, D0t, Z1, Z1t, xscale);
  prof_count_launch();
}

void launch_ndb_stage2_init(const __half* Y, int nf, int B, float zs, __half* D0, __half* D0t, __half* Z1,
                            __half* Z1t, cudaStream_t st) {
  dim3 grid(B / 32, B / 32, nf);
  ndb_stage2_init_kernel<<<grid, dim3(32, 8), 0, st>>>(Y, B, zs, D0, D0t, Z1, Z1t);
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

void launch_gather(const BlockDesc* blocks, const ParamDev* params, int nb, int B, __half* Gs, cudaStream_t st) {
  dim3 grid(B / 32, B / 32, nb);
  gather_kernel<<<grid, dim3(32, 8), 0, st>>>(blocks, params, B, Gs);
  prof_count_launch();
}

void launch_init_factors(float* F, int nf, int B, float init_scale, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(static_cast<size_t>(B) * B / 1024), nf);
  init_factors_kernel<<<grid, 256, 0, st>>>(F, B, init_scale);
  prof_count_launch();
}

void launch_adam(const ParamDev* params, const long long* item_prefix, int n_params, long long n_items, int B,
                 float beta1, float beta2, float adam_eps, float bc1, float bc2, float* pnorm, cudaStream_t st) {
  adam_kernel<<<static_cast<unsigned>(n_items), 256, 0, st>>>(params, item_prefix, n_params, B, beta1, beta2,
                                                               adam_eps, 1.0f / bc1, 1.0f / bc2, pnorm);
  prof_count_launch();
}

void launch_update(const ParamDev* params, const long long* item_prefix, int n_params, long long n_items, int B,
                   float lr, const float* U, const float* pnorm, const float* unorm, cudaStream_t st) {
  update_kernel<<<static_cast<unsigned>(n_items), 256, 0, st>>>(params, item_prefix, n_params, B, lr, U, pnorm,
                                                                unorm);
  prof_count_launch();
}

}  // namespace dash
