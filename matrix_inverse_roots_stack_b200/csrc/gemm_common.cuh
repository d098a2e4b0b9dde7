// Pieces shared by the two split-fp16 GEMM kernels (gemm.cu: 128 x 128 tiles
// with a parked output stage; gemm_wide.cu: 128 x 256 tiles written out by
// the accumulator warps): problem indexing, the MN-major operand descriptor,
// the split-fp16 helpers, the epilogue arithmetic of one output row
// segment, out = s_p * (alpha * a_p * acc + beta * Cin + gamma * I), and the
// shared-memory staging of 32 x 32 output steps for TMA tensor stores.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace dash {

__device__ __forceinline__ int gemm_at(const Idx& i, int p) {
  return i.base + (i.stride > 0 ? i.stride : 1) * (i.mod > 0 ? p % i.mod : p);
}

__device__ __forceinline__ void gemm_fail_timeout(volatile int* abort_flag, unsigned* status) {
  *abort_flag = 1;
  if (status) atomicOr(status, kStatusTimeout);
}

// Descriptor of an MN-major operand tile: K-rows of 128 bytes (64 columns)
// per block, blocks block_bytes apart (leading byte offset; 8 KB for blocks
// of 64 K-rows), 8-row swizzle atoms of 1024 bytes (stride byte offset),
// 128-byte swizzle.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t block_bytes = 8192u) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(block_bytes >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// out(col0 + j, row) = v[j]: for a fixed j the 32 lanes (consecutive rows)
// write consecutive addresses.
__device__ __forceinline__ void store_split16_t(__half* base, size_t B, size_t BB, int row, int col0, const float* v,
                                                bool& bad) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    __half2 h, l;
    split_f16x2(v[j], v[j + 1], h, l);
    bad |= f16_overflows(v[j]) || f16_overflows(v[j + 1]);
    base[(col0 + j) * B + row] = __low2half(h);
    base[(col0 + j + 1) * B + row] = __high2half(h);
    base[BB + (col0 + j) * B + row] = __low2half(l);
    base[BB + (col0 + j + 1) * B + row] = __high2half(l);
  }
}

// Raw 16-element chunk of a split row (hi and lo planes, 32 bytes each).
struct SplitChunk {
  uint4 h[2], l[2];
};

__device__ __forceinline__ void join_chunk(const SplitChunk& c, float* out) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const __half2* ah = reinterpret_cast<const __half2*>(&c.h[q]);
    const __half2* bh = reinterpret_cast<const __half2*>(&c.l[q]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __half22float2(ah[e]);
      const float2 y = __half22float2(bh[e]);
      out[q * 8 + 2 * e] = x.x + y.x * kLoUnscale;
      out[q * 8 + 2 * e + 1] = x.y + y.y * kLoUnscale;
    }
  }
}

// Epilogue of one problem's output for a run of 16-column chunks of one row:
// v = s_p * (alpha * a_p * acc + beta * Cin + gamma * I), written as split
// fp16 (times 2^-e when split_norm is set, 2^(e-1) <= s_p < 2^e) and/or fp32
// (mirrored for symmetric launches), or scattered into parameter layout with
// its sum of squares.
struct GemmEpilogue {
  float s, alpha, beta, gamma, ss;  // s_p, alpha * a_p, beta, gamma; split-output factor
  const __half* cin;
  const float* cinf;
  __half* os;
  float* of;
  bool scatter;
  BlockDesc bd;
  float sumsq;
  bool bad;

  __device__ __forceinline__ void init(const GemmOp& g, int p, size_t B, size_t BB) {
    (void)B;
    s = g.scale ? g.scale[gemm_at(g.scale_i, p)] : 1.0f;
    ss = 1.0f;  // split outputs of root stacks carry s_p's power of two back out (fp16 range)
    if (g.split_norm && isfinite(s) && s != 0.0f) {
      int e;
      frexpf(s, &e);
      ss = ldexpf(1.0f, -e);
    }
    alpha = g.acc_scale ? g.alpha * g.acc_scale[gemm_at(g.accs_i, p)] : g.alpha;
    beta = g.beta;
    gamma = g.gamma;
    cin = g.cin_split ? g.cin_split + static_cast<size_t>(gemm_at(g.cin_i, p)) * 2 * BB : nullptr;
    cinf = g.cin_f32 ? g.cin_f32 + static_cast<size_t>(gemm_at(g.cinf_i, p)) * BB : nullptr;
    os = g.out_split ? g.out_split + static_cast<size_t>(gemm_at(g.out_i, p)) * 2 * BB : nullptr;
    of = g.out_f32 ? g.out_f32 + static_cast<size_t>(gemm_at(g.outf_i, p)) * BB : nullptr;
    scatter = g.blocks != nullptr;
    if (scatter) bd = g.blocks[p];
    sumsq = 0.0f;
    bad = false;
  }

  // Raw Cin of one 16-column chunk (64 bytes: split hi and lo planes, or
  // fp32), so that several chunks can be in flight before any is used.
  struct CinRaw {
    uint4 q[4];
  };
  __device__ __forceinline__ bool has_cin() const { return cin != nullptr || cinf != nullptr; }
  __device__ __forceinline__ CinRaw load_cin(size_t B, size_t BB, int row, int col0) const {
    CinRaw r;
    if (cin) {
      const uint4* h = reinterpret_cast<const uint4*>(cin + row * B + col0);
      const uint4* l = reinterpret_cast<const uint4*>(cin + BB + row * B + col0);
      r.q[0] = h[0];
      r.q[1] = h[1];
      r.q[2] = l[0];
      r.q[3] = l[1];
    } else {
      const uint4* f = reinterpret_cast<const uint4*>(cinf + row * B + col0);
#pragma unroll
      for (int i = 0; i < 4; ++i) r.q[i] = f[i];
    }
    return r;
  }
  __device__ __forceinline__ void join_cin(const CinRaw& r, float* cj) const {
    if (cin) {
      SplitChunk c;
      c.h[0] = r.q[0];
      c.h[1] = r.q[1];
      c.l[0] = r.q[2];
      c.l[1] = r.q[3];
      join_chunk(c, cj);
    } else {
      const float* f = reinterpret_cast<const float*>(r.q);
#pragma unroll
      for (int j = 0; j < 16; ++j) cj[j] = f[j];
    }
  }

  // v = s_p * (alpha * a_p * acc + beta * Cin + gamma * I) for one
  // 16-column chunk, in packed fp32 pairs and in this order: alpha a_p acc
  // (rounded), plus beta Cin (one fused multiply-add), plus gamma on the
  // diagonal, times s_p.  The order is part of the result: for factors whose
  // smallest eigenvalues sit near the rounding level of their diagonal (the
  // exponential moving average of G G^T at condition numbers of 1e7 and
  // more), folding the scalars into one multiply-add doubled the distance of
  // the update from the float64 reference.  cj holds Cin's chunk in fp32
  // when has_cin().  Callers check the result's range (check_finite, or the
  // fp16 overflow test of the split store, which also catches non-finite
  // values).
  __device__ __forceinline__ void apply(int row, int col0, float* v, const float* cj) const {
    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float2 r = __fmul2_rn(make_float2(v[j], v[j + 1]), a2);
      v[j] = r.x;
      v[j + 1] = r.y;
    }
    if (has_cin()) {
      const float2 b2 = make_float2(beta, beta);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 r = __ffma2_rn(b2, make_float2(cj[j], cj[j + 1]), make_float2(v[j], v[j + 1]));
        v[j] = r.x;
        v[j + 1] = r.y;
      }
    }
    const int d = row - col0;
    if (gamma != 0.0f && d >= 0 && d < 16) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j == d) v[j] += gamma;
    }
    if (s != 1.0f) {
      const float2 s2 = make_float2(s, s);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 r = __fmul2_rn(make_float2(v[j], v[j + 1]), s2);
        v[j] = r.x;
        v[j + 1] = r.y;
      }
    }
  }

  __device__ __forceinline__ void check_finite(const float* v) {
#pragma unroll
    for (int j = 0; j < 16; ++j) bad |= !isfinite(v[j]);
  }

  // Scatter of an applied chunk into parameter layout (rows and columns
  // past the block's extent are dropped), with its sum of squares.
  __device__ __forceinline__ void scatter_chunk(const GemmOp& g, int row, int col0, const float* v) {
    if (row >= bd.br) return;
    float* dst = g.u_out + bd.off + static_cast<long long>(bd.r0 + row) * bd.pitch + bd.c0 + col0;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (col0 + j < bd.bc) {
        dst[j] = v[j];
        sumsq += v[j] * v[j];
      }
  }

  // Transposed copy of an applied chunk (symmetric launches): for a fixed
  // column the 32 lanes (consecutive rows) write consecutive addresses.
  __device__ __forceinline__ void store_mirror(size_t B, size_t BB, int row, int col0, const float* v) {
    if (os) {
      float w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) w[j] = v[j] * ss;
      store_split16_t(os, B, BB, row, col0, w, bad);
    }
    if (of) {
#pragma unroll
      for (int j = 0; j < 16; ++j) of[(col0 + j) * B + row] = v[j];
    }
  }

  // Warp-collective: the non-finite flag and the scattered sum of squares.
  __device__ __forceinline__ void finish(const GemmOp& g, int p, unsigned* status) {
    if (bad) atomicOr(status, kStatusNonFinite);
    if (scatter) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
      if ((threadIdx.x & 31) == 0 && sumsq != 0.0f) atomicAdd(&g.unorm[p], sumsq);
    }
  }
};

// Epilogue tensor maps of a launch, per op: split and fp32 outputs and Cin
// (split or fp32), boxes of 32 rows x 32 columns (encoded for what an op
// has; scattering ops read no Cin).
struct OutMaps {
  CUtensorMap split[2], f32[2], cin[2];
};

// Staging layouts; lane l holds row l of a 32 x 32 step.
// - Split (and split Cin): plane k (hi, lo) at k * 2 KB, row l at 64 l, its
//   16-byte quarter h (columns 8h..8h+7) at h ^ ((l >> 1) & 3) (64-byte
//   swizzle: address bits 5:4 ^= bits 8:7).
// - fp32: row l at 128 l, its 16-byte eighth h (columns 4h..4h+3) at
//   h ^ (l & 7) (128-byte swizzle: bits 6:4 ^= bits 9:7).
// Eight consecutive lanes cover all 32 banks, so each 16-byte access takes
// the minimum four wavefronts.  Buffers are 4 KB-aligned.
__device__ __forceinline__ uint32_t split_slot(int lane, int plane, int h) {
  return static_cast<uint32_t>(plane * 2048 + lane * 64 + ((h ^ ((lane >> 1) & 3)) << 4));
}

// v[0], v[1]: the step's two 16-column chunks (already times the split factor)
__device__ __forceinline__ void stage_split32(uint8_t* buf, int lane, const float (*v)[16], bool& bad) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    __half2 hi[8], lo[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      split_f16x2(v[c][2 * j], v[c][2 * j + 1], hi[j], lo[j]);
      bad |= f16_overflows(v[c][2 * j]) || f16_overflows(v[c][2 * j + 1]);
    }
    *reinterpret_cast<uint4*>(buf + split_slot(lane, 0, 2 * c)) = *reinterpret_cast<const uint4*>(&hi[0]);
    *reinterpret_cast<uint4*>(buf + split_slot(lane, 0, 2 * c + 1)) = *reinterpret_cast<const uint4*>(&hi[4]);
    *reinterpret_cast<uint4*>(buf + split_slot(lane, 1, 2 * c)) = *reinterpret_cast<const uint4*>(&lo[0]);
    *reinterpret_cast<uint4*>(buf + split_slot(lane, 1, 2 * c + 1)) = *reinterpret_cast<const uint4*>(&lo[4]);
  }
}

__device__ __forceinline__ void stage_f32x32(uint8_t* buf, int lane, const float (*v)[16]) {
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const float* x = &v[h >> 2][4 * (h & 3)];
    *reinterpret_cast<float4*>(buf + lane * 128 + ((h ^ (lane & 7)) << 4)) = make_float4(x[0], x[1], x[2], x[3]);
  }
}

// The transpose of a step into a split staging buffer: lane l's value of
// column j goes to row j, column l (v already times the split factor; the
// non-finite check is the one stage_split32 made on the same values).  For
// a fixed j the 32 lanes write one 64-byte row, so the stores do not
// conflict.
__device__ __forceinline__ void stage_split32_t(uint8_t* buf, int lane, const float (*v)[16]) {
  const uint32_t col = static_cast<uint32_t>((lane & 7) * 2);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      __half2 hi, lo;
      split_f16x2(v[c][j], v[c][j + 1], hi, lo);
      const int r = 16 * c + j;  // rows r and r + 1 share the swizzle phase (r even)
      const uint32_t o = static_cast<uint32_t>(r * 64 + (((lane >> 3) ^ ((r >> 1) & 3)) << 4)) + col;
      *reinterpret_cast<__half*>(buf + o) = __low2half(hi);
      *reinterpret_cast<__half*>(buf + o + 64) = __high2half(hi);
      *reinterpret_cast<__half*>(buf + 2048 + o) = __low2half(lo);
      *reinterpret_cast<__half*>(buf + 2048 + o + 64) = __high2half(lo);
    }
  }
}

// The transpose of a step into an fp32 staging buffer: lane l's value of
// column j goes to row j, column l (one 128-byte row per j).
__device__ __forceinline__ void stage_f32x32_t(uint8_t* buf, int lane, const float (*v)[16]) {
  const uint32_t col = static_cast<uint32_t>((lane & 3) * 4);
#pragma unroll
  for (int j = 0; j < 32; ++j)
    *reinterpret_cast<float*>(buf + j * 128 + ((((lane >> 2) ^ (j & 7))) << 4) + col) = v[j >> 4][j & 15];
}

// Cin of chunk c (0, 1) of a step from a split staging buffer, joined to fp32
__device__ __forceinline__ void read_cin_chunk(const uint8_t* buf, int lane, int c, float* cj) {
  SplitChunk r;
  r.h[0] = *reinterpret_cast<const uint4*>(buf + split_slot(lane, 0, 2 * c));
  r.h[1] = *reinterpret_cast<const uint4*>(buf + split_slot(lane, 0, 2 * c + 1));
  r.l[0] = *reinterpret_cast<const uint4*>(buf + split_slot(lane, 1, 2 * c));
  r.l[1] = *reinterpret_cast<const uint4*>(buf + split_slot(lane, 1, 2 * c + 1));
  join_chunk(r, cj);
}

// fp32 Cin of chunk c (0, 1) of a step from an fp32 staging buffer
__device__ __forceinline__ void read_cin_f32_chunk(const uint8_t* buf, int lane, int c, float* cj) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = *reinterpret_cast<const float4*>(buf + lane * 128 + (((4 * c + i) ^ (lane & 7)) << 4));
    cj[4 * i] = x.x;
    cj[4 * i + 1] = x.y;
    cj[4 * i + 2] = x.z;
    cj[4 * i + 3] = x.w;
  }
}

// The warp's writes to buf go out as one tensor store at (c0, c1, c2).
__device__ __forceinline__ void store_step(int lane, const CUtensorMap* map, const uint8_t* buf, int c0, int c1,
                                           int c2) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(map, buf, c0, c1, c2);
    bulk_commit();
  }
}

// A staged fp32 step (stage_f32x32) scattered into parameter layout: lane l
// writes column col0 + l of rows row0.. (coalesced across the lanes), inside
// the block's extent only, and adds its squares to sumsq.
__device__ __forceinline__ void scatter_step(const uint8_t* buf, int lane, const GemmOp& g, const BlockDesc& bd,
                                             int row0, int col0, float& sumsq) {
  const int col = col0 + lane;
  if (col >= bd.bc) return;
  float* dst = g.u_out + bd.off + static_cast<long long>(bd.r0) * bd.pitch + bd.c0 + col;
  const int nr = bd.br - row0 < 32 ? bd.br - row0 : 32;
#pragma unroll 4
  for (int r = 0; r < nr; ++r) {
    const float x =
        *reinterpret_cast<const float*>(buf + r * 128 + ((((lane >> 2) ^ (r & 7)) << 4) | ((lane & 3) << 2)));
    dst[static_cast<long long>(row0 + r) * bd.pitch] = x;
    sumsq += x * x;
  }
}

// The epilogue maps of a launch's ops (see OutMaps).
cudaError_t encode_out_maps(const GemmArgs& a, OutMaps* om);

int gemm_sm_count();

// The 128 x 256 tile kernel (gemm_wide.cu): whether it takes a launch, and
// its launch on the four encoded operand maps (A0, B0, A1, B1; B maps with
// 256-row boxes when K-major).
bool gemm_wide_supported(const GemmArgs& a);
cudaError_t launch_gemm_wide(const CUtensorMap* maps, const GemmArgs& a, long long nprob, cudaStream_t stream);

}  // namespace dash
