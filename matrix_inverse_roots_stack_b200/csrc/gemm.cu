// Batched split-fp16 GEMM on tcgen05 tensor cores (sm_100a).
//
// One CTA computes one 128 x 128 output tile of one problem.  Warp 0 (one
// lane) streams the four operand tiles of each 64-wide K slab (A hi/lo,
// Bm hi/lo; 16 KB each) into a 3-stage shared-memory ring with TMA; warp 1
// (one lane) issues the tcgen05.mma instructions: per 16-wide K step
// hi*hi into accumulator 0 and hi*lo + lo*hi into accumulator 1, both in
// tensor memory (2 x 128 fp32 columns).  After the last commit all four warps
// read their 32 rows back with tcgen05.ld, combine acc0 + 2^-11 acc1, apply
// the epilogue and write split and/or fp32 results.
#include "gemm.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace dash {
namespace {

constexpr int kTile = 128;
constexpr int kKBlk = 64;                          // fp16 elements per 128-byte row
constexpr int kStages = 3;
constexpr int kTileBytes = kTile * kKBlk * 2;      // 16 KB
constexpr int kStageBytes = 4 * kTileBytes;        // A hi, A lo, Bm hi, Bm lo
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 256;                // two 128-column accumulators
constexpr uint32_t kIdesc = f16_idesc(128, 128);

__device__ __forceinline__ int at(const Idx& i, int p) {
  return i.base + (i.stride > 0 ? i.stride : 1) * (i.mod > 0 ? p % i.mod : p);
}

// Tile t of a problem -> (tile row, tile column).  sym: upper triangle only,
// enumerated row by row.
__device__ __forceinline__ void tile_coords(int t, int nt, int sym, int& ti, int& tj) {
  if (!sym) {
    ti = t / nt;
    tj = t % nt;
    return;
  }
  int r = 0;
  while (t >= nt - r) {
    t -= nt - r;
    ++r;
  }
  ti = r;
  tj = r + t;
}

__device__ __forceinline__ void load_split32(const __half* hi, const __half* lo, float* out) {
  const uint4* h4 = reinterpret_cast<const uint4*>(hi);
  const uint4* l4 = reinterpret_cast<const uint4*>(lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 a = h4[q], b = l4[q];
    const __half2* ah = reinterpret_cast<const __half2*>(&a);
    const __half2* bh = reinterpret_cast<const __half2*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 x = __half22float2(ah[e]);
      float2 y = __half22float2(bh[e]);
      out[q * 8 + 2 * e] = x.x + y.x * kLoUnscale;
      out[q * 8 + 2 * e + 1] = x.y + y.y * kLoUnscale;
    }
  }
}

__device__ __forceinline__ void fail_timeout(volatile int* abort_flag, unsigned* status) {
  *abort_flag = 1;
  if (status) atomicOr(status, kStatusTimeout);
}

__global__ void __launch_bounds__(128, 1)
    gemm_split_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                      const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int which = (static_cast<int>(blockIdx.y) < args.op[0].nprob) ? 0 : 1;
  const int p = static_cast<int>(blockIdx.y) - (which ? args.op[0].nprob : 0);
  const GemmOp& g = args.op[which];
  const CUtensorMap* tmA = which ? &tmA1 : &tmA0;
  const CUtensorMap* tmB = which ? &tmB1 : &tmB0;
  const int nt = args.B / kTile;
  int ti, tj;
  tile_coords(blockIdx.x, nt, args.sym, ti, tj);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(tmB);
  }
  if (warp == 0) {
    tmem_alloc(tslot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  const int nk = args.B / kKBlk;
  const int am = at(g.a, p);
  const int bm = at(g.b, p);

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int kb = 0;
    for (; kb < nk; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (kb / kStages) & 1u;
      if (kb >= kStages && !mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
        fail_timeout(abort_flag, args.status);
        break;
      }
      uint8_t* st = smem + s * kStageBytes;
      mbar_arrive_expect_tx(&full[s], kStageBytes);
      tma_load_3d(st, tmA, &full[s], kb * kKBlk, ti * kTile, 2 * am);
      tma_load_3d(st + kTileBytes, tmA, &full[s], kb * kKBlk, ti * kTile, 2 * am + 1);
      tma_load_3d(st + 2 * kTileBytes, tmB, &full[s], kb * kKBlk, tj * kTile, 2 * bm);
      tma_load_3d(st + 3 * kTileBytes, tmB, &full[s], kb * kKBlk, tj * kTile, 2 * bm + 1);
    }
    if (*abort_flag) {
      // Let this CTA's own copies land before it can exit.
      volatile int never = 0;
      for (int j = (kb > kStages ? kb - kStages : 0); j < kb; ++j)
        mbar_wait(&full[j % kStages], (j / kStages) & 1u, &never);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (kb / kStages) & 1u;
      if (!mbar_wait(&full[s], ph, abort_flag)) {
        fail_timeout(abort_flag, args.status);
        break;
      }
      tc_fence_after();
      const uint32_t st = smem_u32(smem + s * kStageBytes);
#pragma unroll
      for (int kk = 0; kk < kKBlk / 16; ++kk) {
        const uint64_t ah = sw128_kmajor_desc(st + kk * 32);
        const uint64_t al = sw128_kmajor_desc(st + kTileBytes + kk * 32);
        const uint64_t bh = sw128_kmajor_desc(st + 2 * kTileBytes + kk * 32);
        const uint64_t bl = sw128_kmajor_desc(st + 3 * kTileBytes + kk * 32);
        const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
        mma_f16_ss(tbase, ah, bh, kIdesc, acc);
        mma_f16_ss(tbase + 128u, ah, bl, kIdesc, acc);
        mma_f16_ss(tbase + 128u, al, bh, kIdesc, 1u);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(done);  // also after an abort: fires once issued MMAs retire
  }
  __syncwarp();

  // ---------------- epilogue (all 128 threads; warp w owns rows 32w..32w+31)
  volatile int never = 0;
  const bool ok = mbar_wait(done, 0u, &never) && (*abort_flag == 0);
  if (!ok && threadIdx.x == 0) atomicOr(args.status, kStatusTimeout);
  tc_fence_after();
  __syncwarp();
  if (ok) {
    const int row = ti * kTile + warp * 32 + lane;
    const uint32_t trow = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    const size_t B = static_cast<size_t>(args.B);
    const size_t BB = B * B;
    const float s = g.scale ? g.scale[at(g.scale_i, p)] : 1.0f;
    const __half* cin = g.cin_split ? g.cin_split + static_cast<size_t>(at(g.cin_i, p)) * 2 * BB : nullptr;
    const float* cinf = g.cin_f32 ? g.cin_f32 + static_cast<size_t>(at(g.cinf_i, p)) * BB : nullptr;
    __half* os = g.out_split ? g.out_split + static_cast<size_t>(at(g.out_i, p)) * 2 * BB : nullptr;
    __half* ot = g.outt_split ? g.outt_split + static_cast<size_t>(at(g.outt_i, p)) * 2 * BB : nullptr;
    float* of = g.out_f32 ? g.out_f32 + static_cast<size_t>(at(g.outf_i, p)) * BB : nullptr;
    float* oft = g.outt_f32 ? g.outt_f32 + static_cast<size_t>(at(g.outtf_i, p)) * BB : nullptr;
    const bool mirror = args.sym && (ti != tj);
    BlockDesc bd;
    if (g.blocks) bd = g.blocks[p];
    bool bad = false;
    float sumsq = 0.0f;

    for (int cc = 0; cc < kTile / 32; ++cc) {
      uint32_t r0[32], r1[32];
      tmem_ld_32x32b_x32(trow + cc * 32, r0);
      tmem_ld_32x32b_x32(trow + 128u + cc * 32, r1);
      tmem_ld_wait();
      const int col0 = tj * kTile + cc * 32;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = g.alpha * (__uint_as_float(r0[j]) + __uint_as_float(r1[j]) * kLoUnscale);
      if (cin) {
        float c[32];
        if (g.cin_trans) {
#pragma unroll
          for (int j = 0; j < 32; ++j) c[j] = join_f16(cin[(col0 + j) * B + row], cin[BB + (col0 + j) * B + row]);
        } else {
          load_split32(cin + row * B + col0, cin + BB + row * B + col0, c);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += g.beta * c[j];
      }
      if (cinf) {
        const float4* c4 = reinterpret_cast<const float4*>(cinf + row * B + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 c = c4[q];
          v[4 * q] += g.beta * c.x;
          v[4 * q + 1] += g.beta * c.y;
          v[4 * q + 2] += g.beta * c.z;
          v[4 * q + 3] += g.beta * c.w;
        }
      }
      if (g.gamma != 0.0f) {
        const int d = row - col0;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j == d) v[j] += g.gamma;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] *= s;
        bad |= !isfinite(v[j]);
      }

      if (g.blocks) {
        if (row < bd.br) {
          float* dst = g.u_out + bd.off + static_cast<long long>(bd.r0 + row) * bd.pitch + bd.c0 + col0;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < bd.bc) {
              dst[j] = v[j];
              sumsq += v[j] * v[j];
            }
        }
        continue;
      }
      if (os || ot) {
        __half hi[32], lo[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          split_f16(v[j], hi[j], lo[j]);
          bad |= (__hisinf(hi[j]) != 0);
        }
        if (os) {
          uint4* dh = reinterpret_cast<uint4*>(os + row * B + col0);
          uint4* dl = reinterpret_cast<uint4*>(os + BB + row * B + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            dh[q] = *reinterpret_cast<const uint4*>(&hi[8 * q]);
            dl[q] = *reinterpret_cast<const uint4*>(&lo[8 * q]);
          }
          if (mirror) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              os[(col0 + j) * B + row] = hi[j];
              os[BB + (col0 + j) * B + row] = lo[j];
            }
          }
        }
        if (ot) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            ot[(col0 + j) * B + row] = hi[j];
            ot[BB + (col0 + j) * B + row] = lo[j];
          }
        }
      }
      if (of) {
        float4* d4 = reinterpret_cast<float4*>(of + row * B + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        if (mirror) {
#pragma unroll
          for (int j = 0; j < 32; ++j) of[(col0 + j) * B + row] = v[j];
        }
      }
      if (oft) {
#pragma unroll
        for (int j = 0; j < 32; ++j) oft[(col0 + j) * B + row] = v[j];
      }
    }
    if (bad) atomicOr(args.status, kStatusNonFinite);
    if (g.blocks) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
      if (lane == 0 && sumsq != 0.0f) atomicAdd(&g.unorm[p], sumsq);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_split(const OpBuffers* bufs, const GemmArgs& args, cudaStream_t stream) {
  if (args.nops < 1 || args.nops > 2) return cudaErrorInvalidValue;
  const int nprob = args.op[0].nprob + (args.nops == 2 ? args.op[1].nprob : 0);
  if (nprob <= 0) return cudaSuccess;
  if (args.B % kTile != 0 || args.B <= 0 || nprob > 65535) return cudaErrorInvalidValue;
  CUtensorMap maps[4];
  for (int o = 0; o < 2; ++o) {
    const OpBuffers& b = bufs[o < args.nops ? o : 0];
    cudaError_t e = encode_split_stack_map(&maps[2 * o], b.a, args.B, b.a_nmat);
    if (e != cudaSuccess) return e;
    e = encode_split_stack_map(&maps[2 * o + 1], b.b, args.B, b.b_nmat);
    if (e != cudaSuccess) return e;
  }
  GemmArgs a = args;
  if (a.nops == 1) a.op[1].nprob = 0;
  cudaError_t e = cudaFuncSetAttribute(gemm_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nt = a.B / kTile;
  const int tiles = a.sym ? nt * (nt + 1) / 2 : nt * nt;
  dim3 grid(tiles, nprob);
  // useful flops: each computed 128 x 128 tile is one 2*128*128*B product
  const double flops = 2.0 * kTile * kTile * static_cast<double>(a.B) * tiles * nprob;
  const int slot = prof_begin(kProfGemm, stream, flops);
  gemm_split_kernel<<<grid, 128, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], a);
  prof_end(slot, stream);
  prof_count_launch();
  return cudaGetLastError();
}

}  // namespace dash
