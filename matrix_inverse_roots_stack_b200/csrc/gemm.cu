// Batched split-fp16 GEMM on tcgen05 tensor cores (sm_100a), persistent and
// warp-specialised.
//
// Each CTA (one per SM) walks a static round-robin list of 128 x 128 output
// tiles of all problems of the launch.  Roles (320 threads):
//   warp 0, one lane   TMA producer: streams the A hi/lo and B hi/lo tiles of
//                      each 64-wide K slab into a 3-stage shared-memory ring
//                      (A always K-major; B K-major, or MN-major as two
//                      64-column boxes when the op multiplies by B itself);
//   warp 1, one lane   MMA issuer;
//   warps 2-9          epilogue; warp w reads tensor-memory lanes 32*(w%4)..
//                      and columns 64*((w-2)/4).. of each accumulator, so
//                      every thread owns 64 columns of one output row.
// Tensor memory (512 columns): a ring of three 128-column hi*hi accumulators
// and one 128-column lo accumulator.
//
// The tensor core's fp32 accumulation truncates (the bias grows linearly
// with the number of MMAs accumulated).  The hi*hi products, which carry the
// result's magnitude, are therefore accumulated in tensor memory over one
// flush segment only (args.flush K=16 MMAs, default one) and then added
// with round-to-nearest into fp32 registers of the epilogue warps (packed
// f32x2 adds), while the MMA warp fills the next ring buffer.  The hi*lo + lo*hi products enter the
// result scaled by 2^-11 and stay in tensor memory for the whole K range;
// they are read into the registers as soon as a tile's last MMA retires, so
// the next tile can start while the epilogue writes the previous one out.
#include "gemm.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

#include <atomic>

namespace dash {
namespace {

constexpr int kTile = 128;
constexpr int kKBlk = 64;                          // fp16 elements per 128-byte row
constexpr int kStages = 3;
constexpr int kTileBytes = kTile * kKBlk * 2;      // 16 KB
constexpr int kStageBytes = 4 * kTileBytes;        // A hi, A lo, B hi, B lo
#ifndef DASH_EPI_WARPS
#define DASH_EPI_WARPS 8
#endif
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = DASH_EPI_WARPS;          // 4 or 8
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kCols = kTile * 4 / kEpiWarps;       // accumulator columns per epilogue thread
constexpr int kRing = 3;                           // hi*hi accumulators
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColLO = kRing * 128;           // lo accumulator
#ifndef DASH_FLUSH_MMAS
#define DASH_FLUSH_MMAS 1
#endif
constexpr int kDefaultFlush = DASH_FLUSH_MMAS;     // K=16 MMAs per hi*hi flush

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t hh_full[kRing], hh_empty[kRing];
  uint64_t lo_full, lo_empty;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
};
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + static_cast<int>(sizeof(Bars)) + 64;

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

// Flattened tile index -> (op, problem, tile row, tile column).
__device__ __forceinline__ void decode(const GemmArgs& args, int tpp, int nt, long long t, int& op, int& p,
                                       int& ti, int& tj) {
  const long long n0 = static_cast<long long>(args.op[0].nprob) * tpp;
  op = t < n0 ? 0 : 1;
  const long long u = op ? t - n0 : t;
  p = static_cast<int>(u / tpp);
  tile_coords(static_cast<int>(u % tpp), nt, args.sym, ti, tj);
}

__device__ __forceinline__ void fail_timeout(volatile int* abort_flag, unsigned* status) {
  *abort_flag = 1;
  if (status) atomicOr(status, kStatusTimeout);
}

// Descriptor of an MN-major operand tile: 64 K-rows of 128 bytes per
// 64-column box, two boxes 8 KB apart (leading byte offset), 8-row swizzle
// atoms of 1024 bytes (stride byte offset), 128-byte swizzle.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(8192u >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ void store_split16(__half* base, size_t BB, size_t idx, const float* v, bool& bad) {
  __half hi[16], lo[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    split_f16(v[j], hi[j], lo[j]);
    bad |= (__hisinf(hi[j]) != 0);
  }
  uint4* dh = reinterpret_cast<uint4*>(base + idx);
  uint4* dl = reinterpret_cast<uint4*>(base + BB + idx);
  dh[0] = *reinterpret_cast<const uint4*>(&hi[0]);
  dh[1] = *reinterpret_cast<const uint4*>(&hi[8]);
  dl[0] = *reinterpret_cast<const uint4*>(&lo[0]);
  dl[1] = *reinterpret_cast<const uint4*>(&lo[8]);
}

// out(col0 + j, row) = v[j]: for a fixed j the 32 lanes (consecutive rows)
// write consecutive addresses.
__device__ __forceinline__ void store_split16_t(__half* base, size_t B, size_t BB, int row, int col0, const float* v,
                                                bool& bad) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    __half h, l;
    split_f16(v[j], h, l);
    bad |= (__hisinf(h) != 0);
    base[(col0 + j) * B + row] = h;
    base[BB + (col0 + j) * B + row] = l;
  }
}

// Raw 16-element chunk of a split row (hi and lo planes, 32 bytes each).
struct SplitChunk {
  uint4 h[2], l[2];
};

__device__ __forceinline__ SplitChunk ld_chunk(const __half* base, size_t BB, size_t idx) {
  SplitChunk c;
  const uint4* h4 = reinterpret_cast<const uint4*>(base + idx);
  const uint4* l4 = reinterpret_cast<const uint4*>(base + BB + idx);
  c.h[0] = h4[0];
  c.h[1] = h4[1];
  c.l[0] = l4[0];
  c.l[1] = l4[1];
  return c;
}

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

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// FL: K=16 MMAs per hi*hi flush segment (1, 2 or 4), or 0 for one segment per tile.
template <int FL>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_split_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                      const GemmArgs args, const long long total) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + kStages * kStageBytes);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = args.B / kTile;
  const int tpp = args.sym ? nt * (nt + 1) / 2 : nt * nt;
  const int nk = args.B / kKBlk;
  const int nseg = FL == 0 ? 1 : nk * (kKBlk / 16) / FL;  // flush segments per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < kRing; ++b) {
      mbar_init(&bars->hh_full[b], 1);
      mbar_init(&bars->hh_empty[b], kEpiWarps);
    }
    mbar_init(&bars->lo_full, 1);
    mbar_init(&bars->lo_empty, kEpiWarps);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t sc = 0, s = 0, epar = 1;  // loads issued, stage, parity of the stage's next release
      bool stop = args.skip_loads != 0;
      for (long long t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        int op, p, ti, tj;
        decode(args, tpp, nt, t, op, p, ti, tj);
        const GemmOp& g = args.op[op];
        const int am = at(g.a, p), bm = at(g.b, p);
        const CUtensorMap* ta = op ? &tmA1 : &tmA0;
        const CUtensorMap* tb = op ? &tmB1 : &tmB0;
        for (int kb = 0; kb < nk; ++kb, ++sc) {
          if (!mbar_wait(&bars->empty[s], epar, abort_flag)) {  // fresh barriers pass on parity 1
            fail_timeout(abort_flag, args.status);
            stop = true;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
          tma_load_3d(st, ta, &bars->full[s], kb * kKBlk, ti * kTile, 2 * am);
          tma_load_3d(st + kTileBytes, ta, &bars->full[s], kb * kKBlk, ti * kTile, 2 * am + 1);
          if (g.b_mn) {  // rows kb*64.. of B, columns tj*128.. as two 64-column boxes
#pragma unroll
            for (int pl = 0; pl < 2; ++pl) {
              uint8_t* dst = st + (2 + pl) * kTileBytes;
              tma_load_3d(dst, tb, &bars->full[s], tj * kTile, kb * kKBlk, 2 * bm + pl);
              tma_load_3d(dst + kTileBytes / 2, tb, &bars->full[s], tj * kTile + 64, kb * kKBlk, 2 * bm + pl);
            }
          } else {
            tma_load_3d(st + 2 * kTileBytes, tb, &bars->full[s], kb * kKBlk, tj * kTile, 2 * bm);
            tma_load_3d(st + 3 * kTileBytes, tb, &bars->full[s], kb * kKBlk, tj * kTile, 2 * bm + 1);
          }
          if (++s == kStages) {
            s = 0;
            epar ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let this CTA's own copies land before it can exit
        volatile int never = 0;
        for (uint32_t j = (sc > kStages ? sc - kStages : 0); j < sc; ++j)
          mbar_wait(&bars->full[j % kStages], (j / kStages) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // One thread issues every MMA of the CTA, so this loop is kept to a few
    // scalar instructions per K=16 step: descriptors are a base plus
    // compile-time offsets, ring positions advance without division, and
    // the release barriers start out passable (parity 1 on a fresh barrier).
    if (lane == 0) {
      const uint32_t sbase = smem_u32(smem);
      const uint64_t kd0 = sw128_kmajor_desc(sbase), md0 = sw128_mnmajor_desc(sbase);
      constexpr uint32_t kTileD = kTileBytes >> 4;  // descriptor address units
      uint32_t s = 0, fpar = 0;                     // stage, parity of its next fill
      uint32_t hb = 0, hpar = (1u << kRing) - 1u;   // hh buffer, parity bits of the next release per buffer
      uint32_t lpar = 1u;                           // parity of the lo accumulator's next release
      bool ok = true;
      const uint32_t lo_t = tbase + kColLO;
      for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int op, p, ti, tj;
        decode(args, tpp, nt, t, op, p, ti, tj);
        const bool bmn = args.op[op].b_mn != 0;
        const uint32_t idesc = f16_idesc(128, 128) | (bmn ? (1u << 16) : 0u);
        const uint64_t bd0 = (bmn ? md0 : kd0) + 2 * kTileD;
        const uint32_t bstep = bmn ? (2048u >> 4) : (32u >> 4);
        ok = mbar_wait(&bars->lo_empty, lpar, abort_flag);
        lpar ^= 1u;
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          ok = mbar_wait(&bars->full[s], fpar, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t so = s * (kStageBytes >> 4);
          const uint64_t ah = kd0 + so, al = ah + kTileD, bh = bd0 + so, bl = bh + kTileD;
#pragma unroll
          for (int kk = 0; kk < kKBlk / 16; ++kk) {
            const bool seg_start = FL == 0 ? (kb == 0 && kk == 0) : (kk % FL) == 0;
            const bool seg_end = FL == 0 ? (kb == nk - 1 && kk == kKBlk / 16 - 1) : (kk % FL) == FL - 1;
            if (seg_start) {
              ok = mbar_wait(&bars->hh_empty[hb], (hpar >> hb) & 1u, abort_flag);
              hpar ^= 1u << hb;
              if (!ok) break;
              tc_fence_after();
            }
            const uint32_t ka = 2u * kk, kbo = bstep * kk;
            mma_f16_ss(tbase + hb * 128u, ah + ka, bh + kbo, idesc, seg_start ? 0u : 1u);
            mma_f16_ss(lo_t, ah + ka, bl + kbo, idesc, (kb == 0 && kk == 0) ? 0u : 1u);
            mma_f16_ss(lo_t, al + ka, bh + kbo, idesc, 1u);
            if (seg_end) {
              mma_commit(&bars->hh_full[hb]);
              hb = hb == kRing - 1 ? 0u : hb + 1u;
            }
          }
          if (!ok) break;
          mma_commit(&bars->empty[s]);
          if (kb == nk - 1) mma_commit(&bars->lo_full);
          if (++s == kStages) {
            s = 0;
            fpar ^= 1u;
          }
        }
      }
      if (!ok) fail_timeout(abort_flag, args.status);
      // all issued MMAs must retire before tensor memory is released
      mma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0u, &never);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;  // tensor-memory lane quadrant of this warp
    const int half = (warp - kEpiWarp0) >> 2;
    const uint32_t lane_off = (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(half * kCols);
    const size_t B = static_cast<size_t>(args.B);
    const size_t BB = B * B;
    uint32_t hb = 0, hpar = 0, lpar = 0;  // hh buffer and fill parities, lo fill parity
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      int op, p, ti, tj;
      decode(args, tpp, nt, t, op, p, ti, tj);
      const GemmOp& g = args.op[op];
      const int row = ti * kTile + quad * 32 + lane;
      const int cbase = tj * kTile + half * kCols;
      {  // pull this thread's Cin row segment into L2 while the mainloop runs
        const size_t prow = static_cast<size_t>(row) * B + static_cast<size_t>(cbase);
        if (g.cin_split && !g.cin_trans) {
          const __half* cb = g.cin_split + static_cast<size_t>(at(g.cin_i, p)) * 2 * BB + prow;
          prefetch_l2(cb);
          prefetch_l2(cb + BB);
        }
        if (g.cin_f32) {
          const float* cb = g.cin_f32 + static_cast<size_t>(at(g.cinf_i, p)) * BB + prow;
          prefetch_l2(cb);
          prefetch_l2(cb + 32);
        }
      }
      float S[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) S[j] = 0.0f;

      bool ok = true;
      for (int sg = 0; sg < nseg; ++sg) {
        // epilogue warps sleep in the barrier while they wait, leaving the
        // issue slots of their scheduler to the MMA and TMA threads
        if (!mbar_wait_sleep(&bars->hh_full[hb], (hpar >> hb) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        hpar ^= 1u << hb;
        tc_fence_after();
        const uint32_t src = tbase + lane_off + hb * 128u;
#pragma unroll
        for (int c = 0; c < kCols / 64; ++c) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(src + 64 * c, r0);
          tmem_ld_32x32b_x32(src + 64 * c + 32, r1);
          tmem_ld_wait();
          if (c + 1 == kCols / 64) {  // registers hold the whole segment now
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->hh_empty[hb]);
            hb = hb == kRing - 1 ? 0u : hb + 1u;
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
#ifdef DASH_PLAIN_FADD
            S[64 * c + j] += __uint_as_float(r0[j]);
            S[64 * c + j + 1] += __uint_as_float(r0[j + 1]);
            S[64 * c + 32 + j] += __uint_as_float(r1[j]);
            S[64 * c + 32 + j + 1] += __uint_as_float(r1[j + 1]);
#else
            add_f32x2(S[64 * c + j], S[64 * c + j + 1], r0[j], r0[j + 1]);
            add_f32x2(S[64 * c + 32 + j], S[64 * c + 32 + j + 1], r1[j], r1[j + 1]);
#endif
          }
        }
      }
      if (ok) {
        ok = mbar_wait_sleep(&bars->lo_full, lpar, abort_flag);
        lpar ^= 1u;
      }
      if (!ok) {
        if (threadIdx.x == kEpiWarp0 * 32) fail_timeout(abort_flag, args.status);
        break;
      }
      tc_fence_after();
      {
        const uint32_t src = tbase + lane_off + kColLO;
#pragma unroll
        for (int h = 0; h < kCols / 32; ++h) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(src + 32 * h, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) S[32 * h + j] += __uint_as_float(r[j]) * kLoUnscale;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->lo_empty);  // the next tile may start accumulating
      }

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
      const bool cin_rows = cin && !g.cin_trans;
      SplitChunk nxt;
      if (cin_rows) nxt = ld_chunk(cin, BB, row * B + cbase);

#pragma unroll
      for (int c = 0; c < kCols / 16; ++c) {
        const int col0 = cbase + c * 16;
        float* v = &S[c * 16];  // finished in place
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] *= g.alpha;
        if (cin_rows) {  // this chunk's Cin was loaded one chunk ahead
          const SplitChunk cur = nxt;
          if (c + 1 < kCols / 16) nxt = ld_chunk(cin, BB, row * B + col0 + 16);
          float cj[16];
          join_chunk(cur, cj);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] += g.beta * cj[j];
        } else if (cin) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            v[j] += g.beta * join_f16(cin[(col0 + j) * B + row], cin[BB + (col0 + j) * B + row]);
        }
        if (cinf) {
          const float4* c4 = reinterpret_cast<const float4*>(cinf + row * B + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 cq = c4[q];
            v[4 * q] += g.beta * cq.x;
            v[4 * q + 1] += g.beta * cq.y;
            v[4 * q + 2] += g.beta * cq.z;
            v[4 * q + 3] += g.beta * cq.w;
          }
        }
        if (g.gamma != 0.0f) {
          const int d = row - col0;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j == d) v[j] += g.gamma;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          v[j] *= s;
          bad |= !isfinite(v[j]);
        }
        if (g.blocks) {
          if (row < bd.br) {
            float* dst = g.u_out + bd.off + static_cast<long long>(bd.r0 + row) * bd.pitch + bd.c0 + col0;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (col0 + j < bd.bc) {
                dst[j] = v[j];
                sumsq += v[j] * v[j];
              }
          }
          continue;
        }
        if (os) {
          store_split16(os, BB, row * B + col0, v, bad);
          if (mirror) store_split16_t(os, B, BB, row, col0, v, bad);
        }
        if (ot) store_split16_t(ot, B, BB, row, col0, v, bad);
        if (of) {
          float4* d4 = reinterpret_cast<float4*>(of + row * B + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          if (mirror) {
#pragma unroll
            for (int j = 0; j < 16; ++j) of[(col0 + j) * B + row] = v[j];
          }
        }
        if (oft) {
#pragma unroll
          for (int j = 0; j < 16; ++j) oft[(col0 + j) * B + row] = v[j];
        }
      }
      if (bad) atomicOr(args.status, kStatusNonFinite);
      if (g.blocks) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
        if (lane == 0 && sumsq != 0.0f) atomicAdd(&g.unorm[p], sumsq);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

std::atomic<int> g_load_fault{0};

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

}  // namespace

cudaError_t launch_gemm_split(const OpBuffers* bufs, const GemmArgs& args, cudaStream_t stream) {
  if (args.nops < 1 || args.nops > 2) return cudaErrorInvalidValue;
  const int nprob = args.op[0].nprob + (args.nops == 2 ? args.op[1].nprob : 0);
  if (nprob <= 0) return cudaSuccess;
  if (args.B % kTile != 0 || args.B <= 0) return cudaErrorInvalidValue;
  GemmArgs a = args;
  if (a.nops == 1) a.op[1] = a.op[0], a.op[1].nprob = 0;
  if (g_load_fault.exchange(0) != 0) a.skip_loads = 1;
  CUtensorMap maps[4];
  for (int o = 0; o < 2; ++o) {
    const OpBuffers& b = bufs[o < args.nops ? o : 0];
    cudaError_t e = encode_split_stack_map(&maps[2 * o], b.a, a.B, b.a_nmat, 128);
    if (e != cudaSuccess) return e;
    e = encode_split_stack_map(&maps[2 * o + 1], b.b, a.B, b.b_nmat, a.op[o].b_mn ? 64 : 128);
    if (e != cudaSuccess) return e;
  }
  const int nm = (a.B / kKBlk) * (kKBlk / 16);  // K=16 MMAs per tile
  if (a.flush <= 0) a.flush = kDefaultFlush;
  void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const GemmArgs,
               const long long) = a.flush >= nm  ? gemm_split_kernel<0>
                                  : a.flush >= 4 ? gemm_split_kernel<4>
                                  : a.flush >= 2 ? gemm_split_kernel<2>
                                                 : gemm_split_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nt = a.B / kTile;
  const long long tpp = a.sym ? nt * (nt + 1) / 2 : nt * nt;
  const long long total = tpp * nprob;
  const long long sms = sm_count();
  const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
  // useful flops: each computed 128 x 128 tile is one 2*128*128*B product
  const double flops = 2.0 * kTile * kTile * static_cast<double>(a.B) * static_cast<double>(total);
  const int slot = prof_begin(kProfGemm, stream, flops);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], a, total);
  prof_end(slot, stream);
  prof_count_launch();
  return cudaGetLastError();
}

void arm_load_fault() { g_load_fault.store(1); }

}  // namespace dash
