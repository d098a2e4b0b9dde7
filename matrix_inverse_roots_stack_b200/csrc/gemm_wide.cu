// Batched split-fp16 GEMM with 128 x 256 output tiles (sm_100a), for
// launches whose block size is a multiple of 256 (split-fp16 products, or
// single-pass fp16 products for the fp16 coupled Newton; symmetric launches
// take the tiles that reach the upper triangle).
//
// Split-fp16 products as in gemm.cu (hi*lo + lo*hi into a fresh
// tensor-memory buffer, then hi*hi with that buffer scaled by 2^-11), with a
// tile twice as wide and one buffer per two K=16 steps instead of per step:
// the buffer takes the cross terms of both steps, then hi*hi of the first
// step plus 2^-11 times them, then hi*hi of the second, and the buffer's fp32
// product is added into fp32 registers with round-to-nearest.  Every
// tensor-core accumulation rounds toward zero once per MMA, relative to the
// running partial sum in the buffer; with two steps per buffer that partial
// is at most twice a step's, which measured within 10% of per-step adds on
// the update error of blocks with condition numbers near 1e8, while four
// steps per buffer raised it by about 1.7x.  Two steps halve the register
// flush work (loads from tensor memory and fp32 adds) per product.
// Every MMA issues as much tensor work as it can (M=128, N=256); a buffer's
// fp32 product takes 256 of the 512 tensor-memory columns, so the ring holds
// two buffers and there is no room to park a finished tile.  The accumulator
// warps therefore write their own tile out.
//
// Shared memory: two 96 KB operand stages, 32 KB of epilogue staging (4 KB
// per accumulator warp; stage 1 lends 12 KB more per warp during a tile's
// epilogue), the barriers (about 225 KB of the 227 KB a block may hold).
//
// Roles (384 threads = three warpgroups, one CTA per SM, persistent over a
// static round-robin list of the launch's tiles):
//   warps 0-7          accumulators (warpgroups 0 and 1): warp w reads
//                      lanes 32*(w%4).. and 128 of the 256 columns, so each
//                      thread sums 128 columns of one output row in
//                      registers; at the end of a tile the same thread applies
//                      the epilogue to its row segment, in four steps of 32
//                      columns.  Each step leaves through a 4 KB shared-memory
//                      buffer and one TMA tensor store (a store instruction
//                      whose 32 lanes each write a different row would touch
//                      32 lines); its Cin arrives in the same buffer by TMA.
//   warp 8, one lane   TMA producer: A hi/lo (128 x 64) and B hi/lo
//                      (256 x 64, or four 64 x 64 boxes when B is read
//                      MN-major) of each 64-wide K slab into a 2-stage ring
//                      of 96 KB stages.  No multicast.
//   warp 9, one lane   MMA issuer: six tcgen05.mma kind::f16 per two K=16
//                      steps into one of two 256-column tensor-memory buffers.
//   warps 10-11        idle (they complete warpgroup 2).
// Register split: the kernel is launched at 168 registers a thread (384 x
// 168 = 64,512 of the SM's 65,536); warpgroup 2 gives registers back with
// setmaxnreg.dec to 72 and the accumulator warpgroups take them with
// setmaxnreg.inc to 216: 2 x 128 x 216 + 128 x 72 = 64,512, the launch's
// total, and per scheduler (warps w, w+4, w+8) 2 x 32 x 216 + 32 x 72 =
// 16,128 of 16,384.  The host launches the kernel only when it was compiled
// at exactly 168 registers, so the increase can always be granted.
#include "gemm.cuh"
#include "gemm_common.cuh"
#include "launch_util.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

#include <atomic>
#include <cstring>

namespace dash {
namespace {

constexpr int kM = 128, kN = 256;
constexpr int kKBlk = 64;                              // fp16 elements per 128-byte row
constexpr int kABytes = kM * kKBlk * 2;                // 16 KB per plane and slab
constexpr int kBBytes = kN * kKBlk * 2;                // 32 KB per plane and slab
constexpr int kStageBytes = 2 * kABytes + 2 * kBBytes;  // A hi, A lo, B hi, B lo
constexpr int kStages = 2;
constexpr int kRing = 2;                               // product buffers of kN columns
constexpr int kChunk = 32;                             // columns per tensor-memory load batch of a flush
constexpr uint32_t kTmemCols = 512;
constexpr int kAccWarps = 8;                           // warps 0-7
constexpr int kProdWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;                       // registers a thread at launch (65536 / 384, rounded to 8)
constexpr int kLowRegs = 72, kHighRegs = 216;          // after setmaxnreg: warpgroup 2 / warpgroups 0-1
static_assert(2 * 128 * kHighRegs + 128 * kLowRegs <= kThreads * kLaunchRegs, "register split exceeds the launch");
static_assert(2 * 32 * kHighRegs + 32 * kLowRegs <= 16384, "register split exceeds a scheduler's file");
constexpr int kCols = 128;                             // columns summed per accumulator thread
constexpr int kPrefetchSlabs = 2;                      // 64-wide K slabs before a tile's end when its Cin is prefetched

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[kRing], acc_empty[kRing];
  uint64_t drain;
  uint64_t stg_free;              // a tile's epilogue no longer uses operand stage 1
  uint64_t cin0_full[kAccWarps];  // Cin of a warp's first epilogue step has landed in its own buffer
  uint64_t cin_full[kAccWarps];   // Cin of its other three steps has landed in stage 1
  uint32_t tmem_slot;
  int abort;
};
// Epilogue staging: an epilogue step covers 32 rows x 32 columns of a warp's
// row segment, 4 KB as split fp16 (both planes) or fp32.  Each accumulator
// warp owns one 4 KB buffer in a region of its own (the 32 KB after the
// operand stages) and, while its epilogue runs, three more in operand stage
// 1 (12 KB of its 96 KB): one buffer per step of its 128-column segment.
// Stage 1 is free then: a tile's last K slab has been read from it (K
// slabs alternate between the stages and every tile has an even number),
// and the producer loads the next tile's second slab into it only after
// every warp's epilogue has released it (stg_free).  The MMA cannot run
// ahead meanwhile anyway: its other tensor-memory buffer still holds the
// finished tile.
constexpr int kStageBufBytes = 4096;
constexpr int kStagingOff = kStages * kStageBytes;
constexpr int kBarsOff = kStagingOff + kAccWarps * kStageBufBytes;
static_assert(kStages == 2 && kAccWarps * 3 * kStageBufBytes <= kStageBytes, "borrowed staging exceeds a stage");
constexpr int kSmemBytes = kBarsOff + 1024 + static_cast<int>(sizeof(Bars)) + 64;
static_assert(kSmemBytes <= 232448, "shared memory exceeds the per-block limit");


// Tiles of one problem.  Symmetric launches take the 128 x 256 tiles that
// reach the upper triangle, 2 tj + 1 >= ti in 128-column units: row ti has
// ntn - ti/2 of them.
__host__ __device__ __forceinline__ int wide_tiles_per_problem(int B, int sym) {
  const int ntm = B / 128, ntn = B / 256;
  if (!sym) return ntm * ntn;
  int n = 0;
  for (int ti = 0; ti < ntm; ++ti) n += ntn - ti / 2;
  return n;
}

// Flattened tile index -> (op, problem, tile row, tile column); the two ops
// of a problem are adjacent when both ops have the same problems.
__device__ __forceinline__ void decode_wide(const GemmArgs& args, int tpp, int ntn, long long t, int& op, int& p,
                                            int& ti, int& tj) {
  int r;
  if (args.op[1].nprob == args.op[0].nprob) {
    const long long pair = 2ll * tpp;
    p = static_cast<int>(t / pair);
    r = static_cast<int>(t - static_cast<long long>(p) * pair);
    op = r >= tpp ? 1 : 0;
    if (op) r -= tpp;
  } else {
    const long long n0 = static_cast<long long>(args.op[0].nprob) * tpp;
    op = t < n0 ? 0 : 1;
    const long long u = op ? t - n0 : t;
    p = static_cast<int>(u / tpp);
    r = static_cast<int>(u % tpp);
  }
  if (!args.sym) {
    ti = r / ntn;
    tj = r % ntn;
    return;
  }
  int row = 0;
  while (r >= ntn - row / 2) {
    r -= ntn - row / 2;
    ++row;
  }
  ti = row;
  tj = row / 2 + r;
}

// This CTA's tile in round k of the launch's static schedule.  Round k
// covers tiles k*G .. k*G + G - 1 (G CTAs), and a CTA's place in the round
// moves by one each round, so tiles that recur at fixed places in every
// problem's tile list (the half-width tiles of symmetric launches) are
// spread over all CTAs instead of falling to the same few.  A result at or
// past the launch's total is a place in the last round with no tile.
__device__ __forceinline__ long long round_tile(long long k) {
  const long long g = gridDim.x;
  return k * g + (static_cast<long long>(blockIdx.x) + k) % g;
}

// L2 prefetch of one row segment [cbase, cbase + kCols) of problem p's Cin
// (split hi and lo planes, or fp32): 128-byte lines, no registers held.
__device__ __forceinline__ void prefetch_cin_l2(const GemmOp& g, int p, size_t B, size_t BB, int row, int cbase) {
  if (g.cin_split) {
    const __half* c = g.cin_split + static_cast<size_t>(gemm_at(g.cin_i, p)) * 2 * BB + row * B + cbase;
#pragma unroll
    for (int i = 0; i < kCols * 2; i += 128) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(c) + i));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(c + BB) + i));
    }
  } else if (g.cin_f32) {
    const float* c = g.cin_f32 + static_cast<size_t>(gemm_at(g.cinf_i, p)) * BB + row * B + cbase;
#pragma unroll
    for (int i = 0; i < kCols * 4; i += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(c) + i));
  }
}

template <bool kSingle>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_wide_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                     const __grid_constant__ OutMaps om, const GemmArgs args, const long long total) {
  constexpr int kFillSteps = kSingle ? 4 : 2;          // K=16 steps a buffer takes before its flush
  constexpr int kFills = kKBlk / 16 / kFillSteps;      // buffer fills per K slab
  static_assert(kFills * kFillSteps * 16 == kKBlk, "fills must tile the K slab");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarsOff);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = args.B / kN;
  const int tpp = wide_tiles_per_problem(args.B, args.sym);
  const int nk = args.B / kKBlk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < kRing; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], kAccWarps);
    }
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->stg_free, kAccWarps);
    for (int w = 0; w < kAccWarps; ++w) {
      mbar_init(&bars->cin0_full[w], 1);
      mbar_init(&bars->cin_full[w], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_slot;

  // each warpgroup changes its register count at one instruction that
  // dominates its roles (warpgroup 2: producer, MMA issuer, two idle warps)
  if (warp >= kProdWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == kProdWarp && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
      uint32_t sc = 0, s = 0, epar = 1;  // loads issued, stage, parity of the stage's next release
      uint32_t fpar = 0;                 // parity of the next stg_free phase
      bool stop = args.skip_loads != 0;
      bool first = true;
      for (long long k = 0; k * gridDim.x < total && !stop; ++k) {
        const long long t = round_tile(k);
        if (t >= total) continue;
        const bool after_epilogue = !first;  // stage 1 holds the previous tile's epilogue staging
        first = false;
        int op, p, ti, tj;
        decode_wide(args, tpp, ntn, t, op, p, ti, tj);
        const GemmOp& g = args.op[op];
        const int am = gemm_at(g.a, p), bm = gemm_at(g.b, p);
        const CUtensorMap* ta = op ? &tmA1 : &tmA0;
        const CUtensorMap* tb = op ? &tmB1 : &tmB0;
        for (int kb = 0; kb < nk; ++kb, ++sc) {
          if (!mbar_wait(&bars->empty[s], epar, abort_flag)) {  // fresh barriers pass on parity 1
            gemm_fail_timeout(abort_flag, args.status);
            stop = true;
            break;
          }
          if (kb == 1 && after_epilogue) {  // slab 1 goes to stage 1 (nk is even)
            if (!mbar_wait(&bars->stg_free, fpar, abort_flag)) {
              gemm_fail_timeout(abort_flag, args.status);
              stop = true;
              break;
            }
            fpar ^= 1u;
          }
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&bars->full[s], kSingle ? kABytes + kBBytes : kStageBytes);
          tma_load_3d(st, ta, &bars->full[s], kb * kKBlk, ti * kM, 2 * am);
          if (!kSingle) tma_load_3d(st + kABytes, ta, &bars->full[s], kb * kKBlk, ti * kM, 2 * am + 1);
#pragma unroll
          for (int pl = 0; pl < (kSingle ? 1 : 2); ++pl) {
            uint8_t* dst = st + 2 * kABytes + pl * kBBytes;
            if (g.b_mn) {  // rows kb*64.. of B, columns tj*256.. as four 64-column boxes
#pragma unroll
              for (int q = 0; q < 4; ++q)
                tma_load_3d(dst + q * (kBBytes / 4), tb, &bars->full[s], tj * kN + 64 * q, kb * kKBlk, 2 * bm + pl);
            } else {
              tma_load_3d(dst, tb, &bars->full[s], kb * kKBlk, tj * kN, 2 * bm + pl);
            }
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
    } else if (warp == kMmaWarp && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
      const uint32_t sbase = smem_u32(smem);
      const uint64_t kd0 = sw128_kmajor_desc(sbase), md0 = sw128_mnmajor_desc(sbase);
      constexpr uint32_t kAD = kABytes >> 4, kBD = kBBytes >> 4;  // descriptor address units
      uint32_t s = 0, fpar = 0;                   // stage, parity of its next fill
      uint32_t hb = 0, hpar = (1u << kRing) - 1u;  // ring buffer, parity bits of the next release per buffer
      bool ok = true;
      for (long long k = 0; k * gridDim.x < total && ok; ++k) {
        const long long t = round_tile(k);
        if (t >= total) continue;
        int op, p, ti, tj;
        decode_wide(args, tpp, ntn, t, op, p, ti, tj);
        const bool bmn = args.op[op].b_mn != 0;
        // a symmetric launch keeps nothing of a tile's left half below the
        // diagonal (the first tile of an odd tile row): its MMAs compute the
        // right half only (N=128, B rows 128.., tensor-memory columns 128..)
        const bool half = args.sym && 2 * tj < ti;
        const uint32_t idesc = f16_idesc(kM, half ? kN / 2 : kN) | (bmn ? (1u << 16) : 0u);
        const uint64_t bd0 = (bmn ? md0 : kd0) + 2 * kAD + (half ? (kBBytes / 2) >> 4 : 0);
        const uint32_t dcol = half ? kN / 2 : 0;
        const uint32_t bstep = bmn ? (2048u >> 4) : (32u >> 4);
        for (int kb = 0; kb < nk; ++kb) {
          ok = mbar_wait(&bars->full[s], fpar, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t so = s * (kStageBytes >> 4);
          const uint64_t ah = kd0 + so, al = ah + kAD, bh = bd0 + so, bl = bh + kBD;
#pragma unroll
          for (int f = 0; f < kFills; ++f) {
            ok = mbar_wait(&bars->acc_empty[hb], (hpar >> hb) & 1u, abort_flag);
            hpar ^= 1u << hb;
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tbase + hb * kN + dcol;
            const int k0 = f * kFillSteps;
            if (kSingle) {  // hi*hi of the slab's four steps into a fresh buffer
#pragma unroll
              for (int kk = k0; kk < k0 + kFillSteps; ++kk)
                mma_f16_ss(d, ah + 2u * kk, bh + bstep * kk, idesc, kk > k0 ? 1u : 0u);
            } else {
              // cross terms hi*lo + lo*hi of the fill's K=16 steps into a
              // fresh buffer, then hi*hi of its first step plus 2^-11 times
              // that sum, then hi*hi of its other steps
#pragma unroll
              for (int kk = k0; kk < k0 + kFillSteps; ++kk) {
                mma_f16_ss(d, ah + 2u * kk, bl + bstep * kk, idesc, kk > k0 ? 1u : 0u);
                mma_f16_ss(d, al + 2u * kk, bh + bstep * kk, idesc, 1u);
              }
              mma_f16_ss_acc_down11(d, ah + 2u * k0, bh + bstep * k0, idesc);
#pragma unroll
              for (int kk = k0 + 1; kk < k0 + kFillSteps; ++kk)
                mma_f16_ss(d, ah + 2u * kk, bh + bstep * kk, idesc, 1u);
            }
            mma_commit(&bars->acc_full[hb]);
            hb ^= 1u;
          }
          if (!ok) break;
          mma_commit(&bars->empty[s]);
          if (++s == kStages) {
            s = 0;
            fpar ^= 1u;
          }
        }
      }
      if (!ok) gemm_fail_timeout(abort_flag, args.status);
      // all issued MMAs must retire before tensor memory is released
      mma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0u, &never);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    // ---------------------------------------------------------------- accumulators + epilogue
    const int quad = warp & 3;  // tensor-memory lane quadrant of this warp
    const int cgrp = warp >> 2;  // 128-column half of the tile
    const uint32_t lane_off = (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(cgrp * kCols);
    const size_t B = static_cast<size_t>(args.B);
    const size_t BB = B * B;
    uint32_t hb = 0, hpar = 0;  // ring buffer, its fill parities
    uint32_t cpar = 0;          // parity of this warp's next Cin arrivals (both barriers)
    bool cin0_pending = false;  // a Cin load of this warp has not been waited for (own buffer,
    bool cin_pending = false;   // stage 1)
    bool ok = true;
    for (long long k = 0; k * gridDim.x < total && ok; ++k) {
      const long long t = round_tile(k);
      if (t >= total) continue;
      float S[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) S[j] = 0.0f;
      // Cin of this thread's row segment is fetched into L2 a few slabs
      // before the epilogue needs it (no registers held)
      int op, p, ti, tj;
      decode_wide(args, tpp, ntn, t, op, p, ti, tj);
      const GemmOp& g = args.op[op];
      const int row = ti * kM + quad * 32 + lane;
      const int cbase = tj * kN + cgrp * kCols;
      const int nfill = nk * kFills;
      const int pf_fill = nk > kPrefetchSlabs ? (nk - kPrefetchSlabs) * kFills : 0;
      // fill sg of the tile: S += its product (the last fill's sums go back
      // into its buffer for the epilogue instead of releasing it)
      // the epilogue's first step takes its Cin from the warp's own buffer
      // (free since the previous epilogue), loaded while the last slabs run
      const int q = 2 * tj + cgrp;
      const bool write = !args.sym || q >= ti;
      const bool cin = write && !g.blocks && (g.cin_split || g.cin_f32);
      uint8_t* const own = smem + kStagingOff + warp * kStageBufBytes;
      uint8_t* const borrowed = smem + kStageBytes + warp * 3 * kStageBufBytes;
      const int row0 = ti * kM + quad * 32;  // first row of this warp's steps
      const int zc = g.cin_split ? 2 * gemm_at(g.cin_i, p) : gemm_at(g.cinf_i, p);
      for (int sg = 0; sg < nfill; ++sg) {
        if (sg == pf_fill) {
          prefetch_cin_l2(g, p, B, BB, row, cbase);
          if (cin) {
            if (lane == 0) {
              mbar_arrive_expect_tx(&bars->cin0_full[warp], kStageBufBytes);
              tma_load_3d(own, &om.cin[op], &bars->cin0_full[warp], cbase, row0, zc);
            }
            cin0_pending = true;
          }
        }
        // waiting warps sleep in the barrier, leaving the issue slots of
        // their scheduler to the MMA and TMA threads
        if (!mbar_wait_sleep(&bars->acc_full[hb], (hpar >> hb) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        hpar ^= 1u << hb;
        tc_fence_after();
        if (!write) {  // nothing of this half is kept (and the MMA may not have written it)
          if (sg + 1 < nfill) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
            hb ^= 1u;
          }
          continue;
        }
        const uint32_t src = tbase + lane_off + hb * kN;
        if (sg + 1 < nfill) {
#pragma unroll
          for (int c = 0; c < kCols / kChunk; ++c) {
            uint32_t r[kChunk];
#pragma unroll
            for (int q = 0; q < kChunk / 16; ++q) tmem_ld_32x32b_x16(src + kChunk * c + 16 * q, r + 16 * q);
            tmem_ld_wait_regs<kChunk>(r);
            if (c + 1 == kCols / kChunk) {  // registers hold the whole fill now
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
            }
#pragma unroll
            for (int j = 0; j < kChunk; j += 2) add_f32x2(S[kChunk * c + j], S[kChunk * c + j + 1], r[j], r[j + 1]);
          }
          hb ^= 1u;
        } else {
#pragma unroll
          for (int c = 0; c < kCols / 16; ++c) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(src + 16 * c, r);
            tmem_ld_wait_regs<16>(r);
#pragma unroll
            for (int j = 0; j < 16; j += 2) add_f32x2(S[16 * c + j], S[16 * c + j + 1], r[j], r[j + 1]);
            tmem_st_32x32b_x16(src + 16 * c, &S[16 * c]);
          }
        }
      }
      if (!ok) {
        if (lane == 0) gemm_fail_timeout(abort_flag, args.status);
        break;
      }
      tmem_st_wait();
      // epilogue of this thread's row segment (128 columns) from the buffer
      // holding the finished sums, in four steps of 32 columns
      const uint32_t src = tbase + lane_off + hb * kN;
      // symmetric launches: this 128-column block q of the tile row ti is
      // written if q >= ti, and mirrored if q > ti (q < ti comes from the
      // mirror of block (q, ti))
      const bool mirror = args.sym && q > ti;
      GemmEpilogue ep;
      ep.init(g, p, B, BB);
      bool released = false;  // tensor-memory buffer handed back to the MMA
      if (write) {
        // step k stages in its own buffer, into which its Cin (split or
        // fp32) arrives by TMA first: no waits on earlier stores.  Steps
        // 1-3 use stage 1, free now that the tile's MMAs are done.
        if (cin) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars->cin_full[warp], 3 * kStageBufBytes);
#pragma unroll
            for (int k = 1; k < 4; ++k)
              tma_load_3d(borrowed + (k - 1) * kStageBufBytes, &om.cin[op], &bars->cin_full[warp], cbase + 32 * k,
                          row0, zc);
          }
          cin_pending = true;
        }
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          const int col0 = cbase + 32 * k;
          uint8_t* buf = k == 0 ? own : borrowed + (k - 1) * kStageBufBytes;
          float v[2][16];
          tmem_ld_32x32b_x16(src + 32 * k, reinterpret_cast<uint32_t*>(v[0]));
          tmem_ld_32x32b_x16(src + 32 * k + 16, reinterpret_cast<uint32_t*>(v[1]));
          tmem_ld_wait_regs<32>(reinterpret_cast<uint32_t*>(v));
          if (k == 3) {  // every tensor-memory read of the tile is done
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
            released = true;
          }
          if (cin && k < 2) {
            if (!mbar_wait_sleep(k == 0 ? &bars->cin0_full[warp] : &bars->cin_full[warp], cpar, abort_flag)) {
              ok = false;
              break;
            }
            if (k == 0) {
              cin0_pending = false;
            } else {
              cpar ^= 1u;
              cin_pending = false;
            }
          }
          // each lane reads, and below rewrites, only its own row of buf
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float cj[16];
            if (cin) {
              if (ep.cin) read_cin_chunk(buf, lane, h, cj);
              else read_cin_f32_chunk(buf, lane, h, cj);
            }
            ep.apply(row, col0 + 16 * h, v[h], cj);
          }
          if (ep.scatter) {
            ep.check_finite(v[0]);
            ep.check_finite(v[1]);
            ep.scatter_chunk(g, row, col0, v[0]);
            ep.scatter_chunk(g, row, col0 + 16, v[1]);
            continue;
          }
          // a mirrored step also goes out transposed (rows col0.., columns
          // row0..) through the same buffer, once the store before it has
          // read the buffer
          if (ep.os) {
            float w[2][16];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int j = 0; j < 16; ++j) w[h][j] = v[h][j] * ep.ss;
            stage_split32(buf, lane, w, ep.bad);
            store_step(lane, &om.split[op], buf, col0, row0, 2 * gemm_at(g.out_i, p));
            if (mirror) {
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
              stage_split32_t(buf, lane, w);
              store_step(lane, &om.split[op], buf, row0, col0, 2 * gemm_at(g.out_i, p));
            }
          }
          if (ep.of) {
            ep.check_finite(v[0]);
            ep.check_finite(v[1]);
            if (ep.os) {  // the split stores must have read buf first
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
            }
            stage_f32x32(buf, lane, v);
            store_step(lane, &om.f32[op], buf, col0, row0, gemm_at(g.outf_i, p));
            if (mirror) {
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
              stage_f32x32_t(buf, lane, v);
              store_step(lane, &om.f32[op], buf, row0, col0, gemm_at(g.outf_i, p));
            }
          }
        }
        if (!ok) {
          if (lane == 0) gemm_fail_timeout(abort_flag, args.status);
          break;
        }
      }
      ep.finish(g, p, args.status);
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
      }
      // the staging buffers (own, and the borrowed part of stage 1) are
      // free once this warp's stores have read them
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->stg_free);
      hb ^= 1u;
    }
    // a Cin load still in flight after an abort lands before the CTA exits
    if (lane == 0) {
      volatile int never = 0;
      if (cin0_pending) mbar_wait(&bars->cin0_full[warp], cpar, &never);
      if (cin_pending) mbar_wait(&bars->cin_full[warp], cpar, &never);
    }
    // this warp's tensor stores complete before the CTA's shared memory goes
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Registers a thread of gemm_wide_kernel was compiled with (once per
// process): the count both instantiations share, or 0 if they differ.
int wide_kernel_regs() {
  static std::atomic<int> regs{-1};
  int r = regs.load();
  if (r < 0) {
    cudaFuncAttributes f0, f1;
    const bool ok = cudaFuncGetAttributes(&f0, gemm_wide_kernel<false>) == cudaSuccess &&
                    cudaFuncGetAttributes(&f1, gemm_wide_kernel<true>) == cudaSuccess;
    r = ok && f0.numRegs == f1.numRegs ? f0.numRegs : 0;
    regs.store(r);
  }
  return r;
}

// One past the largest matrix index that problems [0, nprob) of an op
// reach through i (the host mirror of gemm_at).
long long idx_extent(const Idx& i, int nprob) {
  const long long st = i.stride > 0 ? i.stride : 1;
  const long long n = i.mod > 0 && i.mod < nprob ? i.mod : nprob;
  return i.base + st * (n - 1) + 1;
}

}  // namespace

cudaError_t encode_out_maps(const GemmArgs& a, OutMaps* om) {
  cudaError_t e = cudaSuccess;
  // epilogue maps over the matrices the launch's problems write and read
  std::memset(om, 0, sizeof(*om));
  for (int o = 0; o < a.nops; ++o) {
    const GemmOp& g = a.op[o];
    if (g.nprob <= 0 || g.blocks) continue;  // a scattering op writes from registers
    if (g.out_split) {
      e = encode_epilogue_map(&om->split[o], g.out_split, false, a.B, 2 * idx_extent(g.out_i, g.nprob));
      if (e != cudaSuccess) return e;
    }
    if (g.out_f32) {
      e = encode_epilogue_map(&om->f32[o], g.out_f32, true, a.B, idx_extent(g.outf_i, g.nprob));
      if (e != cudaSuccess) return e;
    }
    if (g.cin_split) {
      e = encode_epilogue_map(&om->cin[o], const_cast<__half*>(g.cin_split), false, a.B,
                              2 * idx_extent(g.cin_i, g.nprob));
      if (e != cudaSuccess) return e;
    } else if (g.cin_f32) {
      e = encode_epilogue_map(&om->cin[o], const_cast<float*>(g.cin_f32), true, a.B, idx_extent(g.cinf_i, g.nprob));
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

bool gemm_wide_supported(const GemmArgs& a) {
  // the register split needs the launch to hold exactly kLaunchRegs a thread.
  // Single-pass products at B = 256 stay on 128 x 128 tiles: their buffers
  // hold one MMA's work per flush, and 128 x 256 tiles cannot skip any of a
  // symmetric launch's lower triangle (3.66 against 3.50 ms for 256 fp16
  // coupled-Newton roots of 256).
  if (a.single_pass && a.B < 512) return false;
  return a.B % kN == 0 && a.B >= kN && wide_kernel_regs() == kLaunchRegs;
}

int gemm_wide_regs() { return wide_kernel_regs(); }

cudaError_t launch_gemm_wide(const CUtensorMap* maps, const GemmArgs& a, long long nprob, cudaStream_t stream) {
  auto kern = a.single_pass ? gemm_wide_kernel<true> : gemm_wide_kernel<false>;
  static std::atomic<unsigned long long> attr_set[2];
  cudaError_t e = smem_limit_once(kern, kSmemBytes, attr_set[a.single_pass ? 1 : 0]);
  if (e != cudaSuccess) return e;
  const long long total = static_cast<long long>(wide_tiles_per_problem(a.B, a.sym)) * nprob;
  const long long sms = gemm_sm_count();
  const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
  // executed tensor-core flops: each 128 x 256 tile is one 2*128*256*B
  // product, done as three fp16 products (one in single-pass mode); in a
  // symmetric launch the first tile of each odd tile row (B/256 a problem)
  // runs at half width
  const double full_tiles = static_cast<double>(total) - (a.sym ? 0.5 * (a.B / kN) * static_cast<double>(nprob) : 0.0);
  const double flops = (a.single_pass ? 1.0 : 3.0) * 2.0 * kM * kN * static_cast<double>(a.B) * full_tiles;
  for (int o = 0; o < a.nops; ++o)  // a scattering op reads no Cin on 128 x 256 tiles
    if (a.op[o].nprob > 0 && a.op[o].blocks && (a.op[o].cin_split || a.op[o].cin_f32)) return cudaErrorInvalidValue;
  OutMaps om;
  e = encode_out_maps(a, &om);
  if (e != cudaSuccess) return e;
  const int slot = prof_begin(kProfGemmWide, stream, flops);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], om, a, total);
  prof_end(slot, stream);
  prof_count_launch();
  return cudaGetLastError();
}

}  // namespace dash
