// Batched split-fp16 GEMM with 128 x 256 output tiles (sm_100a), for
// launches whose block size is a multiple of 256 (split-fp16 products;
// symmetric launches take the tiles that reach the upper triangle).
//
// Same arithmetic as gemm.cu (per K=16 step: hi*lo + lo*hi into a fresh
// tensor-memory buffer, then hi*hi with that buffer scaled by 2^-11, the
// step's product added into fp32 registers with round-to-nearest), with a
// tile twice as wide.  Every MMA issues as much tensor work as it can
// (M=128, N=256), so a step carries twice the work of a 128 x 128 tile for
// the same issue, barrier and hand-off overhead; the price is tensor memory:
// a step's fp32 product takes 256 of the 512 columns, so the ring holds two
// steps and there is no room to park a finished tile.  The accumulator
// warps therefore write their own tile out.
//
// Roles (384 threads = three warpgroups, one CTA per SM, persistent over a
// static round-robin list of the launch's tiles):
//   warps 0-7          accumulators (warpgroups 0 and 1): warp w reads
//                      lanes 32*(w%4).. and 128 of the 256 columns, so each
//                      thread sums 128 columns of one output row in
//                      registers; at the end of a tile the same thread applies
//                      the epilogue to its row segment and stores it.
//   warp 8, one lane   TMA producer: A hi/lo (128 x 64) and B hi/lo
//                      (256 x 64, or four 64 x 64 boxes when B is read
//                      MN-major) of each 64-wide K slab into a 2-stage ring
//                      of 96 KB stages.  No multicast.
//   warp 9, one lane   MMA issuer: three tcgen05.mma kind::f16 per K=16 step
//                      into one of two 256-column tensor-memory buffers.
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

namespace dash {
namespace {

constexpr int kM = 128, kN = 256;
constexpr int kKBlk = 64;                              // fp16 elements per 128-byte row
constexpr int kABytes = kM * kKBlk * 2;                // 16 KB per plane and slab
constexpr int kBBytes = kN * kKBlk * 2;                // 32 KB per plane and slab
constexpr int kStageBytes = 2 * kABytes + 2 * kBBytes;  // A hi, A lo, B hi, B lo
constexpr int kStages = 2;
constexpr int kRing = 2;                               // per-K-step product buffers of kN columns
constexpr uint32_t kTmemCols = 512;
constexpr int kAccWarps = 8;                           // warps 0-7
constexpr int kProdWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;                       // registers a thread at launch (65536 / 384, rounded to 8)
constexpr int kLowRegs = 72, kHighRegs = 216;          // after setmaxnreg: warpgroup 2 / warpgroups 0-1
static_assert(2 * 128 * kHighRegs + 128 * kLowRegs <= kThreads * kLaunchRegs, "register split exceeds the launch");
static_assert(2 * 32 * kHighRegs + 32 * kLowRegs <= 16384, "register split exceeds a scheduler's file");
constexpr int kCols = 128;                             // columns summed per accumulator thread
constexpr int kPrefetchSteps = 6;                      // K=16 steps before a tile's end when its Cin is prefetched
constexpr int kChunk = 32;                             // columns per tensor-memory load batch

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[kRing], acc_empty[kRing];
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
};
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + static_cast<int>(sizeof(Bars)) + 64;

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

__global__ void __launch_bounds__(kThreads, 1)
    gemm_wide_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                     const GemmArgs args, const long long total) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + kStages * kStageBytes);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = args.B / kN;
  const int tpp = wide_tiles_per_problem(args.B, args.sym);
  const int nk = args.B / kKBlk;
  const int nsteps = nk * (kKBlk / 16);

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
      bool stop = args.skip_loads != 0;
      for (long long t = blockIdx.x; t < total && !stop; t += gridDim.x) {
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
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
          tma_load_3d(st, ta, &bars->full[s], kb * kKBlk, ti * kM, 2 * am);
          tma_load_3d(st + kABytes, ta, &bars->full[s], kb * kKBlk, ti * kM, 2 * am + 1);
#pragma unroll
          for (int pl = 0; pl < 2; ++pl) {
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
      for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int op, p, ti, tj;
        decode_wide(args, tpp, ntn, t, op, p, ti, tj);
        const bool bmn = args.op[op].b_mn != 0;
        const uint32_t idesc = f16_idesc(kM, kN) | (bmn ? (1u << 16) : 0u);
        const uint64_t bd0 = (bmn ? md0 : kd0) + 2 * kAD;
        const uint32_t bstep = bmn ? (2048u >> 4) : (32u >> 4);
        for (int kb = 0; kb < nk; ++kb) {
          ok = mbar_wait(&bars->full[s], fpar, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t so = s * (kStageBytes >> 4);
          const uint64_t ah = kd0 + so, al = ah + kAD, bh = bd0 + so, bl = bh + kBD;
#pragma unroll
          for (int kk = 0; kk < kKBlk / 16; ++kk) {
            ok = mbar_wait(&bars->acc_empty[hb], (hpar >> hb) & 1u, abort_flag);
            hpar ^= 1u << hb;
            if (!ok) break;
            tc_fence_after();
            const uint32_t ka = 2u * kk, kbo = bstep * kk;
            const uint32_t d = tbase + hb * kN;
            mma_f16_ss(d, ah + ka, bl + kbo, idesc, 0u);         // hi * lo
            mma_f16_ss(d, al + ka, bh + kbo, idesc, 1u);         // + lo * hi
            mma_f16_ss_acc_down11(d, ah + ka, bh + kbo, idesc);  // hi * hi + 2^-11 * (...)
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
    bool ok = true;
    for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
      float S[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) S[j] = 0.0f;
      // Cin of this thread's row segment is fetched into L2 a few steps
      // before the epilogue needs it (no registers held)
      int op, p, ti, tj;
      decode_wide(args, tpp, ntn, t, op, p, ti, tj);
      const GemmOp& g = args.op[op];
      const int row = ti * kM + quad * 32 + lane;
      const int cbase = tj * kN + cgrp * kCols;
      const int pf_step = nsteps > kPrefetchSteps ? nsteps - kPrefetchSteps : 0;
      for (int sg = 0; sg < nsteps; ++sg) {
        if (sg == pf_step) prefetch_cin_l2(g, p, B, BB, row, cbase);
        // waiting warps sleep in the barrier, leaving the issue slots of
        // their scheduler to the MMA and TMA threads
        if (!mbar_wait_sleep(&bars->acc_full[hb], (hpar >> hb) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        hpar ^= 1u << hb;
        tc_fence_after();
        const uint32_t src = tbase + lane_off + hb * kN;
        const bool last = sg + 1 == nsteps;
#pragma unroll
        for (int c = 0; c < kCols / kChunk; ++c) {
          uint32_t r[kChunk];
#pragma unroll
          for (int q = 0; q < kChunk / 16; ++q) tmem_ld_32x32b_x16(src + kChunk * c + 16 * q, r + 16 * q);
          tmem_ld_wait();
          if (!last && c + 1 == kCols / kChunk) {  // registers hold the whole step now
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
          }
#pragma unroll
          for (int j = 0; j < kChunk; j += 2) add_f32x2(S[kChunk * c + j], S[kChunk * c + j + 1], r[j], r[j + 1]);
          if (last) {  // the tile's sums go back into this buffer for the epilogue
#pragma unroll
            for (int q = 0; q < kChunk / 16; ++q) tmem_st_32x32b_x16(src + kChunk * c + 16 * q, &S[kChunk * c + 16 * q]);
          }
        }
        if (!last) hb ^= 1u;
      }
      if (!ok) {
        if (lane == 0) gemm_fail_timeout(abort_flag, args.status);
        break;
      }
      tmem_st_wait();
      // epilogue of this thread's row segment (128 columns) from the buffer
      // holding the finished sums; the buffer is released afterwards
      const uint32_t src = tbase + lane_off + hb * kN;
      // symmetric launches: this 128-column block q of the tile row ti is
      // written if q >= ti, and mirrored if q > ti (q < ti comes from the
      // mirror of block (q, ti))
      const int q = 2 * tj + cgrp;
      const bool write = !args.sym || q >= ti;
      const bool mirror = args.sym && q > ti;
      GemmEpilogue ep;
      ep.init(g, p, B, BB);
      // Cin streams two 16-column chunks ahead of use (L2 hits by now); a
      // deeper ring would not fit the accumulator warps' registers
      constexpr int kAhead = 2;
      GemmEpilogue::CinRaw pre[kAhead];
      const bool cin = write && ep.has_cin();
      if (cin) {
#pragma unroll
        for (int c = 0; c < kAhead; ++c) pre[c] = ep.load_cin(B, BB, row, cbase + 16 * c);
      }
#pragma unroll 1
      for (int c = 0; c < (write ? kCols / 16 : 0); ++c) {  // pre[0] holds chunk c; the ring rotates
        const int col0 = cbase + c * 16;
        float v[16], cj[16];
        tmem_ld_32x32b_x16(src + 16 * c, reinterpret_cast<uint32_t*>(v));
        tmem_ld_wait();
        if (cin) {
          ep.join_cin(pre[0], cj);
#pragma unroll
          for (int i = 0; i + 1 < kAhead; ++i) pre[i] = pre[i + 1];
          if (c + kAhead < kCols / 16) pre[kAhead - 1] = ep.load_cin(B, BB, row, col0 + 16 * kAhead);
        }
        ep.chunk(g, B, BB, row, col0, v, cj, mirror);
      }
      ep.finish(g, p, args.status);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
      hb ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Registers a thread of gemm_wide_kernel was compiled with (once per process).
int wide_kernel_regs() {
  static std::atomic<int> regs{-1};
  int r = regs.load();
  if (r < 0) {
    cudaFuncAttributes fa;
    r = cudaFuncGetAttributes(&fa, gemm_wide_kernel) == cudaSuccess ? fa.numRegs : 0;
    regs.store(r);
  }
  return r;
}

}  // namespace

bool gemm_wide_supported(const GemmArgs& a) {
  // the register split needs the launch to hold exactly kLaunchRegs a thread
  return a.single_pass == 0 && a.B % kN == 0 && a.B >= kN && wide_kernel_regs() == kLaunchRegs;
}

int gemm_wide_regs() { return wide_kernel_regs(); }

cudaError_t launch_gemm_wide(const CUtensorMap* maps, const GemmArgs& a, long long nprob, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_set;
  cudaError_t e = smem_limit_once(gemm_wide_kernel, kSmemBytes, attr_set);
  if (e != cudaSuccess) return e;
  const long long total = static_cast<long long>(wide_tiles_per_problem(a.B, a.sym)) * nprob;
  const long long sms = gemm_sm_count();
  const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
  // executed tensor-core flops: each 128 x 256 tile is one 2*128*256*B
  // product, done as three fp16 products
  const double flops = 3.0 * 2.0 * kM * kN * static_cast<double>(a.B) * static_cast<double>(total);
  const int slot = prof_begin(kProfGemmWide, stream, flops);
  gemm_wide_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], a, total);
  prof_end(slot, stream);
  prof_count_launch();
  return cudaGetLastError();
}

}  // namespace dash
