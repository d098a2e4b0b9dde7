// Batched split-fp16 GEMM on tcgen05 tensor cores (sm_100a), persistent and
// warp-specialised.
//
// Each CTA (one per SM) walks a static round-robin list of the launch's
// 128 x 128 output tiles over all problems of the launch.  Roles (448 threads):
//   warp 0, one lane   TMA producer: streams the A hi/lo and B hi/lo tiles of
//                      each 64-wide K slab into a 3-stage shared-memory ring
//                      (A always K-major; B K-major, or MN-major as two
//                      64-column boxes when the op multiplies by B itself);
//   warp 1, one lane   MMA issuer;
//   warps 2-9          accumulators: warp w reads tensor-memory lanes
//                      32*(w%4).. and 64 of the 128 columns, so each thread
//                      sums 64 columns of one output row in registers;
//   warps 10-13        output: one thread per row writes the finished tile.
//
// The tensor core's fp32 accumulation truncates, so a sum kept in tensor
// memory over many MMAs drifts low.  Each K=16 step therefore gets a fresh
// tensor-memory buffer from a ring of three: the MMA warp computes hi*lo +
// lo*hi into it and then hi*hi with the buffer's content scaled by 2^-11
// (the MMA's input-scaling operand), so the buffer holds the step's whole
// product after one truncating addition; the accumulator warps add it into
// fp32 registers with round-to-nearest (packed f32x2 adds) and release it.
// At the end of a tile they park the sums in a fourth tensor-memory buffer
// and go on with the next tile at once, while the output warps apply the
// epilogue (scales, Cin, identity shift) and store the parked tile: the
// ring keeps draining while a tile is written out.
#include "gemm.cuh"
#include "gemm_common.cuh"
#include "launch_util.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

#include <atomic>

namespace dash {
namespace {

constexpr int kTile = 128;
constexpr int kKBlk = 64;                          // fp16 elements per 128-byte row
constexpr int kTileBytes = kTile * kKBlk * 2;      // 16 KB per plane and slab
constexpr int kStageBytes = 4 * kTileBytes;        // A hi, A lo, B hi, B lo
constexpr int kStages = 3;
constexpr int kRing = 3;                           // per-K-step product buffers
constexpr uint32_t kColPark = kRing * 128;         // finished-tile buffer
constexpr uint32_t kTmemCols = 512;
constexpr int kAccWarp0 = 2, kAccWarps = 8;
constexpr int kOutWarp0 = kAccWarp0 + kAccWarps, kOutWarps = 4;
constexpr int kThreads = 32 * (kOutWarp0 + kOutWarps);
constexpr int kCols = 64;                          // columns summed per accumulator thread

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[kRing], acc_empty[kRing];
  uint64_t park_full, park_empty;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
};
// Output staging: per output warp two 4 KB buffers, each one 32 x 32 step of
// split fp16 (both planes) or fp32 output in the TMA swizzle, stored with one
// tensor store; a buffer is rewritten once the store from it two steps ago
// has read it.
constexpr int kStageBufBytes = 4096;
constexpr int kStagingOff = kStages * kStageBytes;
constexpr int kBarsOff = kStagingOff + kOutWarps * 2 * kStageBufBytes;
constexpr int kSmemBytes = kBarsOff + 1024 + static_cast<int>(sizeof(Bars)) + 64;
static_assert(kSmemBytes <= 232448, "shared memory exceeds the per-block limit");

// Tile t of a problem -> (tile row, tile column).  sym: upper triangle of
// the nt x nt square tile grid only, enumerated row by row.
__device__ __forceinline__ void tile_coords(int t, int ntn, int sym, int& ti, int& tj) {
  if (!sym) {
    ti = t / ntn;
    tj = t % ntn;
    return;
  }
  int r = 0;
  while (t >= ntn - r) {
    t -= ntn - r;
    ++r;
  }
  ti = r;
  tj = r + t;
}

// Flattened tile index -> (op, problem, tile row, tile column).  When both
// ops of a launch have the same problems, the two ops of a problem are
// adjacent in the order, so operands they share are read from L2 once.
__device__ __forceinline__ void decode(const GemmArgs& args, int tpp, int ntn, long long t, int& op, int& p,
                                       int& ti, int& tj) {
  if (args.op[1].nprob == args.op[0].nprob) {
    const long long pair = 2ll * tpp;
    p = static_cast<int>(t / pair);
    const int r = static_cast<int>(t - static_cast<long long>(p) * pair);
    op = r >= tpp ? 1 : 0;
    tile_coords(op ? r - tpp : r, ntn, args.sym, ti, tj);
    return;
  }
  const long long n0 = static_cast<long long>(args.op[0].nprob) * tpp;
  op = t < n0 ? 0 : 1;
  const long long u = op ? t - n0 : t;
  p = static_cast<int>(u / tpp);
  tile_coords(static_cast<int>(u % tpp), ntn, args.sym, ti, tj);
}

// kSingle: one pass of hi*hi only (fp16 operands, fp32 accumulation); the lo
// planes are neither loaded nor multiplied and each K=64 slab is one segment.
template <bool kSingle>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_split_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                      const __grid_constant__ OutMaps om, const GemmArgs args, const long long total) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarsOff);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = args.B / kTile;
  const int tpp = args.sym ? nt * (nt + 1) / 2 : nt * nt;
  const int nk = args.B / kKBlk;
  const int nsteps = kSingle ? nk : nk * (kKBlk / 16);  // accumulator segments per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < kRing; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], kAccWarps);
    }
    mbar_init(&bars->park_full, kAccWarps);
    mbar_init(&bars->park_empty, kOutWarps);
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
          mbar_arrive_expect_tx(&bars->full[s], kSingle ? kStageBytes / 2 : kStageBytes);
          tma_load_3d(st, ta, &bars->full[s], kb * kKBlk, ti * kTile, 2 * am);
          if (!kSingle) tma_load_3d(st + kTileBytes, ta, &bars->full[s], kb * kKBlk, ti * kTile, 2 * am + 1);
#pragma unroll
          for (int pl = 0; pl < (kSingle ? 1 : 2); ++pl) {
            uint8_t* dst = st + (2 + pl) * kTileBytes;
            if (g.b_mn) {  // rows kb*64.. of B, columns tj*128.. as two 64-column boxes
              tma_load_3d(dst, tb, &bars->full[s], tj * kTile, kb * kKBlk, 2 * bm + pl);
              tma_load_3d(dst + kTileBytes / 2, tb, &bars->full[s], tj * kTile + 64, kb * kKBlk, 2 * bm + pl);
            } else {
              tma_load_3d(dst, tb, &bars->full[s], kb * kKBlk, tj * kTile, 2 * bm + pl);
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
      constexpr uint32_t kTD = kTileBytes >> 4;   // descriptor address units
      uint32_t s = 0, fpar = 0;                    // stage, parity of its next fill
      uint32_t hb = 0, hpar = (1u << kRing) - 1u;  // ring buffer, parity bits of the next release per buffer
      bool ok = true;
      for (long long t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int op, p, ti, tj;
        decode(args, tpp, nt, t, op, p, ti, tj);
        const bool bmn = args.op[op].b_mn != 0;
        const uint32_t idesc = f16_idesc(kTile, kTile) | (bmn ? (1u << 16) : 0u);
        const uint64_t bd0 = (bmn ? md0 : kd0) + 2 * kTD;
        const uint32_t bstep = bmn ? (2048u >> 4) : (32u >> 4);
        for (int kb = 0; kb < nk; ++kb) {
          ok = mbar_wait(&bars->full[s], fpar, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t so = s * (kStageBytes >> 4);
          const uint64_t ah = kd0 + so, al = ah + kTD, bh = bd0 + so, bl = bh + kTD;
          if (kSingle) {  // the whole slab into one buffer
            ok = mbar_wait(&bars->acc_empty[hb], (hpar >> hb) & 1u, abort_flag);
            hpar ^= 1u << hb;
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tbase + hb * 128u;
#pragma unroll
            for (int kk = 0; kk < kKBlk / 16; ++kk)
              mma_f16_ss(d, ah + 2u * kk, bh + bstep * kk, idesc, kk ? 1u : 0u);
            mma_commit(&bars->acc_full[hb]);
            hb = hb == kRing - 1 ? 0u : hb + 1u;
          } else {
#pragma unroll
            for (int kk = 0; kk < kKBlk / 16; ++kk) {
              ok = mbar_wait(&bars->acc_empty[hb], (hpar >> hb) & 1u, abort_flag);
              hpar ^= 1u << hb;
              if (!ok) break;
              tc_fence_after();
              const uint32_t ka = 2u * kk, kbo = bstep * kk;
              const uint32_t d = tbase + hb * 128u;
              mma_f16_ss(d, ah + ka, bl + kbo, idesc, 0u);         // hi * lo
              mma_f16_ss(d, al + ka, bh + kbo, idesc, 1u);         // + lo * hi
              mma_f16_ss_acc_down11(d, ah + ka, bh + kbo, idesc);  // hi * hi + 2^-11 * (...)
              mma_commit(&bars->acc_full[hb]);
              hb = hb == kRing - 1 ? 0u : hb + 1u;
            }
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
  } else if (warp < kOutWarp0) {
    // ---------------------------------------------------------------- accumulators
    const int quad = warp & 3;                 // tensor-memory lane quadrant of this warp
    const int cgrp = (warp - kAccWarp0) >> 2;  // 64-column half of the tile
    const uint32_t lane_off = (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(cgrp * kCols);
    uint32_t hb = 0, hpar = 0, ppar = 1;  // ring buffer, its fill parities, park release parity
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      float S[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) S[j] = 0.0f;
      bool ok = true;
      for (int sg = 0; sg < nsteps; ++sg) {
        // waiting warps sleep in the barrier, leaving the issue slots of
        // their scheduler to the MMA and TMA threads
        if (!mbar_wait_sleep(&bars->acc_full[hb], (hpar >> hb) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        hpar ^= 1u << hb;
        tc_fence_after();
        const uint32_t src = tbase + lane_off + hb * 128u;
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x16(src + 32 * c, r);
          tmem_ld_32x32b_x16(src + 32 * c + 16, r + 16);
          tmem_ld_wait_regs<32>(r);
          if (c + 1 == kCols / 32) {  // registers hold the whole step now
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
            hb = hb == kRing - 1 ? 0u : hb + 1u;
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) add_f32x2(S[32 * c + j], S[32 * c + j + 1], r[j], r[j + 1]);
        }
      }
      // hand the tile to the output warps through the park buffer
      if (ok) {
        ok = mbar_wait_sleep(&bars->park_empty, ppar, abort_flag);
        ppar ^= 1u;
      }
      if (!ok) {
        if (threadIdx.x == kAccWarp0 * 32) gemm_fail_timeout(abort_flag, args.status);
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c) tmem_st_32x32b_x16(tbase + lane_off + kColPark + 16 * c, &S[16 * c]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->park_full);
    }
  } else {
    // ---------------------------------------------------------------- output
    const int quad = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const size_t B = static_cast<size_t>(args.B);
    const size_t BB = B * B;
    uint32_t ppar = 0;
    uint8_t* const stg = smem + kStagingOff + (warp - kOutWarp0) * 2 * kStageBufBytes;
    int nb = 0;  // next staging buffer
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      int op, p, ti, tj;
      decode(args, tpp, nt, t, op, p, ti, tj);
      const GemmOp& g = args.op[op];
      const int row = ti * kTile + quad * 32 + lane;
      const int cbase = tj * kTile;
      const bool mirror = args.sym && (ti != tj);
      GemmEpilogue ep;
      ep.init(g, p, B, BB);
      const bool cin = ep.has_cin();
      const int row0 = ti * kTile + quad * 32;  // first row of this warp's steps
      if (!mbar_wait_sleep(&bars->park_full, ppar, abort_flag)) {
        if (threadIdx.x == kOutWarp0 * 32) gemm_fail_timeout(abort_flag, args.status);
        break;
      }
      ppar ^= 1u;
      tc_fence_after();
      // four steps of 32 columns; row-major outputs leave through the
      // staging buffers (a store instruction whose 32 lanes each write a
      // different row would touch 32 lines), the mirror's stores are
      // already coalesced, scattered outputs go straight to the parameters
#pragma unroll 1
      for (int k = 0; k < kTile / 32; ++k) {
        const int col0 = cbase + 32 * k;
        GemmEpilogue::CinRaw pre[2];  // in flight during the tensor-memory loads
        if (cin) {
          pre[0] = ep.load_cin(B, BB, row, col0);
          pre[1] = ep.load_cin(B, BB, row, col0 + 16);
        }
        float v[2][16];
        tmem_ld_32x32b_x16(tbase + lane_off + kColPark + 32 * k, reinterpret_cast<uint32_t*>(v[0]));
        tmem_ld_32x32b_x16(tbase + lane_off + kColPark + 32 * k + 16, reinterpret_cast<uint32_t*>(v[1]));
        tmem_ld_wait_regs<32>(reinterpret_cast<uint32_t*>(v));
        if (k + 1 == kTile / 32) {  // the park buffer is free for the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->park_empty);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float cj[16];
          if (cin) ep.join_cin(pre[h], cj);
          ep.apply(row, col0 + 16 * h, v[h], cj);
        }
        if (ep.scatter) {  // through fp32 staging: lane l writes column l, row by row
          ep.check_finite(v[0]);
          ep.check_finite(v[1]);
          uint8_t* buf = stg + nb * kStageBufBytes;
          __syncwarp();
          stage_f32x32(buf, lane, v);
          __syncwarp();
          scatter_step(buf, lane, g, ep.bd, row0, col0, ep.sumsq);
          nb ^= 1;
          continue;
        }
        if (mirror) {
          ep.store_mirror(B, BB, row, col0, v[0]);
          ep.store_mirror(B, BB, row, col0 + 16, v[1]);
        }
        if (ep.of) {
          ep.check_finite(v[0]);
          ep.check_finite(v[1]);
          uint8_t* buf = stg + nb * kStageBufBytes;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          stage_f32x32(buf, lane, v);
          store_step(lane, &om.f32[op], buf, col0, row0, gemm_at(g.outf_i, p));
          nb ^= 1;
        }
        if (ep.os) {  // split output, scaled in place
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 16; ++j) v[h][j] *= ep.ss;
          uint8_t* buf = stg + nb * kStageBufBytes;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          stage_split32(buf, lane, v, ep.bad);
          store_step(lane, &om.split[op], buf, col0, row0, 2 * gemm_at(g.out_i, p));
          nb ^= 1;
        }
      }
      ep.finish(g, p, args.status);
    }
    // this warp's tensor stores complete before the CTA's shared memory goes
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

std::atomic<int> g_load_fault{0};

}  // namespace

int gemm_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

cudaError_t launch_gemm_split(const OpBuffers* bufs, const GemmArgs& args, cudaStream_t stream) {
  if (args.nops < 1 || args.nops > 2) return cudaErrorInvalidValue;
  const int nprob = args.op[0].nprob + (args.nops == 2 ? args.op[1].nprob : 0);
  if (nprob <= 0) return cudaSuccess;
  if (args.B % kTile != 0 || args.B <= 0) return cudaErrorInvalidValue;
  GemmArgs a = args;
  if (a.nops == 1) a.op[1] = a.op[0], a.op[1].nprob = 0;
  if (take_load_fault()) a.skip_loads = 1;
  const bool wide = gemm_wide_supported(a);
  CUtensorMap maps[4];
  for (int o = 0; o < 2; ++o) {
    const OpBuffers& b = bufs[o < a.nops ? o : 0];
    cudaError_t e = encode_split_stack_map(&maps[2 * o], b.a, a.B, b.a_nmat, kTile);
    if (e != cudaSuccess) return e;
    e = encode_split_stack_map(&maps[2 * o + 1], b.b, a.B, b.b_nmat, a.op[o].b_mn ? 64 : (wide ? 256 : kTile));
    if (e != cudaSuccess) return e;
  }
  if (wide) return launch_gemm_wide(maps, a, nprob, stream);
  OutMaps om;
  cudaError_t me = encode_out_maps(a, &om);
  if (me != cudaSuccess) return me;
  void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const OutMaps,
               const GemmArgs, const long long) = a.single_pass ? gemm_split_kernel<true> : gemm_split_kernel<false>;
  static std::atomic<unsigned long long> attr_set[2];
  cudaError_t e = smem_limit_once(kern, kSmemBytes, attr_set[a.single_pass ? 1 : 0]);
  if (e != cudaSuccess) return e;
  const long long nt = a.B / kTile;
  const long long tpp = a.sym ? nt * (nt + 1) / 2 : nt * nt;
  const long long total = tpp * nprob;
  const long long sms = gemm_sm_count();
  const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
  // executed tensor-core flops: each computed 128 x 128 tile is one
  // 2*128*128*B product, done as three fp16 products (one in single-pass mode)
  const double flops = (a.single_pass ? 1.0 : 3.0) * 2.0 * kTile * kTile * static_cast<double>(a.B) *
                       static_cast<double>(total);
  const int slot = prof_begin(kProfGemm, stream, flops);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(maps[0], maps[1], maps[2], maps[3], om, a, total);
  prof_end(slot, stream);
  prof_count_launch();
  return cudaGetLastError();
}

void arm_load_fault() { g_load_fault.store(1); }

bool take_load_fault() { return g_load_fault.exchange(0) != 0; }

}  // namespace dash
