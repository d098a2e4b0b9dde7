// Newton-DB iterations on 128 x 128 factors held in shared memory (sm_100a).
//
// "Building blocks", Newton-DB: each iteration forms D = (I - Z Y)/2 and
// updates Y <- Y + Y D, Z <- Z + D Z (E = I + D applied in correction
// form, products in the page's order; Z is kept as Zhat = Z / zs).  At
// B = 128 a factor's Y, Zhat and D, as split fp16 (hi and lo planes), take
// 3 x 64 KB: one CTA keeps them in shared memory and runs a stage's
// iterations on them with no trip through HBM and no launch per product:
// the first (Y + Y D0, D0 from the stage's prologue), the full middle ones,
// and a last one that updates Y only.  The final iteration of the second
// stage, whose output is the root in fp32 and split form, stays on the
// batched GEMM.
//
// Arithmetic: the same as the 128 x 128 GEMM, step for step.  Every K=16
// step of a product is three tcgen05.mma kind::f16 (hi*lo, + lo*hi, then
// hi*hi plus 2^-11 times that sum) into a fresh 128-column tensor-memory
// buffer; the accumulator warps add the buffer into fp32 registers with
// round-to-nearest; the epilogue computes alpha*acc (+ Cin) (+ gamma on the
// diagonal) in packed fp32 and splits the result into hi and lo fp16.
//
// Layout: each plane of a matrix is stored the way a TMA load with a
// {64, 128} box and 128-byte swizzle leaves it: two 16 KB blocks of 64
// columns, 128 rows of 128 bytes each, the 16-byte chunks of row r permuted
// by r mod 8.  The same bytes serve as a K-major A operand (a 64-wide K slab
// per block) and as an MN-major B operand (a 64-wide N slab per block, K
// rows 128 bytes apart), so a result written back by the epilogue is the
// next product's operand as it stands.
//
// Roles (320 threads, one CTA per SM, persistent over the factors):
//   warp 0, one lane   loads a factor's Y and Zhat (and D0) by TMA and
//                      stores them back when its iterations are done;
//   warp 1, one lane   MMA issuer (warp 1 owns the tensor memory);
//   warps 2-9          accumulators: warp w reads tensor-memory lanes
//                      32*(w%4).. and 64 of the 128 columns, sums them per
//                      row in registers, and writes D, Y and Zhat back into
//                      shared memory (then a proxy fence, so that the tensor
//                      core reads what they wrote).
// Per full iteration the MMA issues 24 steps (D = Zhat Y, then Y D, then
// D Zhat) through a ring of four buffers; it waits for D before the second
// product and for Y and Zhat before the next iteration's first.
#include "gemm.cuh"
#include "gemm_common.cuh"
#include "launch_util.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

#include <atomic>

namespace dash {
namespace {

constexpr int kN = 128;                     // matrix size
constexpr int kColBlk = kN * 128;           // 16 KB: 64 columns x 128 rows of one plane
constexpr int kPlaneBytes = 2 * kColBlk;    // 32 KB
constexpr int kMatBytes = 2 * kPlaneBytes;  // 64 KB: hi and lo planes
constexpr int kYOff = 0, kZOff = kMatBytes, kDOff = 2 * kMatBytes;
constexpr int kRing = 4;                    // per-step product buffers of 128 columns
constexpr uint32_t kTmemCols = 512;
constexpr int kAccWarp0 = 2, kAccWarps = 8;
constexpr int kThreads = 32 * (kAccWarp0 + kAccWarps);
constexpr int kCols = 64;                   // columns summed per accumulator thread
constexpr int kSteps = kN / 16;             // K=16 steps per product

struct Bars {
  uint64_t acc_full[kRing], acc_empty[kRing];
  uint64_t ld_full;   // a factor's Y and Zhat have landed
  uint64_t d_ready;   // D is in shared memory (one arrival per accumulator warp)
  uint64_t yz_ready;  // Y and Zhat are back, before a factor's last iteration
  uint64_t yz_final;  // ... after its last iteration
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
};
constexpr int kBarsOff = 3 * kMatBytes;

// Steps of one launch, the same for every factor: groups run in order, each
// ending with Y (and Zhat) back in shared memory.
//   first   Y <- Y + Y D, with D loaded from HBM beside Y and Zhat (a
//           stage's first iteration, whose D comes from its prologue);
//   iters   full iterations: D = alpha_d Zhat Y + I/2, Y <- Y + Y D,
//           Zhat <- Zhat + D Zhat;
//   last_y  one more iteration that updates Y only (the last of a stage
//           whose Zhat is not used afterwards; Zhat is then not stored).
struct FusedPlan {
  int first, iters, last_y;
};
enum GroupKind { kFirstY = 0, kFull = 1, kLastY = 2 };
__host__ __device__ __forceinline__ int plan_groups(const FusedPlan& pl) { return pl.first + pl.iters + pl.last_y; }
__device__ __forceinline__ int group_kind(const FusedPlan& pl, int gi) {
  if (pl.first && gi == 0) return kFirstY;
  return pl.last_y && gi == plan_groups(pl) - 1 ? kLastY : kFull;
}
constexpr int kSmemBytes = kBarsOff + static_cast<int>(sizeof(Bars)) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory exceeds the per-block limit");
static_assert(kRing * 128 <= static_cast<int>(kTmemCols), "ring exceeds tensor memory");

// Byte offset, inside a plane, of the 16-byte chunk j (columns 8j..8j+7 of
// the 64-column block cb) of row r.
__device__ __forceinline__ uint32_t chunk_off(int cb, int r, int j) {
  return static_cast<uint32_t>(cb * kColBlk + r * 128 + ((j ^ (r & 7)) << 4));
}

// One K=16 step of A (K-major, matrix at byte offset ma) times B (MN-major,
// at mb) into buffer d: hi*lo, + lo*hi, then hi*hi plus 2^-11 times that.
__device__ __forceinline__ void mma_step(uint32_t d, uint64_t kd, uint64_t md, int ma, int mb, int kk,
                                         uint32_t idesc) {
  const uint64_t ah = kd + static_cast<uint32_t>((ma + (kk >> 2) * kColBlk) >> 4) + 2u * (kk & 3);
  const uint64_t al = ah + (kPlaneBytes >> 4);
  const uint64_t bh = md + static_cast<uint32_t>(mb >> 4) + static_cast<uint32_t>(kk) * (2048u >> 4);
  const uint64_t bl = bh + (kPlaneBytes >> 4);
  mma_f16_ss(d, ah, bl, idesc, 0u);
  mma_f16_ss(d, al, bh, idesc, 1u);
  mma_f16_ss_acc_down11(d, ah, bh, idesc);
}

// Writes this thread's 64 values (row r, columns 64*cb..) of a result as
// split fp16 into the matrix at buf: out = alpha*S (+ Cin read from the same
// place) (+ gamma where the column is r), in the GEMM epilogue's order.
__device__ __forceinline__ void write_row(uint8_t* buf, int cb, int r, const float* S, float alpha, bool cin,
                                          float gamma, bool& bad) {
#pragma unroll
  for (int q = 0; q < kCols / 16; ++q) {
    float v[16];
    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float2 x = __fmul2_rn(make_float2(S[16 * q + j], S[16 * q + j + 1]), a2);
      v[j] = x.x;
      v[j + 1] = x.y;
    }
    if (cin) {
      SplitChunk c;
      c.h[0] = *reinterpret_cast<const uint4*>(buf + chunk_off(cb, r, 2 * q));
      c.h[1] = *reinterpret_cast<const uint4*>(buf + chunk_off(cb, r, 2 * q + 1));
      c.l[0] = *reinterpret_cast<const uint4*>(buf + kPlaneBytes + chunk_off(cb, r, 2 * q));
      c.l[1] = *reinterpret_cast<const uint4*>(buf + kPlaneBytes + chunk_off(cb, r, 2 * q + 1));
      float cj[16];
      join_chunk(c, cj);
      const float2 b2 = make_float2(1.0f, 1.0f);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 x = __ffma2_rn(b2, make_float2(cj[j], cj[j + 1]), make_float2(v[j], v[j + 1]));
        v[j] = x.x;
        v[j + 1] = x.y;
      }
    }
    const int dcol = r - (64 * cb + 16 * q);
    if (gamma != 0.0f && dcol >= 0 && dcol < 16) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j == dcol) v[j] += gamma;
    }
    __half2 hi[8], lo[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      split_f16x2(v[2 * j], v[2 * j + 1], hi[j], lo[j]);
      bad |= f16_overflows(v[2 * j]) || f16_overflows(v[2 * j + 1]);
    }
    *reinterpret_cast<uint4*>(buf + chunk_off(cb, r, 2 * q)) = *reinterpret_cast<const uint4*>(&hi[0]);
    *reinterpret_cast<uint4*>(buf + chunk_off(cb, r, 2 * q + 1)) = *reinterpret_cast<const uint4*>(&hi[4]);
    *reinterpret_cast<uint4*>(buf + kPlaneBytes + chunk_off(cb, r, 2 * q)) = *reinterpret_cast<const uint4*>(&lo[0]);
    *reinterpret_cast<uint4*>(buf + kPlaneBytes + chunk_off(cb, r, 2 * q + 1)) =
        *reinterpret_cast<const uint4*>(&lo[4]);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    ndb_fused_kernel(const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmZ,
                     const __grid_constant__ CUtensorMap tmD, const int n, const float alpha_d, const FusedPlan plan,
                     const int skip_loads, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarsOff);
  volatile int* abort_flag = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int b = 0; b < kRing; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], kAccWarps);
    }
    mbar_init(&bars->ld_full, 1);
    mbar_init(&bars->d_ready, kAccWarps);
    mbar_init(&bars->yz_ready, kAccWarps);
    mbar_init(&bars->yz_final, kAccWarps);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmY);
    tma_prefetch_desc(&tmZ);
    tma_prefetch_desc(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_slot;
  const int groups = plan_groups(plan);
  // Zhat is stored back only when the last group is a full iteration: after
  // a last_y group the caller has no further use for it (and after first
  // alone it is unchanged)
  const bool store_z = group_kind(plan, groups - 1) == kFull;

  if (warp == 0) {
    // ---------------------------------------------------------------- loads and stores
    if (lane == 0) {
      uint32_t fpar = 0;   // parity of the next yz_final phase
      int loads = 0;       // factors loaded (ld_full phases issued)
      int prev = -1;       // factor whose results are still in shared memory
      bool ok = true;
      auto store = [&](int p) {
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
#pragma unroll
          for (int cb = 0; cb < 2; ++cb) {
            const uint32_t o = pl * kPlaneBytes + cb * kColBlk;
            tma_store_3d(&tmY, smem + kYOff + o, 64 * cb, 0, 2 * p + pl);
            if (store_z) tma_store_3d(&tmZ, smem + kZOff + o, 64 * cb, 0, 2 * p + pl);
          }
        bulk_commit();
      };
      for (int t = blockIdx.x; t < n && ok; t += gridDim.x) {
        if (prev >= 0) {  // the previous factor's results leave before this one's operands arrive
          ok = mbar_wait_sleep(&bars->yz_final, fpar, abort_flag);
          fpar ^= 1u;
          if (!ok) break;
          store(prev);
          bulk_wait_read<0>();
        }
        if (!skip_loads) {  // (test hook: with skip_loads the operands never arrive)
          mbar_arrive_expect_tx(&bars->ld_full, (plan.first ? 3 : 2) * kMatBytes);
#pragma unroll
          for (int pl = 0; pl < 2; ++pl)
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
              const uint32_t o = pl * kPlaneBytes + cb * kColBlk;
              tma_load_3d(smem + kYOff + o, &tmY, &bars->ld_full, 64 * cb, 0, 2 * t + pl);
              tma_load_3d(smem + kZOff + o, &tmZ, &bars->ld_full, 64 * cb, 0, 2 * t + pl);
              if (plan.first) tma_load_3d(smem + kDOff + o, &tmD, &bars->ld_full, 64 * cb, 0, 2 * t + pl);
            }
          ++loads;
        }
        prev = t;
      }
      if (ok && prev >= 0) {
        ok = mbar_wait_sleep(&bars->yz_final, fpar, abort_flag);
        if (ok) store(prev);
      }
      if (!ok) {
        gemm_fail_timeout(abort_flag, status);
        // the last load lands before the CTA's shared memory goes
        volatile int never = 0;
        if (loads > 0) mbar_wait(&bars->ld_full, static_cast<uint32_t>(loads - 1) & 1u, &never);
      }
      bulk_wait_all();
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t sbase = smem_u32(smem);
      const uint64_t kd = sw128_kmajor_desc(sbase), md = sw128_mnmajor_desc(sbase, kColBlk);
      const uint32_t idesc = f16_idesc(kN, kN) | (1u << 16);  // B read MN-major: out = A B
      uint32_t hb = 0, hpar = (1u << kRing) - 1u;  // ring buffer, parity bits of the next release per buffer
      uint32_t lpar = 0, dpar = 0, ypar = 0;
      bool ok = true;
      auto product = [&](int ma, int mb) -> bool {
        for (int kk = 0; kk < kSteps; ++kk) {
          if (!mbar_wait(&bars->acc_empty[hb], (hpar >> hb) & 1u, abort_flag)) return false;
          hpar ^= 1u << hb;
          tc_fence_after();
          mma_step(tbase + hb * 128u, kd, md, ma, mb, kk, idesc);
          mma_commit(&bars->acc_full[hb]);
          hb = hb == kRing - 1 ? 0u : hb + 1u;
        }
        return true;
      };
      for (int t = blockIdx.x; t < n && ok; t += gridDim.x) {
        ok = mbar_wait(&bars->ld_full, lpar, abort_flag);
        lpar ^= 1u;
        if (!ok) break;
        tc_fence_after();
        for (int gi = 0; gi < groups && ok; ++gi) {
          const int kind = group_kind(plan, gi);
          if (gi > 0) {  // Y and Zhat of the previous group are back
            ok = mbar_wait(&bars->yz_ready, ypar, abort_flag);
            ypar ^= 1u;
            if (!ok) break;
            tc_fence_after();
          }
          if (kind == kFirstY) {
            ok = product(kYOff, kDOff);  // Y D0
            continue;
          }
          ok = product(kZOff, kYOff);  // Zhat Y
          if (!ok) break;
          ok = mbar_wait(&bars->d_ready, dpar, abort_flag);
          dpar ^= 1u;
          if (!ok) break;
          tc_fence_after();
          ok = product(kYOff, kDOff);  // Y D
          if (ok && kind == kFull) ok = product(kDOff, kZOff);  // D Zhat
        }
      }
      if (!ok) gemm_fail_timeout(abort_flag, status);
      // all issued MMAs must retire before tensor memory is released
      mma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0u, &never);
    }
  } else {
    // ---------------------------------------------------------------- accumulators
    const int quad = warp & 3;                 // tensor-memory lane quadrant of this warp
    const int cgrp = (warp - kAccWarp0) >> 2;  // 64-column block of the product
    const int r = quad * 32 + lane;            // this thread's row
    const uint32_t lane_off = (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(cgrp * kCols);
    uint32_t hb = 0, hpar = 0, lpar = 0;
    bool ok = true, bad = false;
    // S = one product, K step by K step (every lane of the warp agrees on
    // the outcome of each wait)
    auto flush = [&](float* S) -> bool {
#pragma unroll
      for (int j = 0; j < kCols; ++j) S[j] = 0.0f;
      for (int sg = 0; sg < kSteps; ++sg) {
        const bool got = mbar_wait_sleep(&bars->acc_full[hb], (hpar >> hb) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) return false;
        hpar ^= 1u << hb;
        tc_fence_after();
        const uint32_t src = tbase + lane_off + hb * 128u;
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          uint32_t q[32];
          tmem_ld_32x32b_x16(src + 32 * c, q);
          tmem_ld_32x32b_x16(src + 32 * c + 16, q + 16);
          tmem_ld_wait_regs<32>(q);
          if (c + 1 == kCols / 32) {  // registers hold the whole step now
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[hb]);
            hb = hb == kRing - 1 ? 0u : hb + 1u;
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) add_f32x2(S[32 * c + j], S[32 * c + j + 1], q[j], q[j + 1]);
        }
      }
      return true;
    };
    for (int t = blockIdx.x; t < n && ok; t += gridDim.x) {
      // the factor's Y and Zhat (the first Cin) come from the TMA load
      ok = __all_sync(0xffffffffu, mbar_wait_sleep(&bars->ld_full, lpar, abort_flag));
      lpar ^= 1u;
      for (int gi = 0; gi < groups && ok; ++gi) {
        const int kind = group_kind(plan, gi);
        float S[kCols];
        if (kind != kFirstY) {
          ok = flush(S);  // Zhat Y
          if (!ok) break;
          write_row(smem + kDOff, cgrp, r, S, alpha_d, false, 0.5f, bad);  // D = alpha_d Zhat Y + I/2
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->d_ready);
        }
        // Y D's MMAs are done once its last step is here, so Y may be
        // rewritten (D Zhat, still running, does not read Y)
        ok = flush(S);
        if (!ok) break;
        write_row(smem + kYOff, cgrp, r, S, 1.0f, true, 0.0f, bad);  // Y + Y D
        if (kind == kFull) {
          ok = flush(S);  // D Zhat
          if (!ok) break;
          write_row(smem + kZOff, cgrp, r, S, 1.0f, true, 0.0f, bad);  // Zhat + D Zhat
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(gi + 1 < groups ? &bars->yz_ready : &bars->yz_final);
      }
    }
    if (!ok && lane == 0) gemm_fail_timeout(abort_flag, status);
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kStatusNonFinite);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_ndb_fused(__half* Y, __half* Zhat, const __half* D, int n, int B, float alpha_d, int first,
                             int iters, int last_y, unsigned* status, cudaStream_t stream) {
  if (B != kN || iters < 0 || (first != 0 && first != 1) || (last_y != 0 && last_y != 1))
    return cudaErrorNotSupported;
  const FusedPlan plan{first, iters, last_y};
  if (n <= 0 || plan_groups(plan) == 0) return cudaSuccess;
  CUtensorMap my, mz, md;
  cudaError_t e = encode_split_stack_map(&my, Y, kN, n, kN);
  if (e != cudaSuccess) return e;
  e = encode_split_stack_map(&mz, Zhat, kN, n, kN);
  if (e != cudaSuccess) return e;
  e = encode_split_stack_map(&md, D, kN, n, kN);
  if (e != cudaSuccess) return e;
  static std::atomic<unsigned long long> attr_set;
  e = smem_limit_once(ndb_fused_kernel, kSmemBytes, attr_set);
  if (e != cudaSuccess) return e;
  const int sms = gemm_sm_count();
  const unsigned grid = static_cast<unsigned>(n < sms ? n : sms);
  // executed tensor-core flops: products of 2*128^3 (one for first, three
  // per full iteration, two for last_y), three fp16 MMAs each
  const double products = first + 3.0 * iters + 2.0 * last_y;
  const double flops = 3.0 * 2.0 * kN * kN * static_cast<double>(kN) * products * static_cast<double>(n);
  const int slot = prof_begin(kProfNdbFused, stream, flops);
  const int skip = take_load_fault() ? 1 : 0;
  ndb_fused_kernel<<<grid, kThreads, kSmemBytes, stream>>>(my, mz, md, n, alpha_d, plan, skip, status);
  prof_end(slot, stream);
  prof_count_launch();
  return cudaGetLastError();
}

}  // namespace dash
