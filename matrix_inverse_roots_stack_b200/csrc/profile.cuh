// Optional kernel-time accounting (host side, off by default).
//
// When enabled, the library records a CUDA event pair around every launch of
// the tensor-core GEMM kernel and around each stage of a step, on the stream
// the work is launched on, and counts every kernel it launches.  Reading the
// totals synchronises the recorded events.
#pragma once

#include <cuda_runtime.h>

namespace dash {

enum ProfStage {
  kProfGemm = 0,         // launches of the split-fp16 GEMM with 128 x 128 tiles (gemm.cu)
  kProfAccumulate = 1,   // gradient gather + factor EMA
  kProfPowerIter = 2,    // multi-start power iteration
  kProfSolver = 3,       // Newton-DB / Chebyshev (prologues + GEMMs)
  kProfPrecond = 4,      // U = X_L G X_R
  kProfAdam = 5,         // Adam moments, graft and update
  kProfGemmWide = 6,     // launches of the split-fp16 GEMM with 128 x 256 tiles (gemm_wide.cu)
  kProfNdbFused = 7,     // launches of the Newton-DB kernel on resident 128 x 128 factors (ndb_fused.cu)
  kProfStages = 8
};

bool prof_on();
// Returns a slot id (>= 0) or -1 when not recording.
int prof_begin(int stage, cudaStream_t st, double flops = 0.0);
void prof_end(int slot, cudaStream_t st);
void prof_count_launch(int n = 1);

}  // namespace dash
