// Host-side launch helpers shared by the tensor-core kernels.
#pragma once

#include <atomic>
#include <cuda_runtime.h>

namespace dash {

// Raise a kernel's dynamic shared-memory limit once per device.  The
// attribute persists, and skipping the call on later launches keeps those
// launches free of non-stream calls, so they can be captured into a CUDA
// graph.  'done' holds one bit per device (devices 0..63).
template <typename Kernel>
cudaError_t smem_limit_once(Kernel kern, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev > 63) return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  const unsigned long long bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

}  // namespace dash
