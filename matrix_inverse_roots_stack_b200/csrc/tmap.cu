#include "tmap.cuh"

#include <mutex>

namespace dash {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

cudaError_t encode_f16_3d_map(CUtensorMap* map, const void* base, int cols, int rows, long long depth,
                              int box_rows) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0 || cols % 64 != 0 || cols < 64 || rows < 1 || depth < 1 ||
      box_rows < 1 || box_rows > 256 || box_rows > rows)
    return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(depth)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2u,
                           static_cast<cuuint64_t>(cols) * static_cast<cuuint64_t>(rows) * 2u};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estride[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_epilogue_map(CUtensorMap* map, void* base, bool f32, int B, long long depth) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0 || B % 32 != 0 || B < 32 || depth < (f32 ? 1 : 2))
    return cudaErrorInvalidValue;
  const cuuint64_t esz = f32 ? 4u : 2u;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(B), static_cast<cuuint64_t>(B), static_cast<cuuint64_t>(depth)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(B) * esz, static_cast<cuuint64_t>(B) * B * esz};
  cuuint32_t box[3] = {32u, 32u, f32 ? 1u : 2u};
  cuuint32_t estride[3] = {1u, 1u, 1u};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims,
                   strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_split_stack_map(CUtensorMap* map, const void* base, int B, int nmat, int box_rows) {
  if (B % 128 != 0 || nmat < 1) return cudaErrorInvalidValue;
  return encode_f16_3d_map(map, base, B, B, 2ll * nmat, box_rows);
}

}  // namespace dash
