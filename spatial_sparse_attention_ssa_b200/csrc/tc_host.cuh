// Host-side helpers of the tensor-core kernels: TMA tensor maps and device facts (internal).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace ssa {
namespace tch {

constexpr int kRows = 128;  // query rows per tile of the tensor-core kernels

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D map over [rows, 64] bf16 with a box of `box_rows` rows (128 by default), 128-byte swizzle.
inline bool map_rows64(CUtensorMap* m, const void* base, int64_t rows, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {64, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map over Q [N, Hq, 64] bf16 with a box of (64, G heads, rows/G tokens): one box is a
// tile of `rows` query rows (128 by default).
inline bool map_q(CUtensorMap* m, const void* base, int64_t n, int hq, int G, int rows = kRows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)hq, (cuuint64_t)n};
  cuuint64_t strides[2] = {128, (cuuint64_t)hq * 128};
  cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(rows / G)};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over per-row fp32 scalars [N, Hq] with a box of (G heads, rows/G tokens), no swizzle:
// one box is the row scalars of a tile of `rows` rows (128 by default) in row order.
inline bool map_rowscalars(CUtensorMap* m, const float* base, int64_t n, int hq, int G, int rows = kRows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)hq, (cuuint64_t)n};
  cuuint64_t strides[1] = {(cuuint64_t)hq * 4};
  cuuint32_t box[2] = {(cuuint32_t)G, (cuuint32_t)(rows / G)};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// 3D map over Q-like [N, Hq, 64] bf16 with a box of one token's G heads (gathered row loads).
inline bool map_q_token(CUtensorMap* m, const void* base, int64_t n, int hq, int G) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)hq, (cuuint64_t)n};
  cuuint64_t strides[2] = {128, (cuuint64_t)hq * 128};
  cuuint32_t box[3] = {64, (cuuint32_t)G, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over per-row fp32 scalars [N, Hq] with a box of one token's G heads.
inline bool map_rowscalars_token(CUtensorMap* m, const float* base, int64_t n, int hq, int G) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)hq, (cuuint64_t)n};
  cuuint64_t strides[1] = {(cuuint64_t)hq * 4};
  cuuint32_t box[2] = {(cuuint32_t)G, 1};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace tch
}  // namespace ssa
