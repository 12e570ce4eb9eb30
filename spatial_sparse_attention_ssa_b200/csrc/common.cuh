// Shared device helpers and launcher declarations of libssa (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssa.h"

namespace ssa {

// Device check bits recorded by kernels (or-ed into the status word).
enum : int { kStatusCoordRange = 1, kStatusSeqlens = 2, kStatusTimeout = 4, kStatusSelection = 8 };

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// element access for the two storage types
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};

template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load 32 consecutive elements (16-byte aligned) as floats.
__device__ __forceinline__ void load32(const float* __restrict__ p, float* out) {
  const float4* p4 = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 v = __ldg(p4 + i);
    out[4 * i + 0] = v.x;
    out[4 * i + 1] = v.y;
    out[4 * i + 2] = v.z;
    out[4 * i + 3] = v.w;
  }
}

__device__ __forceinline__ void load32(const __nv_bfloat16* __restrict__ p, float* out) {
  const uint4* p4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 v = __ldg(p4 + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      out[8 * i + 2 * j + 0] = __uint_as_float(w[j] << 16);
      out[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
}

__device__ __forceinline__ void store32(float* p, const float* v) {
  float4* p4 = reinterpret_cast<float4*>(p);
#pragma unroll
  for (int i = 0; i < 8; ++i) p4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// (x0, x1) = hi + lo with hi the bf16 rounding and lo the bf16 rounding of the
// remainder: hi + lo carries about 16 significant bits.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16x2(x0 - hf.x, x1 - hf.y);
}

__device__ __forceinline__ void store32(__nv_bfloat16* p, const float* v) {
  uint4* p4 = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    p4[i] = make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                       pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  }
}

// Sequence containing token / tile index `x` given an inclusive-exclusive prefix
// array pre[0..n] (pre[0] = 0): largest s with pre[s] <= x (skips empty ranges).
__device__ __forceinline__ int find_segment(const int32_t* __restrict__ pre, int n, int64_t x) {
  int lo = 0, hi = n;  // invariant: pre[lo] <= x < pre[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if ((int64_t)pre[mid] <= x)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

}  // namespace ssa

// ---------------------------------------------------------------------------
// Internal launchers (defined in the .cu files; all enqueue on `st`).
// ---------------------------------------------------------------------------
namespace ssa {

// Device-wide exclusive scan of n int32 values; `tmp` needs scan_tmp_ints(n) ints.
size_t scan_tmp_ints(int64_t n);
cudaError_t exclusive_scan(const int32_t* in, int32_t* out, int64_t n, int32_t* tmp, cudaStream_t st);

// Stable LSD radix sort of (key, val) pairs by the low `bits` bits of key.
// Buffers: keys/vals in (a) and alternate (b); result lands in a or b (returned flag).
size_t radix_tmp_ints(int64_t n);
cudaError_t radix_sort_pairs(uint64_t* keys_a, int32_t* vals_a, uint64_t* keys_b, int32_t* vals_b,
                             int64_t n, int bits, int32_t* tmp, bool* result_in_b, cudaStream_t st);

// Binning of one partition (see ssa_bin).
size_t bin_ws_bytes(int32_t S, int64_t N);
// Synchronises `st` and reads up to three device ints (null sources read as 0) through
// a pinned, mapped host buffer written by a kernel: no copy engine is involved.
cudaError_t read_ints_to_host(const int32_t* s0, const int32_t* s1, const int32_t* s2, int32_t* out,
                              cudaStream_t st);

cudaError_t bin_partition(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N,
                          int32_t R, int32_t m, ssa_partition* out, int32_t* d_count, void* ws,
                          int* d_status, cudaStream_t st);

}  // namespace ssa

namespace ssa {
// Tracing hooks (profile.cu): every library kernel launch is wrapped by these.
void prof_begin(const char* name, cudaStream_t st);
void prof_end(cudaStream_t st);
}  // namespace ssa

// Launch `kernel<<<grid, block, smem, st>>>(args...)` with launch counting and,
// when enabled, per-kernel CUDA-event timing under `name`.
#define SSA_LAUNCH(name, kernel, grid, block, smem, st, ...)  \
  do {                                                       \
    ::ssa::prof_begin(name, st);                             \
    kernel<<<grid, block, smem, st>>>(__VA_ARGS__);          \
    ::ssa::prof_end(st);                                     \
  } while (0)
