// Step 2 of SSA: sparse 3D compression by mean pooling.
//
// Direct3D-S2 (hyper.ai, "方法"): the compression module groups tokens into
// m_cmp^3 blocks and builds one compressed key and value per block by mean
// pooling; LSRM (shuwu5.cn, "空间块划分与键值压缩") uses in-block AvgPool.
//
// One CTA per block.  The K and V rows of a token are split into 16-byte chunks
// (C chunks per token, K's first); thread t always handles chunk t % C of the
// members t / C, t / C + blockDim / C, ... (blockDim is a multiple of C), four
// members per round with their loads in flight together.  Each chunk is copied to
// the block-sorted, head-major K_s / V_s [Hkv, N, d] (a block's keys are one
// contiguous range) and summed in fp64; the per-thread partial sums are added
// across the threads of a chunk in shared memory.  The stored mean is
// fp32(sum) / fp32(n) (IEEE division), then rounded to the storage type (bf16:
// round to nearest even).  fp64 sums of bf16 values are exact, so the order of the
// additions does not change the result.
#include "common.cuh"

namespace ssa {
namespace {

constexpr int kPoolThreads = 256;   // threads per CTA when a token has at most 256 chunks
constexpr int kPoolMaxChunks = 1024;
constexpr int kPoolUnroll = 4;

template <typename T>
struct Chunk;  // elements of a 16-byte chunk
template <>
struct Chunk<__nv_bfloat16> {
  static constexpr int E = 8;
  static __device__ __forceinline__ void widen(const uint4& u, double* x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = (double)__uint_as_float(w[j] << 16);
      x[2 * j + 1] = (double)__uint_as_float(w[j] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint4 narrow(const float* m) {
    return make_uint4(pack_bf16x2(m[0], m[1]), pack_bf16x2(m[2], m[3]), pack_bf16x2(m[4], m[5]),
                      pack_bf16x2(m[6], m[7]));
  }
};
template <>
struct Chunk<float> {
  static constexpr int E = 4;
  static __device__ __forceinline__ void widen(const uint4& u, double* x) {
    x[0] = (double)__uint_as_float(u.x);
    x[1] = (double)__uint_as_float(u.y);
    x[2] = (double)__uint_as_float(u.z);
    x[3] = (double)__uint_as_float(u.w);
  }
  static __device__ __forceinline__ uint4 narrow(const float* m) {
    return make_uint4(__float_as_uint(m[0]), __float_as_uint(m[1]), __float_as_uint(m[2]), __float_as_uint(m[3]));
  }
};

// C = chunks per token (K and V together), cpr = C / 2 chunks per K (or V) row,
// cpd = chunks per head row of d elements.  blockDim.x is a multiple of C.
template <typename T>
__global__ void __launch_bounds__(kPoolMaxChunks) pool_kernel(
    const T* __restrict__ k, const T* __restrict__ v, const int32_t* __restrict__ perm,
    const int32_t* __restrict__ ptr, int count, int64_t N, int C, int cpd, T* __restrict__ ks, T* __restrict__ vs,
    T* __restrict__ kc, T* __restrict__ vc) {
  constexpr int E = Chunk<T>::E;
  extern __shared__ double part[];  // [blockDim / C][C][E]
  const int tid = threadIdx.x;
  const int cpr = C / 2;
  const int c = tid % C;             // chunk of this thread
  const int lane_m = tid / C;        // first member offset
  const int stride_m = blockDim.x / C;
  const bool is_v = c >= cpr;
  const int cr = is_v ? c - cpr : c;  // chunk within the K (or V) row
  const int g = cr / cpd, cc = cr % cpd;
  const uint4* src = reinterpret_cast<const uint4*>(is_v ? v : k);
  uint4* dst_s = reinterpret_cast<uint4*>(is_v ? vs : ks);
  for (int b = blockIdx.x; b < count; b += gridDim.x) {
    const int p0 = ptr[b], p1 = ptr[b + 1];
    double sum[E];
#pragma unroll
    for (int j = 0; j < E; ++j) sum[j] = 0.0;
    for (int p = p0 + lane_m; p < p1; p += kPoolUnroll * stride_m) {
      int64_t t[kPoolUnroll];
      uint4 x[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        const int pu = p + u * stride_m;
        t[u] = pu < p1 ? (int64_t)perm[pu] : -1;
      }
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u)
        x[u] = t[u] >= 0 ? __ldcs(src + t[u] * cpr + cr) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        if (t[u] < 0) continue;
        const int pu = p + u * stride_m;
        dst_s[((int64_t)g * N + pu) * cpd + cc] = x[u];
        double w[E];
        Chunk<T>::widen(x[u], w);
#pragma unroll
        for (int j = 0; j < E; ++j) sum[j] += w[j];
      }
    }
#pragma unroll
    for (int j = 0; j < E; ++j) part[(size_t)tid * E + j] = sum[j];
    __syncthreads();
    if (tid < C) {
      double tot[E];
#pragma unroll
      for (int j = 0; j < E; ++j) tot[j] = 0.0;
      for (int r = 0; r < stride_m; ++r) {
#pragma unroll
        for (int j = 0; j < E; ++j) tot[j] += part[((size_t)r * C + tid) * E + j];
      }
      const float n = (float)(p1 - p0);
      float m[E];
#pragma unroll
      for (int j = 0; j < E; ++j) m[j] = __fdiv_rn(__double2float_rn(tot[j]), n);
      uint4* oc = reinterpret_cast<uint4*>(is_v ? vc : kc);
      oc[((int64_t)g * count + b) * cpd + cc] = Chunk<T>::narrow(m);
    }
    __syncthreads();
  }
}

template <typename T>
cudaError_t pool_t(const void* k, const void* v, const ssa_partition* blk, int64_t N, int hkv, int d, void* ks,
                   void* vs, void* kc, void* vc, cudaStream_t st) {
  constexpr int E = Chunk<T>::E;
  const int cpd = d / E;              // d is a multiple of 8
  const int C = 2 * hkv * cpd;        // chunks per token, K and V
  if (C > kPoolMaxChunks) return cudaErrorInvalidValue;
  const int threads = C <= kPoolThreads ? (kPoolThreads / C) * C : C;
  const size_t smem = sizeof(double) * E * threads;
  const int64_t count = blk->count;
  const int grid = (int)(count < 148 * 64 ? count : 148 * 64);
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(pool_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
    attr_done = true;
  }
  SSA_LAUNCH("pool_kernel", pool_kernel<T>, grid, threads, smem, st, static_cast<const T*>(k),
             static_cast<const T*>(v), blk->perm, blk->ptr, (int)count, N, C, cpd, static_cast<T*>(ks),
             static_cast<T*>(vs), static_cast<T*>(kc), static_cast<T*>(vc));
  return cudaGetLastError();
}

}  // namespace

bool pool_supported(int dtype, int hkv, int d) {
  const int E = dtype == SSA_DTYPE_BF16 ? 8 : 4;
  return d % 8 == 0 && 2 * hkv * (d / E) <= kPoolMaxChunks;
}

cudaError_t launch_pool(int dtype, const void* k, const void* v, const ssa_partition* blk, int64_t N, int hkv,
                        int d, void* ks, void* vs, void* kc, void* vc, cudaStream_t st) {
  if (N == 0 || blk->count == 0) return cudaSuccess;
  if (dtype == SSA_DTYPE_BF16) return pool_t<__nv_bfloat16>(k, v, blk, N, hkv, d, ks, vs, kc, vc, st);
  return pool_t<float>(k, v, blk, N, hkv, d, ks, vs, kc, vc, st);
}

}  // namespace ssa
