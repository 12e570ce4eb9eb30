// Step 2 of SSA: sparse 3D compression by mean pooling.
//
// Direct3D-S2 (hyper.ai, "方法"): the compression module groups tokens into
// m_cmp^3 blocks and builds one compressed key and value per block by mean
// pooling; LSRM (shuwu5.cn, "空间块划分与键值压缩") uses in-block AvgPool.
//
// One CTA per block.  It walks the block's members in ascending token order
// (blk.perm), copies their K/V rows into the block-sorted, head-major copies
// K_s/V_s [Hkv, N, d] (so a block's keys are one contiguous range), and sums
// them in fp64.  The stored mean is fp32(sum) / fp32(n) (IEEE division), then
// rounded to the storage type (bf16: round to nearest even).
#include "common.cuh"

namespace ssa {
namespace {

// Each thread owns two consecutive elements of the [Hkv*d] row of K (threads
// 0 .. hkv*d/2-1) or of V (the next hkv*d/2 threads).
template <typename T>
__global__ void pool_kernel(const T* __restrict__ k, const T* __restrict__ v, const int32_t* __restrict__ perm,
                            const int32_t* __restrict__ ptr, int count, int64_t N, int hkv, int d, T* __restrict__ ks, T* __restrict__ vs, T* __restrict__ kc,
                            T* __restrict__ vc) {
  const int row = hkv * d;
  const int half = row / 2;
  const int tid = threadIdx.x;
  if (tid >= 2 * half) return;
  const bool is_v = tid >= half;
  const int e = 2 * (is_v ? tid - half : tid);  // element within the [hkv, d] row
  const int g = e / d, c = e % d;
  const T* src = is_v ? v : k;
  T* dst_s = is_v ? vs : ks;
  T* dst_c = is_v ? vc : kc;
  for (int b = blockIdx.x; b < count; b += gridDim.x) {
    const int p0 = ptr[b], p1 = ptr[b + 1];
    double s0 = 0.0, s1 = 0.0;
    for (int p = p0; p < p1; ++p) {
      const int64_t t = perm[p];
      const T x0 = src[t * row + e];
      const T x1 = src[t * row + e + 1];
      s0 += (double)Elem<T>::to_f(x0);
      s1 += (double)Elem<T>::to_f(x1);
      T* o = dst_s + ((int64_t)g * N + p) * d + c;
      o[0] = x0;
      o[1] = x1;
    }
    const float n = (float)(p1 - p0);
    const float m0 = __fdiv_rn(__double2float_rn(s0), n);
    const float m1 = __fdiv_rn(__double2float_rn(s1), n);
    T* oc = dst_c + ((int64_t)g * count + b) * d + c;
    oc[0] = Elem<T>::from_f(m0);
    oc[1] = Elem<T>::from_f(m1);
  }
}

}  // namespace

cudaError_t launch_pool(int dtype, const void* k, const void* v, const ssa_partition* blk, int64_t N, int hkv,
                        int d, void* ks, void* vs, void* kc, void* vc, cudaStream_t st) {
  const int64_t count_host = blk->count;
  if (N == 0 || count_host == 0) return cudaSuccess;
  const int threads = ((hkv * d + 31) / 32) * 32;
  const int grid = (int)(count_host < 148 * 64 ? count_host : 148 * 64);
  if (dtype == SSA_DTYPE_BF16) {
    SSA_LAUNCH("pool_kernel", (pool_kernel<__nv_bfloat16>), grid, threads, 0, st, 
        (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, blk->perm, blk->ptr, (int)count_host, N, hkv, d,
        (__nv_bfloat16*)ks, (__nv_bfloat16*)vs, (__nv_bfloat16*)kc, (__nv_bfloat16*)vc);
  } else {
    SSA_LAUNCH("pool_kernel", (pool_kernel<float>), grid, threads, 0, st, (const float*)k, (const float*)v, blk->perm, blk->ptr,
                                                  (int)count_host, N, hkv, d, (float*)ks, (float*)vs, (float*)kc, (float*)vc);
  }
  return cudaGetLastError();
}

}  // namespace ssa
