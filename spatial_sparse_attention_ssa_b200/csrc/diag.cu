// Diagnostics of the device building blocks (no counterpart on the pages): they let
// tests exercise, on the GPU and through the C ABI, the bounded mbarrier waits that
// every tensor-core kernel relies on, and the exponential the kernels evaluate on the
// FMA pipe.
#include "common.cuh"
#include "tc.cuh"

namespace ssa {
namespace {

// One warp waits on an mbarrier that nothing ever arrives at: first lane 0 alone
// (mbar_wait), then the whole warp (mbar_wait_warp).  Each wait gives up after its
// bound; the kernel then records the timeout in the device check word and returns,
// as the attention kernels do.  out[0] / out[1] = 1 if the respective wait gave up.
__global__ void diag_wait_timeout_kernel(int* status, int* out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) out[0] = tc::mbar_wait(&bar, 0) ? 0 : 1;
  __syncwarp();
  const bool ok = tc::mbar_wait_warp(&bar, 0);
  if (threadIdx.x == 0) {
    out[1] = ok ? 0 : 1;
    if (!ok || out[0]) atomicOr(status, kStatusTimeout);
  }
}

// y_poly[i] = ex2_poly2(x[i]), y_mufu[i] = ex2.approx(x[i]).
__global__ void diag_ex2_kernel(const float* __restrict__ x, float* __restrict__ y_poly, float* __restrict__ y_mufu,
                                int64_t n) {
  for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n;
       i += 2 * (int64_t)gridDim.x * blockDim.x) {
    const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
    const float2 p = tc::ex2_poly2(make_float2(a, b));
    y_poly[i] = p.x;
    y_mufu[i] = tc::ex2(a);
    if (i + 1 < n) {
      y_poly[i + 1] = p.y;
      y_mufu[i + 1] = tc::ex2(b);
    }
  }
}

}  // namespace

cudaError_t diag_wait_timeout(int* status, int* out, cudaStream_t st) {
  SSA_LAUNCH("diag_wait_timeout_kernel", diag_wait_timeout_kernel, 1, 32, 0, st, status, out);
  return cudaGetLastError();
}

cudaError_t diag_ex2(const float* x, float* y_poly, float* y_mufu, int64_t n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n / 2 + 255) / 256;
  SSA_LAUNCH("diag_ex2_kernel", diag_ex2_kernel, (int)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, st, x, y_poly,
             y_mufu, n);
  return cudaGetLastError();
}

}  // namespace ssa
