// Reading a few device ints on the host (cell counts, check words) without a copy
// engine.  A cudaMemcpy of 4 bytes is a DMA transfer: on a stream that runs beside
// bulk copies of other streams (a pipeline that downloads the previous step's results
// while this step bins), it can wait in the engine's queue behind gigabytes of those
// transfers and stall the caller for their whole duration.  Instead, a one-thread
// kernel stores the values into a small pinned, mapped host buffer (writes across
// PCIe, no engine), and the host reads them after the stream synchronises.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

__global__ void ints_to_host_kernel(const int32_t* s0, const int32_t* s1, const int32_t* s2, int32_t* dst) {
  dst[0] = s0 ? *s0 : 0;
  dst[1] = s1 ? *s1 : 0;
  dst[2] = s2 ? *s2 : 0;
  __threadfence_system();
}

// 64 bytes of pinned, mapped host memory per calling thread, allocated on its first
// read and kept until the process exits (portable: usable from every device).
int32_t* host_slot() {
  static thread_local int32_t* slot = nullptr;
  if (!slot) {
    void* p = nullptr;
    if (cudaHostAlloc(&p, 64, cudaHostAllocMapped | cudaHostAllocPortable) != cudaSuccess) return nullptr;
    slot = static_cast<int32_t*>(p);
  }
  return slot;
}

}  // namespace

cudaError_t read_ints_to_host(const int32_t* s0, const int32_t* s1, const int32_t* s2, int32_t* out,
                              cudaStream_t st) {
  int32_t* h = host_slot();
  if (!h) return cudaErrorMemoryAllocation;
  void* d = nullptr;
  cudaError_t e = cudaHostGetDevicePointer(&d, h, 0);
  if (e != cudaSuccess) return e;
  SSA_LAUNCH("ints_to_host_kernel", ints_to_host_kernel, 1, 1, 0, st, s0, s1, s2, static_cast<int32_t*>(d));
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  const volatile int32_t* v = h;
  out[0] = v[0];
  out[1] = v[1];
  out[2] = v[2];
  return cudaSuccess;
}

}  // namespace ssa
