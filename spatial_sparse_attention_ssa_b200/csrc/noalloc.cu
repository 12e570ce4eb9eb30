// ssa_bin_noalloc: coordinate binning for callers that cannot allocate device memory.
//
// ssa_bin needs a caller-provided workspace for its radix sort and scans.  Some
// callers cannot get one on demand: a plugin whose host application owns all
// device memory through its own pool and forbids allocations from outside it,
// a latency-critical loop where cudaMalloc / cudaFree would synchronise the
// device, or a process that reserved nearly all GPU memory up front.  This
// entry point runs the same binning kernels with their scratch in a fixed,
// file-scope device array instead, so it allocates nothing.
//
// Cost of that choice: every GPU that loads the library keeps the array
// (kNoallocBytes, about 11 MB) until the process exits, inputs are limited to
// SSA_BIN_NOALLOC_MAX_TOKENS tokens, and all calls on a device share the one
// array -- calls whose work overlaps on the GPU (different streams, or host
// threads racing) corrupt each other's results.
#include "common.cuh"

namespace {

// Scratch for binning up to SSA_BIN_NOALLOC_MAX_TOKENS tokens: the bytes
// ssa::bin_ws_bytes() needs at that size, plus 256 bytes for the two cell
// counts and the check word.  bin_ws_bytes grows with N only, so the bound
// holds for every smaller N (checked again at run time).
constexpr int64_t kNoallocTokens = SSA_BIN_NOALLOC_MAX_TOKENS;
constexpr size_t kNoallocBytes = 11u << 20;  // 11 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a stand-in for the symbol, never a device address, so
// kernels must be given this looked-up pointer.  It is looked up on every call
// (a cheap runtime query): a cached address would go stale if the program reset
// the device and the module were loaded again at another address.
ssa_status scratch_for_current_device(unsigned char** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess || !ptr) return SSA_ERR_CUDA;
  *out = static_cast<unsigned char*>(ptr);
  return SSA_OK;
}

}  // namespace

extern "C" SSA_API ssa_status ssa_bin_noalloc(const int32_t* coords, const int32_t* cu_seqlens, int32_t S,
                                              int64_t N, int32_t R, int32_t m_cmp, int32_t m_win,
                                              ssa_partition* blk, ssa_partition* win, void* stream) {
  if (S < 1 || N < 0 || R < 1 || R > (1 << 20) || m_cmp < 1 || m_win < 1) return SSA_ERR_INVALID_ARG;
  if (!cu_seqlens || (N > 0 && !coords) || !blk || !win) return SSA_ERR_INVALID_ARG;
  // per-token arrays and cell keys may be null when there are no tokens (nothing is written there)
  if (!blk->ptr || !blk->cu || (N > 0 && (!blk->id || !blk->perm || !blk->key))) return SSA_ERR_INVALID_ARG;
  if (!win->ptr || !win->cu || (N > 0 && (!win->id || !win->perm || !win->key))) return SSA_ERR_INVALID_ARG;
  // Inputs above the fixed scratch are refused before any work is enqueued.
  const size_t need = ssa::bin_ws_bytes(S, N);
  if (N > kNoallocTokens || need + 256 > kNoallocBytes) return SSA_ERR_WORKSPACE;
  int sbits = 0;
  while ((1ll << sbits) < S) ++sbits;
  for (int m : {m_cmp, m_win}) {
    int cbits = 1;
    while ((1ll << cbits) < (R + m - 1) / m) ++cbits;
    if (sbits + 3 * cbits > 64) return SSA_ERR_UNSUPPORTED;
  }

  unsigned char* scratch = nullptr;
  ssa_status st0 = scratch_for_current_device(&scratch);
  if (st0 != SSA_OK) return st0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Layout: [0, need) sort / scan buffers (fully overwritten before being read),
  // then the two cell counts and the check word, which must start at zero.
  int32_t* d_counts = reinterpret_cast<int32_t*>(scratch + need);
  int* d_status = reinterpret_cast<int*>(scratch + need + 2 * sizeof(int32_t));
  cudaError_t e = cudaMemsetAsync(d_counts, 0, 2 * sizeof(int32_t) + sizeof(int), st);
  if (e == cudaSuccess) e = ssa::bin_partition(coords, cu_seqlens, S, N, R, m_cmp, blk, d_counts, scratch, d_status, st);
  if (e == cudaSuccess) e = ssa::bin_partition(coords, cu_seqlens, S, N, R, m_win, win, d_counts + 1, scratch, d_status, st);
  if (e != cudaSuccess) return SSA_ERR_CUDA;
  int32_t h[3] = {0, 0, 0};
  if (ssa::read_ints_to_host(d_counts, d_counts + 1, reinterpret_cast<const int32_t*>(d_status), h, st) != cudaSuccess)
    return SSA_ERR_CUDA;
  blk->count = h[0];
  win->count = h[1];
  if (h[2] & ssa::kStatusTimeout) return SSA_ERR_TIMEOUT;
  if (h[2]) return SSA_ERR_COORD_RANGE;
  return SSA_OK;
}
