// Step 1 of SSA: binning of tokens into m^3 cells of the integer grid.
//
// Direct3D-S2 (hyper.ai, "方法"): SSA partitions tokens into blocks by their 3D
// coordinates (not by 1D index) and runs window attention in non-overlapping
// m_win^3 windows.  A cell id is a function of (sequence, floor(coord / m)) only;
// cells are numbered per sequence in lexicographic (x, y, z) order.
//
// Implementation: a composite integer key (sequence | cx | cy | cz) per token, a
// stable LSD radix sort of (key, token index), then head flags + scan give the
// compacted ids, the CSR pointers and per-sequence offsets.  All integer work,
// bit-exact and deterministic.
#include "common.cuh"

namespace ssa {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanItems = 16;
constexpr int kScanChunk = kScanThreads * kScanItems;  // 4096

constexpr int kRadixThreads = 256;
constexpr int kRadixRounds = 16;
constexpr int kRadixTile = kRadixThreads * kRadixRounds;  // 4096
constexpr int kRadixBins = 256;

__host__ __device__ inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// exclusive scan
// ---------------------------------------------------------------------------

// Block-wide exclusive scan of the 4096-element chunk starting at `base`;
// returns the chunk total.  `sh` holds kScanChunk ints + 8 warp totals.
__device__ int block_scan_chunk(const int32_t* in, int32_t* out, int64_t base, int64_t n, int offset,
                                int* sh) {
  const int tid = threadIdx.x;
  for (int i = tid; i < kScanChunk; i += kScanThreads) {
    int64_t g = base + i;
    sh[i] = g < n ? in[g] : 0;
  }
  __syncthreads();
  int loc[kScanItems];
  int sum = 0;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    loc[j] = sum;
    sum += sh[tid * kScanItems + j];
  }
  // warp inclusive scan of per-thread sums
  const int lane = tid & 31, warp = tid >> 5;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int* wsum = sh + kScanChunk;
  __syncthreads();  // everyone has read sh
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int wofs = 0, total = 0;
  for (int w = 0; w < kScanThreads / 32; ++w) {
    if (w < warp) wofs += wsum[w];
    total += wsum[w];
  }
  const int tofs = offset + wofs + incl - sum;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) sh[tid * kScanItems + j] = tofs + loc[j];
  __syncthreads();
  for (int i = tid; i < kScanChunk; i += kScanThreads) {
    int64_t g = base + i;
    if (g < n) out[g] = sh[i];
  }
  __syncthreads();
  return total;
}

__global__ void scan_reduce_kernel(const int32_t* __restrict__ in, int64_t n, int32_t* __restrict__ sums) {
  __shared__ int red[kScanThreads / 32];
  const int64_t base = (int64_t)blockIdx.x * kScanChunk;
  int s = 0;
  for (int i = threadIdx.x; i < kScanChunk; i += kScanThreads) {
    int64_t g = base + i;
    if (g < n) s += in[g];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) t += red[w];
    sums[blockIdx.x] = t;
  }
}

// Single CTA: exclusive scan of `n` chunk sums in place.
__global__ void scan_sums_kernel(int32_t* sums, int64_t n) {
  __shared__ int sh[kScanChunk + 8];
  int carry = 0;
  for (int64_t base = 0; base < n; base += kScanChunk) {
    carry += block_scan_chunk(sums, sums, base, n, carry, sh);
  }
}

// Single CTA: exclusive scan of a short array (at most kScanSmallChunks chunks) in one
// launch; the plans' scans have S + 1 or W + 1 entries, where the launch gaps of the
// three-kernel form would cost more than the scan.
constexpr int64_t kScanSmallChunks = 8;
__global__ void scan_small_kernel(const int32_t* in, int32_t* out, int64_t n) {
  __shared__ int sh[kScanChunk + 8];
  int carry = 0;
  for (int64_t base = 0; base < n; base += kScanChunk) carry += block_scan_chunk(in, out, base, n, carry, sh);
}

__global__ void scan_apply_kernel(const int32_t* __restrict__ in, int32_t* __restrict__ out, int64_t n,
                                  const int32_t* __restrict__ sums) {
  __shared__ int sh[kScanChunk + 8];
  block_scan_chunk(in, out, (int64_t)blockIdx.x * kScanChunk, n, sums[blockIdx.x], sh);
}

// ---------------------------------------------------------------------------
// radix sort
// ---------------------------------------------------------------------------

__global__ void radix_hist_kernel(const uint64_t* __restrict__ keys, int64_t n, int shift, int num_tiles,
                                  int32_t* __restrict__ counts) {
  __shared__ int hist[kRadixBins];
  hist[threadIdx.x] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kRadixTile;
  for (int i = threadIdx.x; i < kRadixTile; i += kRadixThreads) {
    int64_t g = base + i;
    if (g < n) atomicAdd(&hist[(keys[g] >> shift) & 0xff], 1);
  }
  __syncthreads();
  counts[(int64_t)threadIdx.x * num_tiles + blockIdx.x] = hist[threadIdx.x];
}

// Stable scatter: items are ranked in index order inside the tile (16 rounds of
// 256 consecutive items; warp match + per-warp digit counts give the order).
__global__ void radix_scatter_kernel(const uint64_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in,
                                     uint64_t* __restrict__ keys_out, int32_t* __restrict__ vals_out, int64_t n,
                                     int shift, int num_tiles, const int32_t* __restrict__ offsets) {
  constexpr int kWarps = kRadixThreads / 32;
  __shared__ int running[kRadixBins];
  __shared__ int warp_cnt[kWarps][kRadixBins];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  running[tid] = 0;
  const int64_t base = (int64_t)blockIdx.x * kRadixTile;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < kRadixRounds; ++r) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) warp_cnt[w][tid] = 0;
    __syncthreads();
    const int64_t g = base + (int64_t)r * kRadixThreads + tid;
    const bool valid = g < n;
    uint64_t key = valid ? keys_in[g] : 0ull;
    int val = valid ? vals_in[g] : 0;
    const int digit = valid ? (int)((key >> shift) & 0xff) : kRadixBins;  // sentinel for invalid
    const uint32_t peers = __match_any_sync(0xffffffffu, digit);
    const int lrank = __popc(peers & lt_mask);
    if (valid && lrank == 0) warp_cnt[warp][digit] = __popc(peers);
    __syncthreads();
    {  // thread `tid` owns digit `tid`: prefix over warps, continuing the tile's running count
      int run = running[tid];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        int c = warp_cnt[w][tid];
        warp_cnt[w][tid] = run;
        run += c;
      }
      running[tid] = run;
    }
    __syncthreads();
    if (valid) {
      const int64_t pos = (int64_t)offsets[(int64_t)digit * num_tiles + blockIdx.x] + warp_cnt[warp][digit] + lrank;
      keys_out[pos] = key;
      vals_out[pos] = val;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// binning kernels
// ---------------------------------------------------------------------------

__global__ void check_seqlens_kernel(const int32_t* __restrict__ cu, int32_t S, int64_t N, int* status) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i <= S; i += (int64_t)gridDim.x * blockDim.x) {
    bool bad = false;
    if (i == 0 && cu[0] != 0) bad = true;
    if (i == S && (int64_t)cu[S] != N) bad = true;
    if (i < S && cu[i] > cu[i + 1]) bad = true;
    if (bad) atomicOr(status, kStatusSeqlens);
  }
}

__global__ void make_keys_kernel(const int32_t* __restrict__ coords, const int32_t* __restrict__ cu, int32_t S,
                                 int64_t N, int32_t R, int32_t m, int cbits, uint64_t* __restrict__ keys,
                                 int32_t* __restrict__ vals, int* status) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < N; t += (int64_t)gridDim.x * blockDim.x) {
    const int s = find_segment(cu, S, t);
    uint64_t key = (uint64_t)s;
    bool bad = false;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      int c = coords[3 * t + a];
      if (c < 0 || c >= R) {
        bad = true;
        c = c < 0 ? 0 : R - 1;
      }
      key = (key << cbits) | (uint64_t)(c / m);
    }
    if (bad) atomicOr(status, kStatusCoordRange);
    keys[t] = key;
    vals[t] = (int32_t)t;
  }
}

__global__ void head_flags_kernel(const uint64_t* __restrict__ keys, int64_t N, int32_t* __restrict__ flags) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += (int64_t)gridDim.x * blockDim.x)
    flags[i] = (i == 0 || keys[i] != keys[i - 1]) ? 1 : 0;
}

__global__ void finalize_kernel(const uint64_t* __restrict__ keys, const int32_t* __restrict__ vals,
                                const int32_t* __restrict__ flags, const int32_t* __restrict__ excl, int64_t N,
                                int cbits, int32_t* __restrict__ id, int32_t* __restrict__ perm,
                                int32_t* __restrict__ ptr, int32_t* __restrict__ cellkey, int32_t* d_count) {
  const uint64_t cmask = (1ull << cbits) - 1ull;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += (int64_t)gridDim.x * blockDim.x) {
    const int f = flags[i];
    const int gid = excl[i] + f - 1;
    const int t = vals[i];
    perm[i] = t;
    id[t] = gid;
    if (f) {
      const uint64_t k = keys[i];
      ptr[gid] = (int32_t)i;
      cellkey[3 * (int64_t)gid + 0] = (int32_t)((k >> (2 * cbits)) & cmask);
      cellkey[3 * (int64_t)gid + 1] = (int32_t)((k >> cbits) & cmask);
      cellkey[3 * (int64_t)gid + 2] = (int32_t)(k & cmask);
    }
    if (i == N - 1) {
      const int count = gid + 1;
      ptr[count] = (int32_t)N;
      *d_count = count;
    }
  }
}

__global__ void seq_offsets_kernel(const int32_t* __restrict__ cu_seqlens, int32_t S, int64_t N,
                                   const int32_t* __restrict__ excl, const int32_t* __restrict__ d_count,
                                   int32_t* __restrict__ cu_out) {
  for (int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; s <= S; s += (int64_t)gridDim.x * blockDim.x) {
    int64_t pos = cu_seqlens[s];
    pos = pos < 0 ? 0 : pos;
    cu_out[s] = pos < N ? excl[pos] : *d_count;
  }
}

inline int grid_for(int64_t n, int threads) {
  int64_t b = cdiv(n, threads);
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return (int)b;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

size_t scan_tmp_ints(int64_t n) { return (size_t)cdiv(n, kScanChunk) + 64; }

cudaError_t exclusive_scan(const int32_t* in, int32_t* out, int64_t n, int32_t* tmp, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t nc = cdiv(n, kScanChunk);
  if (nc <= kScanSmallChunks) {
    SSA_LAUNCH("scan_small_kernel", scan_small_kernel, 1, kScanThreads, 0, st, in, out, n);
    return cudaGetLastError();
  }
  SSA_LAUNCH("scan_reduce_kernel", scan_reduce_kernel, (unsigned)nc, kScanThreads, 0, st, in, n, tmp);
  SSA_LAUNCH("scan_sums_kernel", scan_sums_kernel, 1, kScanThreads, 0, st, tmp, nc);
  SSA_LAUNCH("scan_apply_kernel", scan_apply_kernel, (unsigned)nc, kScanThreads, 0, st, in, out, n, tmp);
  return cudaGetLastError();
}

size_t radix_tmp_ints(int64_t n) {
  const int64_t tiles = cdiv(n > 0 ? n : 1, kRadixTile);
  const int64_t m = tiles * kRadixBins;
  return (size_t)(2 * m) + scan_tmp_ints(m) + 64;
}

cudaError_t radix_sort_pairs(uint64_t* keys_a, int32_t* vals_a, uint64_t* keys_b, int32_t* vals_b, int64_t n,
                             int bits, int32_t* tmp, bool* result_in_b, cudaStream_t st) {
  *result_in_b = false;
  if (n <= 1 || bits <= 0) return cudaSuccess;
  const int num_tiles = (int)cdiv(n, kRadixTile);
  const int64_t m = (int64_t)num_tiles * kRadixBins;
  int32_t* counts = tmp;
  int32_t* offsets = tmp + m;
  int32_t* scratch = tmp + 2 * m;
  uint64_t *ki = keys_a, *ko = keys_b;
  int32_t *vi = vals_a, *vo = vals_b;
  for (int shift = 0; shift < bits; shift += 8) {
    SSA_LAUNCH("radix_hist_kernel", radix_hist_kernel, num_tiles, kRadixThreads, 0, st, ki, n, shift, num_tiles, counts);
    cudaError_t e = exclusive_scan(counts, offsets, m, scratch, st);
    if (e != cudaSuccess) return e;
    SSA_LAUNCH("radix_scatter_kernel", radix_scatter_kernel, num_tiles, kRadixThreads, 0, st, ki, vi, ko, vo, n, shift, num_tiles, offsets);
    std::swap(ki, ko);
    std::swap(vi, vo);
    *result_in_b = !*result_in_b;
  }
  return cudaGetLastError();
}

size_t bin_ws_bytes(int32_t S, int64_t N) {
  const int64_t n = N > 0 ? N : 1;
  size_t b = 0;
  b += 2 * align256(sizeof(uint64_t) * n);   // keys a/b
  b += 2 * align256(sizeof(int32_t) * n);    // vals a/b
  b += 2 * align256(sizeof(int32_t) * n);    // flags, excl
  size_t t = radix_tmp_ints(n);
  size_t t2 = scan_tmp_ints(n);
  b += align256(sizeof(int32_t) * (t > t2 ? t : t2));
  (void)S;
  return b;
}

cudaError_t bin_partition(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N, int32_t R,
                          int32_t m, ssa_partition* out, int32_t* d_count, void* ws, int* d_status,
                          cudaStream_t st) {
  int cbits = 1;
  const int64_t cells = cdiv(R, m);
  while ((1ll << cbits) < cells) ++cbits;
  int sbits = 0;
  while ((1ll << sbits) < S) ++sbits;
  const int bits = sbits + 3 * cbits;  // caller checked bits <= 64

  char* p = static_cast<char*>(ws);
  const int64_t n = N > 0 ? N : 1;
  uint64_t* keys_a = reinterpret_cast<uint64_t*>(p); p += align256(sizeof(uint64_t) * n);
  uint64_t* keys_b = reinterpret_cast<uint64_t*>(p); p += align256(sizeof(uint64_t) * n);
  int32_t* vals_a = reinterpret_cast<int32_t*>(p); p += align256(sizeof(int32_t) * n);
  int32_t* vals_b = reinterpret_cast<int32_t*>(p); p += align256(sizeof(int32_t) * n);
  int32_t* flags = reinterpret_cast<int32_t*>(p); p += align256(sizeof(int32_t) * n);
  int32_t* excl = reinterpret_cast<int32_t*>(p); p += align256(sizeof(int32_t) * n);
  int32_t* tmp = reinterpret_cast<int32_t*>(p);

  SSA_LAUNCH("check_seqlens_kernel", check_seqlens_kernel, grid_for(S + 1, 256), 256, 0, st, cu_seqlens, S, N, d_status);
  if (N == 0) {
    cudaMemsetAsync(out->cu, 0, sizeof(int32_t) * (S + 1), st);
    cudaMemsetAsync(out->ptr, 0, sizeof(int32_t), st);
    cudaMemsetAsync(d_count, 0, sizeof(int32_t), st);
    return cudaGetLastError();
  }
  SSA_LAUNCH("make_keys_kernel", make_keys_kernel, grid_for(N, 256), 256, 0, st, coords, cu_seqlens, S, N, R, m, cbits, keys_a, vals_a,
                                                     d_status);
  bool in_b = false;
  cudaError_t e = radix_sort_pairs(keys_a, vals_a, keys_b, vals_b, N, bits, tmp, &in_b, st);
  if (e != cudaSuccess) return e;
  const uint64_t* ks = in_b ? keys_b : keys_a;
  const int32_t* vs = in_b ? vals_b : vals_a;
  SSA_LAUNCH("head_flags_kernel", head_flags_kernel, grid_for(N, 256), 256, 0, st, ks, N, flags);
  e = exclusive_scan(flags, excl, N, tmp, st);
  if (e != cudaSuccess) return e;
  SSA_LAUNCH("finalize_kernel", finalize_kernel, grid_for(N, 256), 256, 0, st, ks, vs, flags, excl, N, cbits, out->id, out->perm, out->ptr,
                                                    out->key, d_count);
  SSA_LAUNCH("seq_offsets_kernel", seq_offsets_kernel, grid_for(S + 1, 256), 256, 0, st, cu_seqlens, S, N, excl, d_count, out->cu);
  return cudaGetLastError();
}

}  // namespace ssa
