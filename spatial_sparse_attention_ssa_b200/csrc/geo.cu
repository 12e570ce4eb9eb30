// 3D-aware block routing (LSRM, shuwu5.cn/article/2502.html, "3D 感知空间块路由机制"),
// voxel-only case: every token selects the k blocks of its sequence whose tokens come
// nearest to it -- the shortest Euclidean distance between voxel centres -- with ties
// going to the lower block id.  Voxel centres differ by integer vectors, so squared
// distances are exact integers and the selection is exact.
//
// One warp per token.  For every block of the sequence a lower bound (the distance to
// the block's m^3 cell) and an upper bound (the distance to the block's first member)
// are computed.  The keff-th smallest of the 32 per-lane minima of the upper bounds, T,
// bounds the keff-th smallest distance from above (keff blocks reach it), so only
// blocks whose lower bound is <= T can be selected.  Those candidates get their exact
// distance (every member scanned, coordinates in block order); the keff smallest
// (distance, id) keys are kept in per-lane sorted lists and merged across the warp.
#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

constexpr int kGeoWarps = 8;    // warps (tokens in flight) per CTA
constexpr int kGeoCand = 512;   // candidate blocks per warp held in shared memory

__device__ __forceinline__ uint32_t dist2(int ax, int ay, int az, int bx, int by, int bz) {
  const int dx = ax - bx, dy = ay - by, dz = az - bz;
  return (uint32_t)(dx * dx) + (uint32_t)(dy * dy) + (uint32_t)(dz * dz);
}
// squared distance from a voxel to the nearest voxel of the cell [lo, lo + m)^3
__device__ __forceinline__ uint32_t cell_dist2(int px, int py, int pz, int cx, int cy, int cz, int m) {
  int d[3];
  const int p[3] = {px, py, pz}, c[3] = {cx, cy, cz};
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const int lo = c[a] * m, hi = lo + m - 1;
    d[a] = p[a] < lo ? lo - p[a] : (p[a] > hi ? p[a] - hi : 0);
  }
  return (uint32_t)(d[0] * d[0]) + (uint32_t)(d[1] * d[1]) + (uint32_t)(d[2] * d[2]);
}

// coordinates in block order: cs[i] = coords[perm[i]]
__global__ void geo_prep_kernel(const int32_t* __restrict__ coords, const int32_t* __restrict__ perm, int64_t N,
                                int4* __restrict__ cs) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = perm[i];
    cs[i] = make_int4(coords[3 * t], coords[3 * t + 1], coords[3 * t + 2], 0);
  }
}

template <int KL>
__global__ void __launch_bounds__(32 * kGeoWarps) geo_select_kernel(
    const int32_t* __restrict__ coords, const int32_t* __restrict__ cu_seqlens, int S, int64_t N,
    const int32_t* __restrict__ bptr, const int32_t* __restrict__ bcu, const int32_t* __restrict__ bkey,
    const int4* __restrict__ cs, int m, int topk, int hkv, int32_t* __restrict__ sel) {
  __shared__ int cand[kGeoWarps][kGeoCand];
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t t = (int64_t)blockIdx.x * kGeoWarps + w; t < N; t += (int64_t)gridDim.x * kGeoWarps) {
    const int s = find_segment(cu_seqlens, S, t);
    const int b0 = bcu[s], nb = bcu[s + 1] - b0;
    const int keff = min(topk, nb);
    const int px = coords[3 * t], py = coords[3 * t + 1], pz = coords[3 * t + 2];
    // 1. per-lane minimum of the upper bounds (distance to each block's first member)
    uint32_t umin = 0xffffffffu;
    for (int j = lane; j < nb; j += 32) {
      const int4 r = cs[bptr[b0 + j]];
      umin = min(umin, dist2(px, py, pz, r.x, r.y, r.z));
    }
    // 2. T = the keff-th smallest lane minimum (ties by lane): keff blocks lie within T
    int rank = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) {
      const uint32_t v2 = __shfl_sync(0xffffffffu, umin, o);
      rank += (v2 < umin || (v2 == umin && o < lane)) ? 1 : 0;
    }
    const unsigned own = __ballot_sync(0xffffffffu, rank == keff - 1);
    const uint32_t T = own ? __shfl_sync(0xffffffffu, umin, __ffs(own) - 1) : 0xffffffffu;
    // 3. candidates: blocks whose cell lies within T
    int n = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      bool c = false;
      if (j < nb) {
        const int* k = bkey + 3 * (int64_t)(b0 + j);
        c = cell_dist2(px, py, pz, k[0], k[1], k[2], m) <= T;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (c) {
        const int slot = n + __popc(bal & lt);
        if (slot < kGeoCand) cand[w][slot] = j;
      }
      n += __popc(bal);
    }
    __syncwarp();
    const bool all = n > kGeoCand;  // too many candidates: every block is one
    const int nc = all ? nb : n;
    // 4. exact distances; each lane keeps its KL smallest (distance, id) keys, ascending
    uint64_t lk[KL];
#pragma unroll
    for (int q = 0; q < KL; ++q) lk[q] = ~0ull;
    for (int c = lane; c < nc; c += 32) {
      const int j = all ? c : cand[w][c];
      uint32_t d = 0xffffffffu;
      const int q1 = bptr[b0 + j + 1];
      for (int q = bptr[b0 + j]; q < q1; ++q) {
        const int4 r = cs[q];
        d = min(d, dist2(px, py, pz, r.x, r.y, r.z));
      }
      const uint64_t key = ((uint64_t)d << 32) | (uint32_t)j;
      if (key < lk[KL - 1]) {
#pragma unroll
        for (int q = KL - 1; q >= 1; --q) {
          if (key < lk[q - 1])
            lk[q] = lk[q - 1];
          else if (key < lk[q])
            lk[q] = key;
        }
        if (key < lk[0]) lk[0] = key;
      }
    }
    __syncwarp();
    // 5. keff rounds of a warp-wide minimum over the list heads
    int chosen = 0x7fffffff;  // lane r keeps the r-th pick
    for (int r = 0; r < keff; ++r) {
      uint64_t v = lk[0];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t v2 = __shfl_xor_sync(0xffffffffu, v, o);
        v = v2 < v ? v2 : v;
      }
      if (lane == r) chosen = (int)(uint32_t)(v & 0xffffffffu);
      if (lk[0] == v) {
#pragma unroll
        for (int q = 0; q < KL - 1; ++q) lk[q] = lk[q + 1];
        lk[KL - 1] = ~0ull;
      }
    }
    // 6. ascending ids; the same selection for every KV group
    int pos = 0;
    for (int r = 0; r < keff; ++r) pos += __shfl_sync(0xffffffffu, chosen, r) < chosen ? 1 : 0;
    for (int g = 0; g < hkv; ++g) {
      int32_t* out = sel + (t * hkv + g) * topk;
      if (lane < keff) out[pos] = b0 + chosen;
      for (int i = keff + lane; i < topk; i += 32) out[i] = -1;
    }
  }
}

}  // namespace

size_t geo_ws_bytes(int64_t N) { return (size_t)N * sizeof(int4) + 256; }

cudaError_t geo_select(const int32_t* coords, const int32_t* cu_seqlens, int S, int64_t N, const ssa_partition* blk,
                       int m, int topk, int hkv, int32_t* sel, void* ws, cudaStream_t st) {
  int4* cs = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  const int64_t pg = (N + 255) / 256, sg = (N + kGeoWarps - 1) / kGeoWarps;
  const int prep_grid = (int)(pg < 148 * 32 ? pg : 148 * 32);
  SSA_LAUNCH("geo_prep_kernel", geo_prep_kernel, prep_grid > 0 ? prep_grid : 1, 256, 0, st, coords, blk->perm, N,
             cs);
  const int grid = (int)(sg < 148 * 16 ? sg : 148 * 16);
  if (topk <= 16)
    SSA_LAUNCH("geo_select_kernel", geo_select_kernel<16>, grid > 0 ? grid : 1, 32 * kGeoWarps, 0, st, coords,
               cu_seqlens, S, N, blk->ptr, blk->cu, blk->key, cs, m, topk, hkv, sel);
  else
    SSA_LAUNCH("geo_select_kernel", geo_select_kernel<32>, grid > 0 ? grid : 1, 32 * kGeoWarps, 0, st, coords,
               cu_seqlens, S, N, blk->ptr, blk->cu, blk->key, cs, m, topk, hkv, sel);
  return cudaGetLastError();
}

}  // namespace ssa
