// 3D-aware block routing (LSRM, shuwu5.cn/article/2502.html, "3D 感知空间块路由机制"),
// voxel-only case: every token selects the k blocks of its sequence whose tokens come
// nearest to it -- the shortest Euclidean distance between voxel centres -- with ties
// going to the lower block id.  Voxel centres differ by integer vectors, so squared
// distances are exact integers and the selection is exact.
//
// Pruning in two levels, both by the same argument: if keff distinct blocks are known
// to lie within T of a token, its keff-th smallest distance is <= T, so a block whose
// lower bound exceeds T is strictly farther than every selected block and can be
// dropped whatever the tie order.
//   1. One CTA per query block Q (its tokens share the m^3 cell).  For every block B of
//      the sequence, the farthest point of Q's cell from B's first member bounds
//      dist(q, B) from above for every q in Q; the keff-th smallest of the 256 per-thread
//      minima of that bound is T_Q.  The candidates of Q are the blocks whose cell lies
//      within T_Q of Q's cell.
//   2. One warp per token q of Q.  Over Q's candidates, the distance to each first member
//      bounds dist(q, B) from above; T_q is the keff-th smallest of the 32 per-lane
//      minima, and the blocks whose cell lies within T_q of q get their exact distance
//      (every member scanned).  The keff smallest (distance, id) keys are kept in
//      per-lane sorted lists and merged across the warp.
#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

constexpr int kGeoThreads = 256;
constexpr int kGeoWarps = kGeoThreads / 32;
constexpr int kGeoBlockCand = 4096;  // candidate blocks of a query block held in shared memory
constexpr int kGeoCand = 512;        // candidate blocks of one token held in shared memory

// squared gap along one axis between the integer ranges [a0, a1] and [b0, b1]
__device__ __forceinline__ uint32_t gap2(int a0, int a1, int b0, int b1) {
  const int g = b0 > a1 ? b0 - a1 : (a0 > b1 ? a0 - b1 : 0);
  return (uint32_t)(g * g);
}
// squared distance from p to the farthest point of [a0, a1] along one axis
__device__ __forceinline__ uint32_t far2(int a0, int a1, int p) {
  const int g = max(p - a0, a1 - p);
  return (uint32_t)(g * g);
}
__device__ __forceinline__ uint32_t dist2(int4 a, int4 b) {
  const int dx = a.x - b.x, dy = a.y - b.y, dz = a.z - b.z;
  return (uint32_t)(dx * dx) + (uint32_t)(dy * dy) + (uint32_t)(dz * dz);
}

// Block-order tables: cs[i] = (x, y, z, token) of the i-th token in block order;
// brep[b] = (first member's x, y, z, ptr[b]); bbox[b] = (cell x, y, z, ptr[b + 1]).
__global__ void geo_prep_kernel(const int32_t* __restrict__ coords, const int32_t* __restrict__ perm,
                                const int32_t* __restrict__ bptr, const int32_t* __restrict__ bkey, int64_t N,
                                int64_t B, int4* __restrict__ cs, int4* __restrict__ brep, int4* __restrict__ bbox) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += stride) {
    const int32_t t = perm[i];
    cs[i] = make_int4(coords[3 * (int64_t)t], coords[3 * (int64_t)t + 1], coords[3 * (int64_t)t + 2], t);
  }
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < B; b += stride) {
    const int32_t p0 = bptr[b], p1 = bptr[b + 1];
    const int32_t t = perm[p0];
    brep[b] = make_int4(coords[3 * (int64_t)t], coords[3 * (int64_t)t + 1], coords[3 * (int64_t)t + 2], p0);
    bbox[b] = make_int4(bkey[3 * b], bkey[3 * b + 1], bkey[3 * b + 2], p1);
  }
}

template <int KL>
__global__ void __launch_bounds__(kGeoThreads) geo_select_kernel(
    int S, int64_t B, const int32_t* __restrict__ bcu, const int4* __restrict__ cs, const int4* __restrict__ brep,
    const int4* __restrict__ bbox, int m, int topk, int hkv, int32_t* __restrict__ sel) {
  __shared__ int qcand[kGeoBlockCand];
  __shared__ int tcand[kGeoWarps][kGeoCand];
  __shared__ uint32_t tmin[kGeoThreads];
  __shared__ uint32_t s_T;
  __shared__ int s_n;
  const int tid = threadIdx.x, w = tid / 32, lane = tid % 32;
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t qb = blockIdx.x; qb < B; qb += gridDim.x) {
    const int s = find_segment(bcu, S, qb);
    const int b0 = bcu[s], nb = bcu[s + 1] - b0;
    const int keff = min(topk, nb);
    const int4 qbox = bbox[qb];
    const int qx0 = qbox.x * m, qy0 = qbox.y * m, qz0 = qbox.z * m;
    const int qx1 = qx0 + m - 1, qy1 = qy0 + m - 1, qz1 = qz0 + m - 1;
    // 1a. per-thread minimum over the sequence's blocks of the upper bound for the cell
    uint32_t umin = 0xffffffffu;
    for (int j = tid; j < nb; j += kGeoThreads) {
      const int4 r = brep[b0 + j];
      umin = min(umin, far2(qx0, qx1, r.x) + far2(qy0, qy1, r.y) + far2(qz0, qz1, r.z));
    }
    tmin[tid] = umin;
    if (tid == 0) s_n = 0;
    __syncthreads();
    // 1b. T_Q = the keff-th smallest of the per-thread minima (ties by thread index)
    {
      int rank = 0;
      for (int o = 0; o < kGeoThreads; ++o) {
        const uint32_t v2 = tmin[o];
        rank += (v2 < umin || (v2 == umin && o < tid)) ? 1 : 0;
      }
      if (rank == keff - 1) s_T = umin;
    }
    __syncthreads();
    const uint32_t TQ = s_T;
    // 1c. candidates of the query block: blocks whose cell lies within T_Q of Q's cell
    for (int j0 = 0; j0 < nb; j0 += kGeoThreads) {
      const int j = j0 + tid;
      bool c = false;
      if (j < nb) {
        const int4 k = bbox[b0 + j];
        const int x0 = k.x * m, y0 = k.y * m, z0 = k.z * m;
        c = gap2(qx0, qx1, x0, x0 + m - 1) + gap2(qy0, qy1, y0, y0 + m - 1) + gap2(qz0, qz1, z0, z0 + m - 1) <= TQ;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      int base = 0;
      if (lane == 0 && bal) base = atomicAdd(&s_n, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (c) {
        const int slot = base + __popc(bal & lt);
        if (slot < kGeoBlockCand) qcand[slot] = j;
      }
    }
    __syncthreads();
    const bool qall = s_n > kGeoBlockCand;  // too many candidates: every block is one
    const int nq = qall ? nb : s_n;
    // 2. one warp per token of the query block
    const int4 qr = brep[qb];
    for (int i = qr.w + w; i < qbox.w; i += kGeoWarps) {
      const int4 p = cs[i];
      // 2a. T_q from the per-lane minima of the distances to the candidates' first members
      uint32_t lmin = 0xffffffffu;
      for (int c = lane; c < nq; c += 32) lmin = min(lmin, dist2(p, brep[b0 + (qall ? c : qcand[c])]));
      int rank = 0;
#pragma unroll
      for (int o = 0; o < 32; ++o) {
        const uint32_t v2 = __shfl_sync(0xffffffffu, lmin, o);
        rank += (v2 < lmin || (v2 == lmin && o < lane)) ? 1 : 0;
      }
      const unsigned own = __ballot_sync(0xffffffffu, rank == keff - 1);
      const uint32_t T = own ? __shfl_sync(0xffffffffu, lmin, __ffs(own) - 1) : 0xffffffffu;
      // 2b. the token's candidates: blocks whose cell lies within T of the token
      int n = 0;
      for (int c0 = 0; c0 < nq; c0 += 32) {
        const int c = c0 + lane;
        int j = 0;
        bool keep = false;
        if (c < nq) {
          j = qall ? c : qcand[c];
          const int4 k = bbox[b0 + j];
          const int x0 = k.x * m, y0 = k.y * m, z0 = k.z * m;
          keep = gap2(p.x, p.x, x0, x0 + m - 1) + gap2(p.y, p.y, y0, y0 + m - 1) + gap2(p.z, p.z, z0, z0 + m - 1) <= T;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (keep) {
          const int slot = n + __popc(bal & lt);
          if (slot < kGeoCand) tcand[w][slot] = j;
        }
        n += __popc(bal);
      }
      __syncwarp();
      const bool tall = n > kGeoCand;  // too many: every candidate of the query block is one
      const int nt = tall ? nq : n;
      // 2c. exact distances; each lane keeps its KL smallest (distance, id) keys, ascending
      uint64_t lk[KL];
#pragma unroll
      for (int q = 0; q < KL; ++q) lk[q] = ~0ull;
      for (int c = lane; c < nt; c += 32) {
        const int j = tall ? (qall ? c : qcand[c]) : tcand[w][c];
        const int q0 = brep[b0 + j].w, q1 = bbox[b0 + j].w;
        uint32_t d = 0xffffffffu;
        for (int q = q0; q < q1; ++q) d = min(d, dist2(p, cs[q]));
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
      // 2d. keff rounds of a warp-wide minimum over the list heads
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
      // 2e. ascending ids; the same selection for every KV group
      int pos = 0;
      for (int r = 0; r < keff; ++r) pos += __shfl_sync(0xffffffffu, chosen, r) < chosen ? 1 : 0;
      for (int g = 0; g < hkv; ++g) {
        int32_t* out = sel + ((int64_t)p.w * hkv + g) * topk;
        if (lane < keff) out[pos] = b0 + chosen;
        for (int x = keff + lane; x < topk; x += 32) out[x] = -1;
      }
    }
    __syncthreads();  // qcand, tmin and s_n are reused by the next query block
  }
}

}  // namespace

size_t geo_ws_bytes(int64_t N) { return (size_t)N * 3 * sizeof(int4) + 256; }

cudaError_t geo_select(const int32_t* coords, const int32_t* cu_seqlens, int S, int64_t N, const ssa_partition* blk,
                       int m, int topk, int hkv, int32_t* sel, void* ws, cudaStream_t st) {
  (void)cu_seqlens;  // the block partition carries the sequences (blk->cu)
  const int64_t B = blk->count;
  int4* cs = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  int4* brep = cs + N;
  int4* bbox = brep + B;
  const int64_t pg = (N + 255) / 256;
  const int prep_grid = (int)(pg < 148 * 32 ? pg : 148 * 32);
  SSA_LAUNCH("geo_prep_kernel", geo_prep_kernel, prep_grid > 0 ? prep_grid : 1, 256, 0, st, coords, blk->perm,
             blk->ptr, blk->key, N, B, cs, brep, bbox);
  const int grid = (int)(B < 148 * 8 ? B : 148 * 8);
  if (topk <= 16)
    SSA_LAUNCH("geo_select_kernel", geo_select_kernel<16>, grid, kGeoThreads, 0, st, S, B, blk->cu, cs, brep, bbox, m,
               topk, hkv, sel);
  else
    SSA_LAUNCH("geo_select_kernel", geo_select_kernel<32>, grid, kGeoThreads, 0, st, S, B, blk->cu, cs, brep, bbox, m,
               topk, hkv, sel);
  return cudaGetLastError();
}

}  // namespace ssa
