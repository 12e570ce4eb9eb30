// Compressed branch of SSA on the tcgen05 tensor cores (bf16 inputs, fp32
// accumulation in TMEM), head dim 64.
//
// Direct3D-S2 (hyper.ai, "方法"): every query attends to all compressed blocks
// of its sequence; the top-k blocks by that attention score are selected.  The
// selection score of a block is its softmax probability summed over the query
// heads of a GQA group (LSRM, shuwu5.cn, "阶段一").
//
// A row tile is 128 query rows = (128/G tokens) x (G heads of one KV group),
// loaded by one 3D TMA box from Q [N, Hq, 64].  A key tile is a run of compressed
// blocks of Kc/Vc [Hkv, B, 64] (2D TMA, 128-byte swizzle): 96 in the output pass,
// 128 in the selection pass and the dK/dV kernel, 64 in the dQ kernel.
//
//   output pass (cmp_fa_tc):     flash attention, thread = row: S = Q Kc^T
//                                (double-buffered), online softmax, P (one bf16 per
//                                block) back into TMEM as the operand of O += P Vc
//                                -> o_cmp and lse.
//   selection pass (cmp_sel_tc): S^T = Kc Q^T, thread = block: p = exp2(s - lse)
//                                with the final lse, summed over the G heads of a
//                                token; a warpgroup picks each token's top-k.
//   backward (cmp_bwd_dq_tc, cmp_bwd_dkv_tc): dQ by rows (bf16), dKc / dVc by
//                                blocks (fp16 operands, from to_f16_kernel).
//
// Roles per CTA: compute warps (thread i <-> TMEM lane i), one warp issuing TMA
// loads, one issuing tcgen05.mma.  Every wait is bounded; on a timeout the kernel
// records kStatusTimeout, drains what it issued (bounded) and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tc_host.cuh"

namespace ssa {
namespace {

using namespace tc;
using namespace tch;

constexpr int kBN = 128;             // compressed blocks per key tile
constexpr int kTile = 128 * 128;     // bytes of a 128 x 64 bf16 tile

struct TileInfo {
  int g, s, t0, t_end, b0, nb;
};

__device__ __forceinline__ TileInfo tile_info(int it, int ntiles, const int32_t* tpre, int S, const int32_t* cu,
                                              const int32_t* bcu, int G) {
  TileInfo ti;
  ti.g = it / ntiles;
  const int tile = it % ntiles;
  ti.s = find_segment(tpre, S, tile);
  ti.t0 = cu[ti.s] + (tile - tpre[ti.s]) * (kRows / G);
  ti.t_end = cu[ti.s + 1];
  ti.b0 = bcu[ti.s];
  ti.nb = bcu[ti.s + 1] - ti.b0;
  return ti;
}

__device__ __forceinline__ void record_timeout(int* status, int* abort_flag) {
  atomicOr(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(abort_flag) = 1;
}

__device__ __forceinline__ bool aborted(const int* abort_flag) {
  return *reinterpret_cast<const volatile int*>(abort_flag) != 0;
}

// ---------------------------------------------------------------------------
// top-k selection (the selection pass below runs it in a warpgroup of its own)
// ---------------------------------------------------------------------------
constexpr int kTopkMax = 32;
constexpr int kCandMax = 128;  // top-k candidates per token kept for exact ranking
// selection pass: warpgroups of compute warps (thread = block), each owning
// kSelRowsPerWg of a row tile's 128 query rows, handled 32 at a time
constexpr int kComputeWarps = 8;
constexpr int kSelRowsPerWg = kRows / (kComputeWarps / 4);
// a warpgroup picks the top-k of the previous row tile while the compute warps work
// on the next one (the score scratch is double-buffered)
constexpr int kOutTopkWarps = 4;
constexpr int kOutTmaWarp = kComputeWarps + kOutTopkWarps;
constexpr int kOutMmaWarp = kOutTmaWarp + 1;
constexpr int kOutThreadsTk = 32 * (kOutMmaWarp + 1);

// (v, id) ranks above (v2, id2): higher score, or equal score and lower id.
__device__ __forceinline__ bool beats(float v, int id, float v2, int id2) { return v > v2 || (v == v2 && id < id2); }

// Sync of the 4 compute warps through an mbarrier (bounded wait, unlike bar.sync).
__device__ __forceinline__ bool cw_sync(uint64_t* bar, uint32_t& phase) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait_warp(bar, phase & 1);
  ++phase;
  return ok;
}

// Top-k of imp[0..nb) (scores of the sequence's blocks for one token) by one
// warp.  Each lane keeps a sorted list of its KL best entries in registers (one
// coalesced pass over the scores), then k rounds of a warp-wide arg-max over the
// list heads pick the winners.  Writes b0 + local id of the picks, ascending,
// padded with -1, to out[0..topk).  Requires topk <= KL.
template <int KL>
__device__ void warp_topk(const float* imp, int nb, int topk, int b0, int32_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int keff = min(topk, nb);
  float lv[KL];
  int li[KL];
#pragma unroll
  for (int k = 0; k < KL; ++k) {
    lv[k] = -CUDART_INF_F;
    li[k] = 0x7fffffff;
  }
  // imp is 16-byte aligned; each lane reads 4 consecutive scores per float4, 4 float4 in flight
  for (int base = 0; base < nb; base += 512) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i0 = base + u * 128 + lane * 4;
      if (i0 + 3 < nb) {
        v[u] = *reinterpret_cast<const float4*>(imp + i0);
      } else {
        v[u].x = i0 + 0 < nb ? imp[i0 + 0] : -CUDART_INF_F;
        v[u].y = i0 + 1 < nb ? imp[i0 + 1] : -CUDART_INF_F;
        v[u].z = i0 + 2 < nb ? imp[i0 + 2] : -CUDART_INF_F;
        v[u].w = -CUDART_INF_F;
        if (i0 + 3 < nb) v[u].w = imp[i0 + 3];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = base + u * 128 + lane * 4 + e;
        const float x = e == 0 ? v[u].x : e == 1 ? v[u].y : e == 2 ? v[u].z : v[u].w;
        if (i >= nb || !beats(x, i, lv[KL - 1], li[KL - 1])) continue;
#pragma unroll
        for (int k = KL - 1; k >= 1; --k) {
          const bool above_prev = beats(x, i, lv[k - 1], li[k - 1]);
          const bool above_cur = beats(x, i, lv[k], li[k]);
          if (above_prev) {
            lv[k] = lv[k - 1];
            li[k] = li[k - 1];
          } else if (above_cur) {
            lv[k] = x;
            li[k] = i;
          }
        }
        if (beats(x, i, lv[0], li[0])) {
          lv[0] = x;
          li[0] = i;
        }
      }
    }
  }
  int chosen = 0x7fffffff;  // lane r keeps the r-th pick (r < keff)
  for (int r = 0; r < keff; ++r) {
    float v = lv[0];
    int id = li[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      const int id2 = __shfl_xor_sync(0xffffffffu, id, o);
      if (beats(v2, id2, v, id)) {
        v = v2;
        id = id2;
      }
    }
    if (lane == r) chosen = id;
    if (id == li[0]) {  // this lane owned the winner: pop its head
#pragma unroll
      for (int k = 0; k < KL - 1; ++k) {
        lv[k] = lv[k + 1];
        li[k] = li[k + 1];
      }
      lv[KL - 1] = -CUDART_INF_F;
      li[KL - 1] = 0x7fffffff;
    }
  }
  int rank = 0;  // ascending ids: rank of each pick among the picks
  for (int r = 0; r < keff; ++r) {
    const int other = __shfl_sync(0xffffffffu, chosen, r);
    if (other < chosen) ++rank;
  }
  if (lane < keff) out[rank] = b0 + chosen;
  for (int i = keff + lane; i < topk; i += 32) out[i] = -1;
}

// Fast exact top-k of imp[0..nb) by one warp (same result as warp_topk):
//  1. each lane's best entry (one pass of float4 loads);
//  2. tau = the keff-th best of the 32 lane bests -- at least keff entries rank
//     at or above tau, so every top-keff entry does;
//  3. entries ranking at or above tau (typically a few dozen) are collected in
//     shared memory and ranked exactly against each other.
// Falls back to warp_topk when more than kCandMax entries pass the threshold.
template <int KL>
__device__ void warp_topk_fast(const float* imp, int nb, int topk, int b0, int32_t* __restrict__ out,
                               float* cv, int* ci) {
  const int lane = threadIdx.x & 31;
  const int keff = min(topk, nb);
  // 1. lane best
  float bv = -CUDART_INF_F;
  int bi = 0x7fffffff;
  for (int base = 0; base < nb; base += 512) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i0 = base + u * 128 + lane * 4;
      if (i0 + 3 < nb) {
        v[u] = *reinterpret_cast<const float4*>(imp + i0);
      } else {
        v[u].x = i0 + 0 < nb ? imp[i0 + 0] : -CUDART_INF_F;
        v[u].y = i0 + 1 < nb ? imp[i0 + 1] : -CUDART_INF_F;
        v[u].z = i0 + 2 < nb ? imp[i0 + 2] : -CUDART_INF_F;
        v[u].w = -CUDART_INF_F;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i0 = base + u * 128 + lane * 4;
      if (i0 < nb && beats(v[u].x, i0, bv, bi)) { bv = v[u].x; bi = i0; }
      if (i0 + 1 < nb && beats(v[u].y, i0 + 1, bv, bi)) { bv = v[u].y; bi = i0 + 1; }
      if (i0 + 2 < nb && beats(v[u].z, i0 + 2, bv, bi)) { bv = v[u].z; bi = i0 + 2; }
      if (i0 + 3 < nb && beats(v[u].w, i0 + 3, bv, bi)) { bv = v[u].w; bi = i0 + 3; }
    }
  }
  // 2. rank of each lane best among the 32; tau = the one of rank keff-1
  int rank = 0;
#pragma unroll
  for (int o = 0; o < 32; ++o) {
    const float v2 = __shfl_sync(0xffffffffu, bv, o);
    const int i2 = __shfl_sync(0xffffffffu, bi, o);
    if (beats(v2, i2, bv, bi)) ++rank;
  }
  const unsigned own = __ballot_sync(0xffffffffu, rank == keff - 1);
  if (keff > 32 || own == 0u) {  // fewer than keff lanes hold entries: exact path
    warp_topk<KL>(imp, nb, topk, b0, out);
    return;
  }
  const int src = __ffs(own) - 1;
  const float tv = __shfl_sync(0xffffffffu, bv, src);
  const int ti = __shfl_sync(0xffffffffu, bi, src);
  // 3. collect entries at or above (tv, ti): 512 entries per round, 4 float4 loads per lane in flight
  int n = 0;
  bool overflow = false;
  for (int base = 0; base < nb && !overflow; base += 512) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i0 = base + u * 128 + lane * 4;
      if (i0 + 3 < nb) {
        v[u] = *reinterpret_cast<const float4*>(imp + i0);
      } else {
        v[u].x = i0 + 0 < nb ? imp[i0 + 0] : -CUDART_INF_F;
        v[u].y = i0 + 1 < nb ? imp[i0 + 1] : -CUDART_INF_F;
        v[u].z = i0 + 2 < nb ? imp[i0 + 2] : -CUDART_INF_F;
        v[u].w = -CUDART_INF_F;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i0 = base + u * 128 + lane * 4;
      const float xs[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      bool tk[4];
      int c = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i0 + e;
        tk[e] = i < nb && (xs[e] == tv ? i <= ti : xs[e] > tv);
        c += tk[e] ? 1 : 0;
      }
      // exclusive prefix of c over the lanes
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int slot = n + incl - c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (tk[e]) {
          if (slot < kCandMax) {
            cv[slot] = xs[e];
            ci[slot] = i0 + e;
          }
          ++slot;
        }
      }
      n += __shfl_sync(0xffffffffu, incl, 31);
    }
    overflow = n > kCandMax;
  }
  if (overflow) {
    __syncwarp();
    warp_topk<KL>(imp, nb, topk, b0, out);
    return;
  }
  __syncwarp();
  // exact ranks among the candidates; picks are those with rank < keff
  int picked_id[kCandMax / 32];
  bool picked[kCandMax / 32];
#pragma unroll
  for (int u = 0; u < kCandMax / 32; ++u) {
    const int c = u * 32 + lane;
    picked[u] = false;
    picked_id[u] = 0x7fffffff;
    if (c < n) {
      const float x = cv[c];
      const int id = ci[c];
      int r = 0;
      for (int j = 0; j < n; ++j) r += beats(cv[j], ci[j], x, id) ? 1 : 0;
      picked[u] = r < keff;
      picked_id[u] = id;
    }
  }
  __syncwarp();
  // write picks in ascending id order: position = number of picks with a lower id
#pragma unroll
  for (int u = 0; u < kCandMax / 32; ++u) {
    const int c = u * 32 + lane;
    if (c < n) ci[c] = picked[u] ? picked_id[u] : 0x7fffffff;
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < kCandMax / 32; ++u) {
    if (picked[u]) {
      int pos = 0;
      for (int j = 0; j < n; ++j) pos += ci[j] < picked_id[u] ? 1 : 0;
      out[pos] = b0 + picked_id[u];
    }
  }
  for (int i = keff + lane; i < topk; i += 32) out[i] = -1;
  __syncwarp();
}


// Exact top-k of imp[0..nb) (the same result as warp_topk) from the scores and their
// group maxima gm[0..ceil(nb/32)) (gm[i] = max of imp[32 i .. 32 i + 31]; scores are
// sums of probabilities, never negative):
//  1. each lane's best group maximum (lane l holds groups l, l + 32, ...);
//  2. tau = the keff-th best of the 32 lane bests: they are scores of keff distinct
//     blocks, so every top-keff score is >= tau;
//  3. only groups whose maximum is >= tau can hold such scores: their members >= tau
//     are collected (32 loads of a group in one coalesced access) and ranked exactly.
// Falls back to warp_topk_fast over all scores for sequences of more than 4096 blocks,
// when fewer than keff lanes hold a group, or when more than kCandMax scores reach tau.
constexpr int kGrpPerLane = 4;
constexpr int kGrpBatch = 8;  // candidate groups loaded together
template <int KL>
__device__ void warp_topk_groups(const float* imp, const float* gm, int nb, int topk, int b0,
                                 int32_t* __restrict__ out, float* cv, int* ci, int* cg) {
  const int lane = threadIdx.x & 31;
  const int keff = min(topk, nb);
  const int ng = (nb + 31) / 32;
  if (keff > 32 || ng > 32 * kGrpPerLane) {
    warp_topk_fast<KL>(imp, nb, topk, b0, out, cv, ci);
    return;
  }
  // 1. lane bests over the group maxima (absent groups read as -1, below every score)
  float gv[kGrpPerLane];
  float bv = -1.f;
  int bi = 0x7fffffff;
#pragma unroll
  for (int u = 0; u < kGrpPerLane; ++u) {
    const int i = lane + 32 * u;
    gv[u] = i < ng ? gm[i] : -1.f;
    if (gv[u] > bv) {
      bv = gv[u];
      bi = i;
    }
  }
  // 2. tau = the lane best of rank keff - 1 among the 32
  int rank = 0;
#pragma unroll
  for (int o = 0; o < 32; ++o) {
    const float v2 = __shfl_sync(0xffffffffu, bv, o);
    const int i2 = __shfl_sync(0xffffffffu, bi, o);
    if (beats(v2, i2, bv, bi)) ++rank;
  }
  const unsigned own = __ballot_sync(0xffffffffu, rank == keff - 1 && bv >= 0.f);
  if (own == 0u) {  // fewer than keff lanes hold a group
    warp_topk_fast<KL>(imp, nb, topk, b0, out, cv, ci);
    return;
  }
  const float tv = __shfl_sync(0xffffffffu, bv, __ffs(own) - 1);
  // 3. candidate groups (maximum >= tau), compacted in index order
  const unsigned lt = (1u << lane) - 1u;
  int ncg = 0;
#pragma unroll
  for (int u = 0; u < kGrpPerLane; ++u) {
    const bool c = gv[u] >= tv;
    const unsigned m = __ballot_sync(0xffffffffu, c);
    if (c) cg[ncg + __popc(m & lt)] = lane + 32 * u;
    ncg += __popc(m);
  }
  __syncwarp();
  // their members >= tau, in index order
  int n = 0;
  for (int c0 = 0; c0 < ncg; c0 += kGrpBatch) {
    float x[kGrpBatch];
    int id[kGrpBatch];
#pragma unroll
    for (int k = 0; k < kGrpBatch; ++k) {
      id[k] = c0 + k < ncg ? 32 * cg[c0 + k] + lane : nb;
      x[k] = id[k] < nb ? imp[id[k]] : -1.f;
    }
#pragma unroll
    for (int k = 0; k < kGrpBatch; ++k) {
      const bool keep = id[k] < nb && x[k] >= tv;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int slot = n + __popc(m & lt);
        if (slot < kCandMax) {
          cv[slot] = x[k];
          ci[slot] = id[k];
        }
      }
      n += __popc(m);
    }
  }
  if (n > kCandMax) {
    __syncwarp();
    warp_topk_fast<KL>(imp, nb, topk, b0, out, cv, ci);
    return;
  }
  __syncwarp();
  // exact ranks among the candidates; picks are those with rank < keff
  int picked_id[kCandMax / 32];
  bool picked[kCandMax / 32];
#pragma unroll
  for (int u = 0; u < kCandMax / 32; ++u) {
    const int c = u * 32 + lane;
    picked[u] = false;
    picked_id[u] = 0x7fffffff;
    if (c < n) {
      const float xv = cv[c];
      const int xi = ci[c];
      int r = 0;
      for (int j = 0; j < n; ++j) r += beats(cv[j], ci[j], xv, xi) ? 1 : 0;
      picked[u] = r < keff;
      picked_id[u] = xi;
    }
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < kCandMax / 32; ++u) {
    const int c = u * 32 + lane;
    if (c < n) ci[c] = picked[u] ? picked_id[u] : 0x7fffffff;
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < kCandMax / 32; ++u) {
    if (picked[u]) {
      int pos = 0;
      for (int j = 0; j < n; ++j) pos += ci[j] < picked_id[u] ? 1 : 0;
      out[pos] = b0 + picked_id[u];
    }
  }
  for (int i = keff + lane; i < topk; i += 32) out[i] = -1;
  __syncwarp();
}

// ---------------------------------------------------------------------------
// output pass (thread = row): flash attention of every query row over all compressed
// blocks of its sequence, producing o_cmp and lse.  A work unit is a pair of 128-row
// Q tiles (sides A, B) of the same (sequence, group), so each Kc / Vc tile of kFaBN
// blocks is loaded once for 256 rows.  One warpgroup per side keeps its rows' running
// max m and sum l (log2 domain, scale folded in).  Per side, S is double-buffered in
// TMEM (two kFaBN-column buffers, then O: 2 x 96 + 64 = 256 columns, 512 for both
// sides): the S of step g + 2 is issued into buffer g % 2 right after P V(g) has been
// issued there (the MMA stream of one thread executes in order), so the tensor pipe
// computes it while the softmax warps work on step g + 1.  p = 2^(s qs2 - m) goes back
// into its S buffer as one bf16 per block (blocks 16c .. 16c+15 in columns 8c .. 8c+7)
// and feeds O += P Vc as the TMEM operand.  A single bf16 is enough here: each row's
// o_cmp is one sum over the blocks of its own sequence, and the rounding (2^-9 relative
// per probability, unbiased) moves it by about 1e-4 at the benchmark's sizes, against
// the sums over millions of rows in the key gradients.  O (TMEM) is rescaled only when
// a row's max grows by more than 2^8 since it was last fixed, so p stays below 2^8
// otherwise.  All exponentials run on the MUFU: with S double-buffered the softmax
// warps are busy enough that moving a share to the FMA pipe (ex2_poly2) costs more
// issue slots than it frees MUFU cycles.  Steps are counted per side across the
// CTA's pairs (g), which sets the buffer (g % 2) and the barrier phases.
// ---------------------------------------------------------------------------
constexpr int kFaBN = 96;                    // compressed blocks per key tile
constexpr int kFaStages = 4;                 // Kc / Vc ring depth (steps g, g + 1, g + 2 in use)
constexpr int kFaSoftmaxWarps = 8;           // warps 0-3: side A, 4-7: side B
constexpr int kFaTmaWarp = kFaSoftmaxWarps;
constexpr int kFaMmaWarp = kFaSoftmaxWarps + 1;
constexpr int kFaThreads = 32 * (kFaSoftmaxWarps + 2);
constexpr int kFaKvTile = kFaBN * 128;       // bytes of a [kFaBN, 64] bf16 tile
constexpr int kFaSideCols = 2 * kFaBN + 64;  // TMEM per side: S buffers 0 and 1, O
constexpr int kFaPolyCols = 0;               // blocks of a key tile whose exponentials use the FMA pipe
                                             // (at 131072 tokens: 0 -> 4.24 ms, 16 -> 4.42, 24 -> 4.49, 48 -> 4.76)
constexpr float kFaRescaleLog2 = 8.f;
static_assert(2 * kFaSideCols <= 512 && kFaBN % 32 == 0, "TMEM");

struct FaSmem {
  uint8_t q[2][2][kTile];  // [buffer][side A / B]
  uint8_t kc[kFaStages][kFaKvTile];
  uint8_t vc[kFaStages][kFaKvTile];
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kFaStages], kv_empty[kFaStages];
  uint64_t s_full[2][2], p_full[2][2];  // [side][S buffer]
  uint64_t pv_done[2], o_full[2], o_empty[2];
  uint64_t mma_done;
  uint32_t tmem;
  int abort_flag;
};

struct PairInfo {
  int g, s, t0, t_end, b0, nb;  // t0: first token of side A; side B starts 128/G tokens later
};

__device__ __forceinline__ PairInfo pair_info(int it, int npairs, const int32_t* ppre, int S, const int32_t* cu,
                                              const int32_t* bcu, int G) {
  PairInfo pi;
  pi.g = it / npairs;
  const int pr = it % npairs;
  pi.s = find_segment(ppre, S, pr);
  pi.t0 = cu[pi.s] + (pr - ppre[pi.s]) * (2 * kRows / G);
  pi.t_end = cu[pi.s + 1];
  pi.b0 = bcu[pi.s];
  pi.nb = bcu[pi.s + 1] - pi.b0;
  return pi;
}

template <int G>
__global__ void __launch_bounds__(kFaThreads, 1) cmp_fa_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kcmap,
    const __grid_constant__ CUtensorMap vcmap, const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu,
    const int32_t* __restrict__ ppre, int S, int64_t N, int hq, int hkv, int btot, float qs2,
    float* __restrict__ o_out, float* __restrict__ lse_out, int* status) {
  constexpr int TPT = kRows / G;  // tokens per Q tile
  extern __shared__ uint8_t smem_raw[];
  FaSmem& sm = *reinterpret_cast<FaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int npairs = ppre[S];
  const int total = npairs * hkv;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.pv_done[i], 1);
      mbar_init(&sm.o_full[i], 1);
      mbar_init(&sm.o_empty[i], 4);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[i][b], 1);
        mbar_init(&sm.p_full[i][b], 4);
      }
    }
    for (int i = 0; i < kFaStages; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;

  if (warp == kFaTmaWarp) {
    // ---------------- TMA producer: the pair's two Q tiles; (Kc, Vc) per key tile
    if (lane == 0) {
      prefetch_tmap(&qmap);
      prefetch_tmap(&kcmap);
      prefetch_tmap(&vcmap);
      uint32_t kv_count = 0, q_count = 0;
      int last_par[kFaStages];
      for (int i = 0; i < kFaStages; ++i) last_par[i] = -1;
      for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
        const PairInfo pi = pair_info(it, npairs, ppre, S, cu, bcu, G);
        const int qb = q_count % 2;
        if (!mbar_wait(&sm.q_empty[qb], ((q_count / 2) & 1) ^ 1)) { record_timeout(status, &sm.abort_flag); break; }
        mbar_expect_tx(&sm.q_full[qb], 2 * kTile);
        tma_load_3d(sm.q[qb][0], &qmap, &sm.q_full[qb], 0, pi.g * G, pi.t0);
        // side B: rows past the last token are never used; keep its box inside the tensor
        const int tb = pi.t0 + TPT < N ? pi.t0 + TPT : pi.t0;
        tma_load_3d(sm.q[qb][1], &qmap, &sm.q_full[qb], 0, pi.g * G, tb);
        ++q_count;
        const int nbt = (pi.nb + kFaBN - 1) / kFaBN;
        bool ok = true;
        for (int j = 0; j < nbt; ++j) {
          const int st = kv_count % kFaStages;
          const uint32_t ph = (kv_count / kFaStages) & 1;
          if (!mbar_wait(&sm.kv_empty[st], ph ^ 1)) { record_timeout(status, &sm.abort_flag); ok = false; break; }
          mbar_expect_tx(&sm.kv_full[st], 2 * kFaKvTile);
          const int row = pi.g * btot + pi.b0 + j * kFaBN;
          tma_load_2d(sm.kc[st], &kcmap, &sm.kv_full[st], 0, row);
          tma_load_2d(sm.vc[st], &vcmap, &sm.kv_full[st], 0, row);
          last_par[st] = (int)ph;
          ++kv_count;
        }
        if (!ok) break;
      }
      for (int i = 0; i < kFaStages; ++i)
        if (last_par[i] >= 0) mbar_wait(&sm.kv_full[i], (uint32_t)last_par[i]);
    }
  } else if (warp == kFaMmaWarp) {
    // ---------------- MMA issuer: S(0), S(1) of both sides; then per key tile j and
    // side: O += P(j) Vc(j) once P(j) is in TMEM, then S(j + 2) into P(j)'s buffer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(kRows, kFaBN);            // S[rows, blocks] = Q Kc^T
      const uint32_t id_o = idesc_bf16(kRows, 64, false, true);  // O[rows, 64] += P[rows, blocks] Vc
      uint32_t kv_count = 0, q_count = 0, g = 0, o_cnt = 0;  // g: steps of either side so far
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !aborted(&sm.abort_flag); it += gridDim.x) {
        const PairInfo pi = pair_info(it, npairs, ppre, S, cu, bcu, G);
        const int qb = q_count % 2;
        if (!mbar_wait(&sm.q_full[qb], (q_count / 2) & 1)) { ok = false; break; }
        ++q_count;
        const int nbt = (pi.nb + kFaBN - 1) / kFaBN;
        // S(j) of both sides from stage kv_count + j into buffer (g + j) % 2
        auto issue_s = [&](int j) -> bool {
          const uint32_t kv_j = kv_count + j;
          const int st = kv_j % kFaStages;
          if (!mbar_wait(&sm.kv_full[st], (kv_j / kFaStages) & 1)) return false;
          tc_fence_after();
          const int b = (g + j) & 1;
#pragma unroll
          for (int side = 0; side < 2; ++side) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16_ss(tmem + side * kFaSideCols + b * kFaBN, sdesc_kmajor_sw128(sm.q[qb][side], 32 * k),
                          sdesc_kmajor_sw128(sm.kc[st], 32 * k), id_s, k > 0);
            mma_commit(&sm.s_full[side][b]);
          }
          return true;
        };
        if (nbt > 0 && !issue_s(0)) { ok = false; break; }
        if (nbt > 1 && !issue_s(1)) { ok = false; break; }
        for (int j = 0; j < nbt && ok; ++j) {
          const uint32_t gj = g + j;
          const int b = gj & 1;
          const int st = (kv_count + j) % kFaStages;
#pragma unroll
          for (int side = 0; side < 2; ++side) {
            if (!mbar_wait(&sm.p_full[side][b], (gj >> 1) & 1) ||
                (j == 0 && !mbar_wait(&sm.o_empty[side], (o_cnt & 1) ^ 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tp = tmem + side * kFaSideCols + b * kFaBN, to = tmem + side * kFaSideCols + 2 * kFaBN;
#pragma unroll
            for (int k = 0; k < kFaBN / 16; ++k)
              mma_bf16_ts(to, tp + 8 * k, sdesc_mnmajor_sw128(sm.vc[st], 2048 * k, kFaKvTile), id_o, j > 0 || k > 0);
            mma_commit(&sm.pv_done[side]);
          }
          if (!ok) break;
          mma_commit(&sm.kv_empty[st]);
          if (j + 2 < nbt && !issue_s(j + 2)) { ok = false; break; }
        }
        if (!ok) break;
        kv_count += nbt;
        g += nbt;
        for (int side = 0; side < 2; ++side) mma_commit(&sm.o_full[side]);
        ++o_cnt;
        mma_commit(&sm.q_empty[qb]);
      }
      if (!ok) record_timeout(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ---------------- softmax warpgroups: thread = row of this side's Q tile
    const int side = warp / 4;
    const int r = threadIdx.x % 128;
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tbase = tmem + side * kFaSideCols + lane_off, tm_o = tbase + 2 * kFaBN;
    const float2 qs = make_float2(qs2, qs2);
    uint32_t g = 0, o_cnt = 0;
    for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
      const PairInfo pi = pair_info(it, npairs, ppre, S, cu, bcu, G);
      const int64_t t = (int64_t)pi.t0 + side * TPT + r / G;
      const int h = pi.g * G + r % G;
      const bool valid = t < pi.t_end;
      const int nbt = (pi.nb + kFaBN - 1) / kFaBN;
      float m = -CUDART_INF_F, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nbt; ++j, ++g) {
        const int b = g & 1;
        if (!mbar_wait_warp(&sm.s_full[side][b], (g >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tm_s = tbase + b * kFaBN;
        float sv[kFaBN];
#pragma unroll
        for (int c = 0; c < kFaBN; c += 32) tmem_ld32(tm_s + c, sv + c);
        tmem_ld_wait();
        const int vcols = min(kFaBN, pi.nb - j * kFaBN);
        if (vcols < kFaBN) {  // ragged last key tile: blocks past the sequence get p = 0
#pragma unroll
          for (int c = 0; c < kFaBN; ++c) sv[c] = c < vcols ? sv[c] : -CUDART_INF_F;
        }
        // row max as 8 independent chains
        float mx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx[c] = sv[c];
#pragma unroll
        for (int c = 8; c < kFaBN; ++c) mx[c % 8] = fmaxf(mx[c % 8], sv[c]);
        const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * qs2;  // qs2 > 0
        float alpha = 1.f;
        bool resc = false;
        if (j == 0) {
          m = mt;
        } else if (mt > m + kFaRescaleLog2) {
          alpha = ex2(m - mt);
          m = mt;
          l *= alpha;
          resc = true;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // O holds the sum of the products of steps .. g-1: wait for the last one, then scale
          if (!mbar_wait_warp(&sm.pv_done[side], (g - 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float o[32];
            tmem_ld32(tm_o + 32 * hh, o);
            tmem_ld_wait();
            uint32_t u[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) u[c] = __float_as_uint(o[c] * alpha);
            tmem_st16(tm_o + 32 * hh, u);
            tmem_st16(tm_o + 32 * hh + 16, u + 16);
          }
        }
        const float2 nm = make_float2(-m, -m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int qq = 0; qq < kFaBN / 32; ++qq) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 x = ffma2(make_float2(sv[32 * qq + c], sv[32 * qq + c + 1]), qs, nm);
            const float2 p = 32 * qq + c < kFaPolyCols ? ex2_poly2(x) : ex2x2(x);
            acc[(c / 2) % 4] = fadd2(acc[(c / 2) % 4], p);
            pk[c / 2] = pack2(p);
          }
          tmem_st16(tm_s + 16 * qq, pk);
        }
        l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[side][b]);
      }
      if (!ok) {
        record_timeout(status, &sm.abort_flag);
        break;
      }
      // O of the pair: wait for the last product, normalise, write o_cmp and lse
      if (!mbar_wait_warp(&sm.o_full[side], o_cnt & 1)) { record_timeout(status, &sm.abort_flag); break; }
      ++o_cnt;
      tc_fence_after();
      float o[64];
      tmem_ld32(tm_o, o);
      tmem_ld32(tm_o + 32, o + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_empty[side]);
      if (valid) {
        const float inv = 1.f / l;
        float4* dst = reinterpret_cast<float4*>(o_out + (t * hq + h) * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
        lse_out[t * hq + h] = (m + log2f(l)) * kLn2;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// selection pass (transposed: thread = block): S^T = Kc Q^T in TMEM, double-
// buffered; p = 2^(s qs2 - lse log2 e) with the final lse of the output pass; the
// block's score for a token is the sum of its G heads' p, written to a per-CTA
// scratch together with the maximum of each group of 32 blocks (one warp-wide
// reduction); a warpgroup picks each token's top-k of the previous row tile from
// those (warp_topk_groups) while the compute warps work on the next one.  The
// exponentials stay on the MUFU (kSelPolyRows = 0): moving a share to the FMA pipe
// (ex2_poly2) measured slower here.
// ---------------------------------------------------------------------------
constexpr int kSelStages = 6;           // Kc ring depth (4.51 ms at 4, 4.38 at 6, at 131072 tokens)
constexpr int kSelPolyRows = 0;  // rows of a key tile whose exponentials use the FMA pipe (at 131072 tokens:
                                  // 0 -> 4.87 ms, a quarter -> 5.12, a half -> 5.46)

struct SelSmem {
  uint8_t q[2][kTile];
  uint8_t kc[kSelStages][kTile];
  __align__(16) float lse2[2][kRows];  // -lse log2(e) of the tile's rows, double-buffered by tile
  float candv[kOutTopkWarps][kCandMax];
  int candi[kOutTopkWarps][kCandMax];
  int candg[kOutTopkWarps][32 * kGrpPerLane];
  uint64_t q_full[2], q_empty[2], mma_done, cw, imp_full[2], imp_empty[2];
  uint64_t kc_full[kSelStages], kc_empty[kSelStages];
  uint64_t s_full[2], s_empty[2];
  uint32_t tmem;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(kOutThreadsTk, 1) cmp_sel_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kcmap,
    const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu, const int32_t* __restrict__ tpre, int S,
    int hq, int hkv, int btot, float qs2, const float* __restrict__ lse_in, int topk, int32_t* __restrict__ sel,
    float* __restrict__ imp_scratch, int64_t imp_stride, int64_t gm_stride, int* status) {
  constexpr int TPT = kRows / G;  // tokens per tile
  extern __shared__ uint8_t smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntiles = tpre[S];
  const int total = ntiles * hkv;
  // this CTA's scores, two buffers of [TPT tokens][imp_stride blocks], and their group
  // maxima, two buffers of [TPT tokens][gm_stride groups of 32 blocks]
  float* imp_cta = imp_scratch + (int64_t)blockIdx.x * 2 * TPT * (imp_stride + gm_stride);
  float* gm_cta = imp_cta + 2 * TPT * imp_stride;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.imp_full[i], kComputeWarps);
      mbar_init(&sm.imp_empty[i], kOutTopkWarps);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_empty[i], kComputeWarps);
    }
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.cw, kComputeWarps);
    for (int i = 0; i < kSelStages; ++i) {
      mbar_init(&sm.kc_full[i], 1);
      mbar_init(&sm.kc_empty[i], 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;  // S^T buffers at columns [0,128) and [128,256)

  if (warp == kOutTmaWarp) {
    // ---------------- TMA producer: Q per tile; Kc per key tile
    if (lane == 0) {
      prefetch_tmap(&qmap);
      prefetch_tmap(&kcmap);
      uint32_t kc_count = 0, q_count = 0;
      int last_par[kSelStages];
      for (int i = 0; i < kSelStages; ++i) last_par[i] = -1;
      for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
        const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
        const int qb = q_count % 2;
        if (!mbar_wait(&sm.q_empty[qb], ((q_count / 2) & 1) ^ 1)) { record_timeout(status, &sm.abort_flag); break; }
        mbar_expect_tx(&sm.q_full[qb], kTile);
        tma_load_3d(sm.q[qb], &qmap, &sm.q_full[qb], 0, ti.g * G, ti.t0);
        ++q_count;
        const int nbt = (ti.nb + kBN - 1) / kBN;
        bool ok = true;
        for (int j = 0; j < nbt; ++j) {
          const int st = kc_count % kSelStages;
          const uint32_t ph = (kc_count / kSelStages) & 1;
          if (!mbar_wait(&sm.kc_empty[st], ph ^ 1)) { record_timeout(status, &sm.abort_flag); ok = false; break; }
          mbar_expect_tx(&sm.kc_full[st], kTile);
          tma_load_2d(sm.kc[st], &kcmap, &sm.kc_full[st], 0, ti.g * btot + ti.b0 + j * kBN);
          last_par[st] = (int)ph;
          ++kc_count;
        }
        if (!ok) break;
      }
      for (int i = 0; i < kSelStages; ++i)
        if (last_par[i] >= 0) mbar_wait(&sm.kc_full[i], (uint32_t)last_par[i]);
    }
  } else if (warp == kOutMmaWarp) {
    // ---------------- MMA issuer: S^T(j) into buffer j % 2 as soon as the compute warps released it
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(kBN, kRows);  // S^T[blocks, rows] = Kc Q^T
      uint32_t kc_count = 0, q_count = 0, s_count = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !aborted(&sm.abort_flag); it += gridDim.x) {
        const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
        const int qb = q_count % 2;
        if (!mbar_wait(&sm.q_full[qb], (q_count / 2) & 1)) { ok = false; break; }
        ++q_count;
        const int nbt = (ti.nb + kBN - 1) / kBN;
        for (int j = 0; j < nbt; ++j) {
          const int st = kc_count % kSelStages;
          const int sb = s_count % 2;
          if (!mbar_wait(&sm.kc_full[st], (kc_count / kSelStages) & 1) ||
              !mbar_wait(&sm.s_empty[sb], ((s_count / 2) & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ss(tmem + sb * kBN, sdesc_kmajor_sw128(sm.kc[st], 32 * k), sdesc_kmajor_sw128(sm.q[qb], 32 * k),
                        id_s, k > 0);
          mma_commit(&sm.s_full[sb]);
          mma_commit(&sm.kc_empty[st]);
          ++kc_count;
          ++s_count;
        }
        if (!ok) break;
        mma_commit(&sm.q_empty[qb]);
      }
      if (!ok) record_timeout(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else if (warp < kComputeWarps) {
    // ---------------- compute warps: thread = block of the key tile; warpgroup wg handles
    // query rows [kSelRowsPerWg wg, +kSelRowsPerWg) of the tile, 32 at a time.
    constexpr int NH = kSelRowsPerWg / 32;
    const int b = threadIdx.x % 128;
    const int wg = warp / 4;
    const int r0 = kSelRowsPerWg * wg;
    uint32_t s_count = 0, cw_phase = 0, n_tile = 0;
    for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x, ++n_tile) {
      const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
      const int lb = n_tile & 1;
      if (wg == 0) {
        const int r = threadIdx.x;
        const int64_t t = min((int64_t)ti.t0 + r / G, (int64_t)ti.t_end - 1);
        sm.lse2[lb][r] = -lse_in[t * hq + ti.g * G + r % G] * kLog2e;  // -lse log2(e)
      }
      if (!cw_sync(&sm.cw, cw_phase)) { record_timeout(status, &sm.abort_flag); break; }
      // the top-k warps have released this tile's importance buffer
      if (!mbar_wait_warp(&sm.imp_empty[lb], ((n_tile >> 1) & 1) ^ 1)) { record_timeout(status, &sm.abort_flag); break; }
      float* imp_base = imp_cta + (int64_t)lb * TPT * imp_stride;
      float* gm_base = gm_cta + (int64_t)lb * TPT * gm_stride;
      const int nbt = (ti.nb + kBN - 1) / kBN;
      bool ok = true;
      const float2 qs = make_float2(qs2, qs2);
      for (int j = 0; j < nbt; ++j) {
        const int sb = s_count % 2;
        if (!mbar_wait_warp(&sm.s_full[sb], (s_count / 2) & 1)) { ok = false; break; }
        tc_fence_after();
        const int bidx = j * kBN + b;  // block index inside the sequence
        const bool bvalid = bidx < ti.nb;
        const uint32_t taddr = tmem + sb * kBN + ((uint32_t)((warp % 4) * 32) << 16) + r0;
        float p[NH][32];
        tmem_ld32(taddr, p[0]);
        tmem_ld_wait();
        ++s_count;
        const int grp = j * (kBN / 32) + (warp % 4);  // this warp's 32 blocks form one group
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          // the next 32 rows land while this half is processed
          if (hh > 0) {
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) asm volatile("" : "+f"(p[hh][i]));  // no use of p[hh] above the wait
          }
          if (hh == NH - 1) {  // every row of this S buffer is in registers: release it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_empty[sb]);
          }
          if (hh + 1 < NH) tmem_ld32(taddr + 32 * (hh + 1), p[hh + 1]);
          if (bvalid) {
#pragma unroll
            for (int r = 0; r < 32; r += 4) {
              const float4 l4 = *reinterpret_cast<const float4*>(&sm.lse2[lb][r0 + 32 * hh + r]);
              const float2 xa = ffma2(make_float2(p[hh][r], p[hh][r + 1]), qs, make_float2(l4.x, l4.y));
              const float2 xb = ffma2(make_float2(p[hh][r + 2], p[hh][r + 3]), qs, make_float2(l4.z, l4.w));
              const bool poly = 32 * hh + r < kSelPolyRows;
              const float2 pa = poly ? ex2_poly2(xa) : ex2x2(xa);
              const float2 pb = poly ? ex2_poly2(xb) : ex2x2(xb);
              p[hh][r] = pa.x;
              p[hh][r + 1] = pa.y;
              p[hh][r + 2] = pb.x;
              p[hh][r + 3] = pb.y;
            }
          }
          // selection score of this block for the pass's tokens: probability summed over the
          // group's heads; and the maximum over the warp's 32 blocks (scores are >= 0, so their
          // bit patterns order as unsigned integers; blocks past the sequence count as 0)
#pragma unroll
          for (int tl = 0; tl < 32 / G; ++tl) {
            float v = 0.f;
            if (bvalid) {
              float2 acc = make_float2(p[hh][tl * G], p[hh][tl * G + 1]);
#pragma unroll
              for (int h2 = 2; h2 < G; h2 += 2) acc = fadd2(acc, make_float2(p[hh][tl * G + h2], p[hh][tl * G + h2 + 1]));
              v = acc.x + acc.y;
              imp_base[(int64_t)((r0 + 32 * hh) / G + tl) * imp_stride + bidx] = v;
            }
            const unsigned gmx = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
            if (lane == 0) gm_base[(int64_t)((r0 + 32 * hh) / G + tl) * gm_stride + grp] = __uint_as_float(gmx);
          }
        }
      }
      if (!ok) {
        record_timeout(status, &sm.abort_flag);
        break;
      }
      // this tile's scores are complete: hand them to the top-k warps
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.imp_full[lb]);
    }
  } else {
    // ---------------- top-k warps: the selection of each tile's tokens (one warp per token)
    const int tw = warp - kComputeWarps;
    uint32_t n_tile = 0;
    for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x, ++n_tile) {
      const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
      const int lb = n_tile & 1;
      if (!mbar_wait_warp(&sm.imp_full[lb], (n_tile >> 1) & 1)) { record_timeout(status, &sm.abort_flag); break; }
      const float* imp_base = imp_cta + (int64_t)lb * TPT * imp_stride;
      const float* gm_base = gm_cta + (int64_t)lb * TPT * gm_stride;
      for (int tk = tw; tk < TPT; tk += kOutTopkWarps) {
        const int64_t t = ti.t0 + tk;
        if (t < ti.t_end) {
          const float* imp = imp_base + (int64_t)tk * imp_stride;
          const float* gm = gm_base + (int64_t)tk * gm_stride;
          int32_t* dst = sel + (t * hkv + ti.g) * topk;
          if (topk <= 16)
            warp_topk_groups<16>(imp, gm, ti.nb, topk, ti.b0, dst, sm.candv[tw], sm.candi[tw], sm.candg[tw]);
          else
            warp_topk_groups<kTopkMax>(imp, gm, ti.nb, topk, ti.b0, dst, sm.candv[tw], sm.candi[tw], sm.candg[tw]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.imp_empty[lb]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// backward, dQ (thread = row): S = Q Kc^T, dP = dO Vc^T in TMEM over 64-block key
// tiles; dS = P (w dP - D) in registers; dQ += dS Kc with dS (bf16) as the TMEM A
// operand.  A CTA holds 256 TMEM columns and ~80 KB of shared memory, so two
// CTAs share an SM and one's exponentials overlap the other's MMAs.
// ---------------------------------------------------------------------------
constexpr int kBwdStages = 3;
constexpr int kDqBN = 64;                 // compressed blocks per key tile
constexpr int kDqThreads = 32 * (4 + 2);  // one compute warpgroup + TMA warp + MMA warp
constexpr int kDqCtasPerSm = 2;

struct DqSmem {
  uint8_t q[kTile];
  uint8_t dout[kTile];
  uint8_t kc[kBwdStages][kTile / 2];  // 64 blocks x 64 bf16
  uint8_t vc[kBwdStages][kTile / 2];
  uint64_t q_full, q_empty, kv_full[kBwdStages], kv_empty[kBwdStages];
  uint64_t sdp_full, sdp_empty, ds_full, ds_empty, dq_full, dq_empty, mma_done;
  uint32_t tmem;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(kDqThreads, kDqCtasPerSm) cmp_bwd_dq_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
    const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap vcmap,
    const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu, const int32_t* __restrict__ tpre, int S, int hq,
    int hkv, int btot, float qs2, float scale, const float* __restrict__ rc, int64_t rows,
    float* __restrict__ dq_out, int* status) {
  extern __shared__ uint8_t smem_raw[];
  DqSmem& sm = *reinterpret_cast<DqSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntiles = tpre[S];
  const int total = ntiles * hkv;
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < kBwdStages; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_empty, 4);
    mbar_init(&sm.ds_full, 4);
    mbar_init(&sm.ds_empty, 1);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_empty, 4);
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  // TMEM columns: S [0,64), dP [64,128), dS (bf16 pairs) [128,160), dQ [192,256)
  const uint32_t tm_s = tmem, tm_dp = tmem + 64, tm_dsh = tmem + 128, tm_dq = tmem + 192;

  if (warp == 4) {
    // ---------------- TMA producer: (Q, dO) per row tile; (Kc, Vc) per key tile
    if (lane == 0) {
      uint32_t kv_count = 0, q_count = 0;
      int last_par[kBwdStages];
      for (int i = 0; i < kBwdStages; ++i) last_par[i] = -1;
      for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
        const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
        if (!mbar_wait(&sm.q_empty, (q_count & 1) ^ 1)) { record_timeout(status, &sm.abort_flag); break; }
        mbar_expect_tx(&sm.q_full, 2 * kTile);
        tma_load_3d(sm.q, &qmap, &sm.q_full, 0, ti.g * G, ti.t0);
        tma_load_3d(sm.dout, &dmap, &sm.q_full, 0, ti.g * G, ti.t0);
        ++q_count;
        const int nbt = (ti.nb + kDqBN - 1) / kDqBN;
        for (int j = 0; j < nbt; ++j) {
          const int st = kv_count % kBwdStages;
          const uint32_t ph = (kv_count / kBwdStages) & 1;
          if (!mbar_wait(&sm.kv_empty[st], ph ^ 1)) { record_timeout(status, &sm.abort_flag); break; }
          mbar_expect_tx(&sm.kv_full[st], kTile);
          const int row = ti.g * btot + ti.b0 + j * kDqBN;
          tma_load_2d(sm.kc[st], &kcmap, &sm.kv_full[st], 0, row);
          tma_load_2d(sm.vc[st], &vcmap, &sm.kv_full[st], 0, row);
          last_par[st] = (int)ph;
          ++kv_count;
        }
      }
      for (int i = 0; i < kBwdStages; ++i)
        if (last_par[i] >= 0) mbar_wait(&sm.kv_full[i], (uint32_t)last_par[i]);
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(kRows, kDqBN);             // S, dP [rows, blocks]
      const uint32_t id_q = idesc_bf16(kRows, 64, false, true);   // dQ[rows, 64] += dS[rows, blocks] Kc
      uint32_t kv_count = 0, q_count = 0, sdp_count = 0, ds_count = 0, dq_count = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !aborted(&sm.abort_flag); it += gridDim.x) {
        const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
        if (!mbar_wait(&sm.q_full, q_count & 1)) { ok = false; break; }
        ++q_count;
        const int nbt = (ti.nb + kDqBN - 1) / kDqBN;
        auto issue_sdp = [&](uint32_t kv_idx) -> bool {
          const int st = kv_idx % kBwdStages;
          if (!mbar_wait(&sm.kv_full[st], (kv_idx / kBwdStages) & 1) ||
              !mbar_wait(&sm.sdp_empty, (sdp_count & 1) ^ 1))
            return false;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mma_bf16_ss(tm_s, sdesc_kmajor_sw128(sm.q, 32 * k), sdesc_kmajor_sw128(sm.kc[st], 32 * k), id_s, k > 0);
            mma_bf16_ss(tm_dp, sdesc_kmajor_sw128(sm.dout, 32 * k), sdesc_kmajor_sw128(sm.vc[st], 32 * k), id_s,
                        k > 0);
          }
          mma_commit(&sm.sdp_full);
          ++sdp_count;
          return true;
        };
        if (nbt > 0 && !issue_sdp(kv_count)) { ok = false; break; }
        for (int j = 0; j < nbt; ++j) {
          const int st = kv_count % kBwdStages;
          if (j + 1 < nbt && !issue_sdp(kv_count + 1)) { ok = false; break; }
          if ((j == 0 && !mbar_wait(&sm.dq_empty, (dq_count & 1) ^ 1)) || !mbar_wait(&sm.ds_full, ds_count & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kDqBN / 16; ++k) {
            const uint64_t bdesc = sdesc_mnmajor_sw128(sm.kc[st], 2048 * k, kTile);
            mma_bf16_ts(tm_dq, tm_dsh + 8 * k, bdesc, id_q, j > 0 || k > 0);
          }
          mma_commit(&sm.ds_empty);
          mma_commit(&sm.kv_empty[st]);
          ++ds_count;
          ++kv_count;
        }
        if (!ok) break;
        mma_commit(&sm.q_empty);
        mma_commit(&sm.dq_full);
        ++dq_count;
      }
      if (!ok) record_timeout(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ---------------- compute warpgroup: thread = row; the key tile's 64 blocks in two passes of 32
    const int r = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t sdp_count = 0, ds_count = 0, dq_count = 0;
    for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
      const TileInfo ti = tile_info(it, ntiles, tpre, S, cu, bcu, G);
      const int64_t t = ti.t0 + r / G;
      const bool valid = t < ti.t_end;
      const int64_t row = min(t, (int64_t)ti.t_end - 1) * hq + ti.g * G + r % G;
      // row constants: -lse log2(e), w, -D
      const float2 nl2 = make_float2(rc[row], rc[row]);
      const float2 w2 = make_float2(rc[rows + row], rc[rows + row]);
      const float2 nd2 = make_float2(rc[2 * rows + row], rc[2 * rows + row]);
      const float2 qs = make_float2(qs2, qs2);
      const int nbt = (ti.nb + kDqBN - 1) / kDqBN;
      bool ok = true;
      for (int j = 0; j < nbt; ++j) {
        if (!mbar_wait_warp(&sm.sdp_full, sdp_count & 1)) { ok = false; break; }
        tc_fence_after();
        const int nvalid = ti.nb - j * kDqBN;  // valid blocks of this key tile
        bool ok_half = true;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float sv[32], dp[32];
          tmem_ld32(tm_s + lane_off + 32 * hh, sv);
          tmem_ld32(tm_dp + lane_off + 32 * hh, dp);
          tmem_ld_wait();
          if (hh == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sdp_empty);
          }
          const int nvh = nvalid - 32 * hh;
          if (nvh < 32) {  // ragged last key tile: blocks past the sequence get p = 0
#pragma unroll
            for (int c = 0; c < 32; ++c) sv[c] = c < nvh ? sv[c] : -CUDART_INF_F;
          }
          // dS = p (w dP - D), p = 2^(s qs2 - lse log2 e), as one bf16 per entry: dQ of a
          // row sums dS Kc over the row's own blocks, so the roundings of its terms are
          // independent and stay far below the 2e-2 bound (unlike the dKc / dVc sums over
          // up to millions of rows, which carry the low parts)
          uint32_t hi[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 p = ex2x2(ffma2(make_float2(sv[c], sv[c + 1]), qs, nl2));
            hi[c / 2] = pack2(fmul2(p, ffma2(w2, make_float2(dp[c], dp[c + 1]), nd2)));
          }
          if (hh == 0) {
            if (!mbar_wait_warp(&sm.ds_empty, (ds_count & 1) ^ 1)) {
              ok_half = false;
              break;
            }
            tc_fence_after();
          }
          tmem_st16(tm_dsh + lane_off + 16 * hh, hi);
        }
        if (!ok_half) {
          ok = false;
          break;
        }
        ++sdp_count;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ds_full);
        ++ds_count;
      }
      if (!ok) {
        record_timeout(status, &sm.abort_flag);
        break;
      }
      if (!mbar_wait_warp(&sm.dq_full, dq_count & 1)) { record_timeout(status, &sm.abort_flag); break; }
      ++dq_count;
      tc_fence_after();
      float g[64];
      tmem_ld32(tm_dq + lane_off, g);
      tmem_ld32(tm_dq + lane_off + 32, g + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.dq_empty);
      if (valid) {
        float4* dst = reinterpret_cast<float4*>(dq_out + row * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          dst[i] = make_float4(g[4 * i] * scale, g[4 * i + 1] * scale, g[4 * i + 2] * scale, g[4 * i + 3] * scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// backward, dKc / dVc (thread = block): a work item is a 128-block key tile of one
// (sequence, group) against a chunk of up to kDkvRowTilesPerItem row tiles of 128
// query rows.  Per row tile: S^T = Kc Q^T and dP^T = Vc dO^T into TMEM; the compute
// warps turn them into P^T w and dS^T = P^T (w dP - D) and store them back into TMEM
// as fp16 (round to nearest even); dVc += (P^T w) dO and dKc += dS^T Q take them as
// the TMEM operand.  Every operand of this kernel is fp16 (kind::f16 wants A and B of
// one type): Q, dO, Kc and Vc come as exact fp16 copies of the bf16 inputs, made by
// the backward preamble.  fp16's 11-bit significand is what keeps the key gradients
// accurate: they sum P w dO and dS Q over millions of query rows, and a bf16 P (8
// bits) carries a rounding error of about 2^-9 relative into sums of magnitude ~10
// coherently, while fp16 brings it 8x lower (a fixed-point or high + low split costs
// twice the products).
// ---------------------------------------------------------------------------
constexpr int kDkvRowTilesPerItem = 128;
constexpr int kDkvQStages = 4;  // Q / dO / row-constant stages: each row tile is used once per item
// four compute warpgroups of 32 rows each (thread = block): enough warps to hide
// the latency of the per-score arithmetic
constexpr int kDkvComputeWarps = 16;
constexpr int kDkvThreads = 32 * (kDkvComputeWarps + 2);

struct DkvSmem {
  uint8_t kc[kTile];
  uint8_t vc[kTile];
  uint8_t q[kDkvQStages][kTile];
  uint8_t dout[kDkvQStages][kTile];
  // row constants, TMA destinations (128-byte aligned): -lse log2(e), -D, w
  __align__(128) float lse2[kDkvQStages][kRows];
  __align__(128) float Dr[kDkvQStages][kRows];
  __align__(128) float wr[kDkvQStages][kRows];
  uint64_t kv_full, kv_empty, q_full[kDkvQStages], q_empty[kDkvQStages];
  uint64_t sdp_full, sdp_empty, pds_full, pds_empty, acc_full, acc_empty, mma_done;
  uint32_t tmem;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(kDkvThreads, 1) cmp_bwd_dkv_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
    const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap vcmap,
    const __grid_constant__ CUtensorMap lsemap, const __grid_constant__ CUtensorMap dcmap,
    const __grid_constant__ CUtensorMap wmap, const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu,
    const int32_t* __restrict__ ipre, int S, int hq, int hkv, int btot, float qs2, float scale,
    float* __restrict__ dkc, float* __restrict__ dvc, unsigned long long* __restrict__ fkc,
    unsigned long long* __restrict__ fvc, int* status) {
  extern __shared__ uint8_t smem_raw[];
  DkvSmem& sm = *reinterpret_cast<DkvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int TPT = kRows / G;
  const int nitems_g = ipre[S];
  const int total = nitems_g * hkv;
  // item -> (g, s, key tile, row-tile range); items of a sequence: nkt x nchunks, key tile fastest
  auto item_of = [&](int it, int& g, int& s, int& kt, int& rt0, int& rt1, int& t_beg, int& t_end, int& b0, int& nb) {
    g = it / nitems_g;
    const int local = it % nitems_g;
    s = find_segment(ipre, S, local);
    const int k = local - ipre[s];
    b0 = bcu[s];
    nb = bcu[s + 1] - b0;
    const int nkt = (nb + kBN - 1) / kBN;
    kt = k % nkt;
    const int chunk = k / nkt;
    t_beg = cu[s];
    t_end = cu[s + 1];
    const int nrt = (t_end - t_beg + TPT - 1) / TPT;
    rt0 = chunk * kDkvRowTilesPerItem;
    rt1 = min(nrt, rt0 + kDkvRowTilesPerItem);
  };
  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_empty, 1);
    for (int i = 0; i < kDkvQStages; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_empty, kDkvComputeWarps);
    mbar_init(&sm.pds_full, kDkvComputeWarps);
    mbar_init(&sm.pds_empty, 1);
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, kDkvComputeWarps);
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  // TMEM columns: S^T [0,128), dP^T [128,256), P^T w [256,320), dS^T [320,384), dKc [384,448), dVc [448,512)
  const uint32_t tm_s = tmem, tm_dp = tmem + 128, tm_p = tmem + 256, tm_ds = tmem + 320, tm_dk = tmem + 384,
                 tm_dv = tmem + 448;

  if (warp == kDkvComputeWarps) {
    // ---------------- producer warp: (Kc, Vc) per item; (Q, dO) + row scalars per row tile
    uint32_t kv_count = 0, q_count = 0;
    bool kv_issued = false;
    uint32_t kv_last_par = 0;
    for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
      int g, s, kt, rt0, rt1, t_beg, t_end, b0, nb;
      item_of(it, g, s, kt, rt0, rt1, t_beg, t_end, b0, nb);
      bool okk = true;
      if (lane == 0) {
        okk = mbar_wait(&sm.kv_empty, (kv_count & 1) ^ 1);
        if (okk) {
          mbar_expect_tx(&sm.kv_full, 2 * kTile);
          const int row = g * btot + b0 + kt * kBN;
          tma_load_2d(sm.kc, &kcmap, &sm.kv_full, 0, row);
          tma_load_2d(sm.vc, &vcmap, &sm.kv_full, 0, row);
          kv_last_par = kv_count & 1;
          kv_issued = true;
        }
      }
      okk = __shfl_sync(0xffffffffu, okk ? 1 : 0, 0) != 0;
      if (!okk) { record_timeout(status, &sm.abort_flag); break; }
      ++kv_count;
      for (int rt = rt0; rt < rt1; ++rt) {
        const int qb = q_count % kDkvQStages;
        bool okw = true;
        if (lane == 0) okw = mbar_wait(&sm.q_empty[qb], ((q_count / kDkvQStages) & 1) ^ 1);
        okw = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
        if (!okw) { record_timeout(status, &sm.abort_flag); break; }
        const int t0 = t_beg + rt * TPT;
        if (lane == 0) {
          // Q, dO tiles and the row scalars (lse, D, gate weight) of the row tile
          mbar_expect_tx(&sm.q_full[qb], 2 * kTile + 3 * kRows * 4);
          tma_load_3d(sm.q[qb], &qmap, &sm.q_full[qb], 0, g * G, t0);
          tma_load_3d(sm.dout[qb], &dmap, &sm.q_full[qb], 0, g * G, t0);
          tma_load_2d(sm.lse2[qb], &lsemap, &sm.q_full[qb], g * G, t0);
          tma_load_2d(sm.Dr[qb], &dcmap, &sm.q_full[qb], g * G, t0);
          tma_load_2d(sm.wr[qb], &wmap, &sm.q_full[qb], g * G, t0);
        }
        ++q_count;
      }
    }
    if (lane == 0 && kv_issued) mbar_wait(&sm.kv_full, kv_last_par);
    (void)kv_last_par;
  } else if (warp == kDkvComputeWarps + 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(kBN, kRows, false, false, true);  // S^T, dP^T [blocks, rows], fp16
      const uint32_t id_a = idesc_bf16(kBN, 64, false, true, true);      // dKc / dVc [blocks, 64] += X^T Y, fp16
      uint32_t kv_count = 0, q_count = 0, sdp_count = 0, pds_count = 0, acc_count = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !aborted(&sm.abort_flag); it += gridDim.x) {
        int g, s, kt, rt0, rt1, t_beg, t_end, b0, nb;
        item_of(it, g, s, kt, rt0, rt1, t_beg, t_end, b0, nb);
        if (!mbar_wait(&sm.kv_full, kv_count & 1)) { ok = false; break; }
        ++kv_count;
        const int nrt = rt1 - rt0;
        auto issue_sdp = [&](uint32_t qi) -> bool {
          const int qb = qi % kDkvQStages;
          if (!mbar_wait(&sm.q_full[qb], (qi / kDkvQStages) & 1) || !mbar_wait(&sm.sdp_empty, (sdp_count & 1) ^ 1))
            return false;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mma_bf16_ss(tm_s, sdesc_kmajor_sw128(sm.kc, 32 * k), sdesc_kmajor_sw128(sm.q[qb], 32 * k), id_s, k > 0);
            mma_bf16_ss(tm_dp, sdesc_kmajor_sw128(sm.vc, 32 * k), sdesc_kmajor_sw128(sm.dout[qb], 32 * k), id_s,
                        k > 0);
          }
          mma_commit(&sm.sdp_full);
          ++sdp_count;
          return true;
        };
        if (nrt > 0 && !issue_sdp(q_count)) { ok = false; break; }
        for (int i = 0; i < nrt; ++i) {
          const int qb = q_count % kDkvQStages;
          if (i == 0 && !mbar_wait(&sm.acc_empty, (acc_count & 1) ^ 1)) { ok = false; break; }
          // S^T / dP^T of the next tile first: the compute warps release this tile's
          // S^T / dP^T before they hand over its P^T w / dS^T, so the next products
          // queue on the tensor pipe ahead of this tile's dKc / dVc and run while the
          // compute warps finish
          if (i + 1 < nrt && !issue_sdp(q_count + 1)) { ok = false; break; }
          if (!mbar_wait(&sm.pds_full, pds_count & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kRows / 16; ++k) {
            mma_bf16_ts(tm_dv, tm_p + 8 * k, sdesc_mnmajor_sw128(sm.dout[qb], 2048 * k, kTile), id_a, i > 0 || k > 0);
            mma_bf16_ts(tm_dk, tm_ds + 8 * k, sdesc_mnmajor_sw128(sm.q[qb], 2048 * k, kTile), id_a, i > 0 || k > 0);
          }
          mma_commit(&sm.pds_empty);
          mma_commit(&sm.q_empty[qb]);
          ++pds_count;
          ++q_count;
        }
        if (!ok) break;
        mma_commit(&sm.kv_empty);
        mma_commit(&sm.acc_full);
        ++acc_count;
      }
      if (!ok) record_timeout(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ---------------- compute warps: thread = block; warpgroup wg owns rows [32 wg, 32 wg + 32)
    const int b = threadIdx.x % 128;
    const int wg = warp / 4;
    const int r0 = 32 * wg;
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    uint32_t sdp_count = 0, pds_count = 0, acc_count = 0, q_count = 0;
    for (int it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
      int g, s, kt, rt0, rt1, t_beg, t_end, b0, nb;
      item_of(it, g, s, kt, rt0, rt1, t_beg, t_end, b0, nb);
      const int nrt = rt1 - rt0;
      bool ok = true;
      for (int i = 0; i < nrt; ++i) {
        const int qb = q_count % kDkvQStages;
        // S^T / dP^T of this tile, and its row constants (-lse log2 e, -D, w), which
        // arrived with q_full[qb]
        if (!mbar_wait_warp(&sm.sdp_full, sdp_count & 1) ||
            !mbar_wait_warp(&sm.q_full[qb], (q_count / kDkvQStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int t_first = t_beg + (rt0 + i) * TPT;
        const int nvr = (int)min((int64_t)kRows, (int64_t)(t_end - t_first) * G) - r0;  // valid rows of this warpgroup
        const float2 qs = make_float2(qs2, qs2);
        // the warpgroup's 32 rows in two passes of 16; S^T / dP^T are released after
        // the second read, P^T w / dS^T (fp16) written once the MMAs of the previous
        // tile consumed them.
        bool ok_half = true;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float sv[16], dp[16];
          tmem_ld16(tm_s + lane_off + r0 + 16 * hh, sv);
          tmem_ld16(tm_dp + lane_off + r0 + 16 * hh, dp);
          tmem_ld_wait();
          if (hh == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sdp_empty);
          }
          const int nvh = nvr - 16 * hh;
          if (nvh < 16) {  // rows of tokens past the sequence get p = 0
#pragma unroll
            for (int c = 0; c < 16; ++c) sv[c] = c < nvh ? sv[c] : -CUDART_INF_F;
          }
          uint32_t pw[8], dsv[8];
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const int rr = r0 + 16 * hh + c;
            const float4 l4 = *reinterpret_cast<const float4*>(&sm.lse2[qb][rr]);
            const float4 d4 = *reinterpret_cast<const float4*>(&sm.Dr[qb][rr]);
            const float4 w4 = *reinterpret_cast<const float4*>(&sm.wr[qb][rr]);
            const float2 wa = make_float2(w4.x, w4.y), wb = make_float2(w4.z, w4.w);
            const float2 pa = ex2x2(ffma2(make_float2(sv[c], sv[c + 1]), qs, make_float2(l4.x, l4.y)));
            const float2 pb = ex2x2(ffma2(make_float2(sv[c + 2], sv[c + 3]), qs, make_float2(l4.z, l4.w)));
            pw[c / 2] = pack_f16x2(fmul2(pa, wa));
            pw[c / 2 + 1] = pack_f16x2(fmul2(pb, wb));
            dsv[c / 2] = pack_f16x2(fmul2(pa, ffma2(wa, make_float2(dp[c], dp[c + 1]), make_float2(d4.x, d4.y))));
            dsv[c / 2 + 1] = pack_f16x2(fmul2(pb, ffma2(wb, make_float2(dp[c + 2], dp[c + 3]), make_float2(d4.z, d4.w))));
          }
          if (hh == 0) {
            if (!mbar_wait_warp(&sm.pds_empty, (pds_count & 1) ^ 1)) {
              ok_half = false;
              break;
            }
            tc_fence_after();
          }
          // rows [r0 + 16 hh, +16): packed TMEM columns [r0/2 + 8 hh, +8)
          tmem_st8(tm_p + lane_off + r0 / 2 + 8 * hh, pw);
          tmem_st8(tm_ds + lane_off + r0 / 2 + 8 * hh, dsv);
        }
        if (!ok_half) {
          ok = false;
          break;
        }
        ++sdp_count;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.pds_full);
        ++pds_count;
        ++q_count;
      }
      if (!ok) {
        record_timeout(status, &sm.abort_flag);
        break;
      }
      if (!mbar_wait_warp(&sm.acc_full, acc_count & 1)) { record_timeout(status, &sm.abort_flag); break; }
      ++acc_count;
      tc_fence_after();
      // warpgroups 0, 1 add dKc columns [0, 32), [32, 64); warpgroups 2, 3 the same of dVc (lane = block)
      float acc[32];
      const uint32_t src = (wg < 2 ? tm_dk : tm_dv) + lane_off + 32 * (wg & 1);
      tmem_ld32(src, acc);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);
      const int bidx = kt * kBN + b;
      if (bidx < nb && nrt > 0) {
        const int64_t off = ((int64_t)g * btot + b0 + bidx) * 64 + 32 * (wg & 1);
        const float mul = wg < 2 ? scale : 1.f;
        if (fkc) {  // deterministic: 64-bit fixed-point sums (integer addition is associative)
          unsigned long long* dst = (wg < 2 ? fkc : fvc) + off;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            atomicAdd(dst + i, (unsigned long long)__float2ll_rn(acc[i] * mul * kFixScale));
        } else {
          float* dst = (wg < 2 ? dkc : dvc) + off;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            atomicAdd(reinterpret_cast<float4*>(dst) + i,
                      make_float4(acc[4 * i] * mul, acc[4 * i + 1] * mul, acc[4 * i + 2] * mul, acc[4 * i + 3] * mul));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Two bf16 arrays of n8 x 8 values -> fp16 copies (exact down to 2^-14, where fp16
// turns subnormal), eight values per thread and step: the operands of the dKc / dVc
// kernel (Q and dO; Kc and Vc).
__global__ void to_f16_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, uint4* __restrict__ a16,
                              uint4* __restrict__ b16, int64_t n8) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < 2 * n8; i += (int64_t)gridDim.x * blockDim.x) {
    const bool second = i >= n8;
    const int64_t j = second ? i - n8 : i;
    const uint4 x = __ldcs((second ? b : a) + j);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      o[c] = pack_f16x2(make_float2(__uint_as_float(w[c] << 16), __uint_as_float(w[c] & 0xffff0000u)));
    (second ? b16 : a16)[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

int to_f16_grid(int64_t n8, int sms) {
  const int64_t blocks = (2 * n8 + 255) / 256;
  return (int)(blocks < 8 * (int64_t)sms ? (blocks > 0 ? blocks : 1) : 8 * (int64_t)sms);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------


size_t smem_bytes_fa() { return sizeof(FaSmem) + 1024; }
size_t smem_bytes_sel() { return sizeof(SelSmem) + 1024; }

// Pairs of 128-row tiles per sequence (per group), for the output pass.
__global__ void pair_plan_kernel(const int32_t* __restrict__ cu, int S, int G, int32_t* __restrict__ cnt) {
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s <= S; s += gridDim.x * blockDim.x) {
    if (s == S) {
      cnt[s] = 0;
      continue;
    }
    const int64_t rows = (int64_t)(cu[s + 1] - cu[s]) * G;
    cnt[s] = (int32_t)((rows + 2 * kRows - 1) / (2 * kRows));
  }
}

template <int G>
cudaError_t cmp_fwd_tc_g(const FwdArgs& a, const int32_t* tpre, int64_t total_tiles_bound, cudaStream_t st) {
  CUtensorMap qm, km, kmf, vmf;  // km: 128-block key tiles (selection pass); kmf, vmf: kFaBN (output pass)
  const int64_t rows_kv = (int64_t)a.hkv * a.blk->count;
  if (!map_q(&qm, a.q, a.N, a.hq, G) || !map_rows64(&km, a.kc, rows_kv) || !map_rows64(&kmf, a.kc, rows_kv, kFaBN) ||
      !map_rows64(&vmf, a.vc, rows_kv, kFaBN))
    return cudaErrorInvalidValue;
  const float qs2 = a.scale * kLog2e;
  const int btot = (int)a.blk->count;
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(cmp_fa_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes_fa());
    cudaFuncSetAttribute(cmp_fa_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes_fa());
    cudaFuncSetAttribute(cmp_sel_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes_sel());
    cudaFuncSetAttribute(cmp_sel_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes_sel());
    attr_done = true;
  }
  // output pass: pairs of row tiles (the per-sequence pair prefix goes to tiles_cnt / tiles_pre,
  // which the tensor-core forward does not otherwise use)
  SSA_LAUNCH("pair_plan_kernel", pair_plan_kernel, (a.S + 256) / 256, 256, 0, st, a.cu_seqlens, a.S, G,
             a.tiles_cnt);
  cudaError_t e = exclusive_scan(a.tiles_cnt, a.tiles_pre, a.S + 1, a.scan_tmp, st);
  if (e != cudaSuccess) return e;
  const int sms = num_sms();
  const int64_t pairs = ((total_tiles_bound + 1) / 2 + a.S) * a.hkv;
  const int g1 = (int)(pairs < sms ? (pairs > 0 ? pairs : 1) : sms);
  SSA_LAUNCH("cmp_fa_tc_kernel", cmp_fa_tc_kernel<G>, g1, kFaThreads, smem_bytes_fa(), st, qm, kmf, vmf, a.cu_seqlens,
             a.blk->cu, a.tiles_pre, a.S, a.N, a.hq, a.hkv, btot, qs2, a.o_branch, a.lse, a.status);
  if (!a.sel_given) {  // a given selection needs no scores
    const int64_t tiles = total_tiles_bound * a.hkv;
    const int smax = sms < kCmpOutCtas ? sms : kCmpOutCtas;  // the score scratch holds kCmpOutCtas CTAs
    const int g2 = (int)(tiles < smax ? (tiles > 0 ? tiles : 1) : smax);
    SSA_LAUNCH("cmp_sel_tc_kernel", cmp_sel_tc_kernel<G>, g2, kOutThreadsTk, smem_bytes_sel(), st, qm, km,
               a.cu_seqlens, a.blk->cu, tpre, a.S, a.hq, a.hkv, btot, qs2, a.lse, a.topk, a.sel, a.imp_scratch,
               (int64_t)((btot + 3) & ~3), (int64_t)(((btot + 31) / 32 + 3) & ~3), a.status);
  }
  return cudaGetLastError();
}


__global__ void dkv_plan_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu, int S, int G,
                                int32_t* __restrict__ cnt) {
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s <= S; s += gridDim.x * blockDim.x) {
    if (s == S) {
      cnt[s] = 0;
      continue;
    }
    const int nb = bcu[s + 1] - bcu[s];
    const int64_t rows = (int64_t)(cu[s + 1] - cu[s]) * G;
    const int64_t nrt = (rows + kRows - 1) / kRows;
    const int64_t nch = (nrt + kDkvRowTilesPerItem - 1) / kDkvRowTilesPerItem;
    cnt[s] = (int32_t)(((nb + kBN - 1) / kBN) * nch);
  }
}

size_t smem_bytes_dq() { return sizeof(DqSmem) + 1024; }
size_t smem_bytes_dkv() { return sizeof(DkvSmem) + 1024; }

template <int G>
cudaError_t cmp_bwd_tc_g(const BwdArgs& a, const int32_t* tpre, int32_t* dkv_cnt, int32_t* dkv_pre,
                         int32_t* scan_tmp, int64_t tiles_bound, cudaStream_t st) {
  CUtensorMap qm, dm;
  const int64_t rows_kv = (int64_t)a.hkv * a.blk->count;
  CUtensorMap km64, vm64;  // 64-block key tiles of the dQ kernel
  if (!a.q16 || !map_q(&qm, a.q, a.N, a.hq, G) || !map_q(&dm, a.dout, a.N, a.hq, G) ||
      !map_rows64(&km64, a.kc, rows_kv, kDqBN) || !map_rows64(&vm64, a.vc, rows_kv, kDqBN))
    return cudaErrorInvalidValue;
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(cmp_bwd_dq_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes_dq());
    cudaFuncSetAttribute(cmp_bwd_dq_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes_dq());
    cudaFuncSetAttribute(cmp_bwd_dkv_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes_dkv());
    cudaFuncSetAttribute(cmp_bwd_dkv_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes_dkv());
    attr_done = true;
  }
  const float qs2 = a.scale * kLog2e;
  const int btot = (int)a.blk->count;
  const int sms = num_sms();
  const int64_t tiles = tiles_bound * a.hkv;
  const int gq = (int)(tiles < kDqCtasPerSm * sms ? (tiles > 0 ? tiles : 1) : kDqCtasPerSm * sms);
  const int64_t rows = a.N * a.hq;
  SSA_LAUNCH("cmp_bwd_dq_tc_kernel", cmp_bwd_dq_tc_kernel<G>, gq, kDqThreads, smem_bytes_dq(), st, qm, dm, km64, vm64,
             a.cu_seqlens, a.blk->cu, tpre, a.S, a.hq, a.hkv, btot, qs2, a.scale, a.rc, rows, a.dq, a.status);
  SSA_LAUNCH("dkv_plan_kernel", dkv_plan_kernel, (a.S + 256) / 256, 256, 0, st, a.cu_seqlens, a.blk->cu, a.S, G,
             dkv_cnt);
  cudaError_t e = exclusive_scan(dkv_cnt, dkv_pre, a.S + 1, scan_tmp, st);
  if (e != cudaSuccess) return e;
  if (a.fx_kc) {  // deterministic: the kernel adds fixed-point integers, converted below
    cudaMemsetAsync(a.fx_kc, 0, sizeof(unsigned long long) * rows_kv * 64, st);
    cudaMemsetAsync(a.fx_vc, 0, sizeof(unsigned long long) * rows_kv * 64, st);
  } else {
    cudaMemsetAsync(a.dkc, 0, sizeof(float) * rows_kv * 64, st);
    cudaMemsetAsync(a.dvc, 0, sizeof(float) * rows_kv * 64, st);
  }
  // row constants of the compressed branch: -lse log2(e), -D, w
  CUtensorMap lm, dcm, wm;
  if (!map_rowscalars(&lm, a.rc, a.N, a.hq, G) || !map_rowscalars(&dcm, a.rc + 2 * rows, a.N, a.hq, G) ||
      !map_rowscalars(&wm, a.rc + rows, a.N, a.hq, G))
    return cudaErrorInvalidValue;
  // the fp16 operands: Q, dO [N, Hq, 64] and Kc, Vc [Hkv, B, 64].  The maps move
  // 2-byte elements without conversion, so the bf16 map layout serves fp16.
  const int64_t q8 = rows * 64 / 8, kv8 = rows_kv * 64 / 8;
  SSA_LAUNCH("to_f16_kernel", to_f16_kernel, to_f16_grid(q8, sms), 256, 0, st, static_cast<const uint4*>(a.q),
             static_cast<const uint4*>(a.dout), static_cast<uint4*>(a.q16), static_cast<uint4*>(a.do16), q8);
  SSA_LAUNCH("to_f16_kernel", to_f16_kernel, to_f16_grid(kv8, sms), 256, 0, st, static_cast<const uint4*>(a.kc),
             static_cast<const uint4*>(a.vc), static_cast<uint4*>(a.kc16), static_cast<uint4*>(a.vc16), kv8);
  CUtensorMap q16m, d16m, k16m, v16m;
  if (!map_q(&q16m, a.q16, a.N, a.hq, G) || !map_q(&d16m, a.do16, a.N, a.hq, G) || !map_rows64(&k16m, a.kc16, rows_kv) ||
      !map_rows64(&v16m, a.vc16, rows_kv))
    return cudaErrorInvalidValue;
  SSA_LAUNCH("cmp_bwd_dkv_tc_kernel", cmp_bwd_dkv_tc_kernel<G>, sms, kDkvThreads, smem_bytes_dkv(), st, q16m, d16m,
             k16m, v16m, lm, dcm, wm, a.cu_seqlens, a.blk->cu, dkv_pre, a.S, a.hq, a.hkv, btot, qs2, a.scale, a.dkc,
             a.dvc, a.fx_kc, a.fx_vc, a.status);
  if (a.fx_kc) {
    e = fix_to_float(a.fx_kc, a.dkc, rows_kv * 64, st);
    if (e == cudaSuccess) e = fix_to_float(a.fx_vc, a.dvc, rows_kv * 64, st);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}
}  // namespace

size_t cmp_tc_scratch_floats(int hq, int hkv, int64_t btot) {
  const int G = hkv > 0 ? hq / hkv : 1;
  const size_t per_token = (size_t)((btot + 3) & ~int64_t(3)) + (size_t)(((btot + 31) / 32 + 3) & ~int64_t(3));
  return (size_t)kCmpOutCtas * 2 * (kRows / (G > 0 ? G : 1)) * per_token + 4;
}

bool cmp_tc_supported(int dtype, int d, int hq, int hkv, int topk) {
  const int G = hkv > 0 ? hq / hkv : 0;
  return dtype == SSA_DTYPE_BF16 && d == 64 && (G == 8 || G == 16) && topk <= kTopkMax && encode_fn() != nullptr;
}

// Compressed branch forward (lse, o_cmp, sel) on the tensor cores; `tpre` is the
// per-sequence prefix of 128-row tiles (per group).
cudaError_t cmp_fwd_tc(const FwdArgs& a, const int32_t* tpre, int64_t total_tiles_bound, cudaStream_t st) {
  const int G = a.hq / a.hkv;
  if (G == 16) return cmp_fwd_tc_g<16>(a, tpre, total_tiles_bound, st);
  if (G == 8) return cmp_fwd_tc_g<8>(a, tpre, total_tiles_bound, st);
  return cudaErrorInvalidValue;
}

}  // namespace ssa

namespace ssa {
// Compressed branch backward on the tensor cores: dQ (written), dKc / dVc (fp32
// workspace, accumulated).  `tpre` is the per-sequence prefix of 128-row tiles.
cudaError_t cmp_bwd_tc(const BwdArgs& a, const int32_t* tpre, int32_t* dkv_cnt, int32_t* dkv_pre, int32_t* scan_tmp,
                       int64_t tiles_bound, cudaStream_t st) {
  const int G = a.hq / a.hkv;
  if (G == 16) return cmp_bwd_tc_g<16>(a, tpre, dkv_cnt, dkv_pre, scan_tmp, tiles_bound, st);
  if (G == 8) return cmp_bwd_tc_g<8>(a, tpre, dkv_cnt, dkv_pre, scan_tmp, tiles_bound, st);
  return cudaErrorInvalidValue;
}
}  // namespace ssa
