// Selected-block branch of SSA on warp-level tensor-core MMAs (mma.sync m16n8k16,
// bf16 operands, fp32 accumulation), head dim 64, G = Hq/Hkv in {8, 16}.
//
// Direct3D-S2 (hyper.ai, "方法"): every query attends to all tokens of the top-k
// blocks its GQA group selected.  The selection favours small blocks, so a
// (token, group) sees a few dozen keys scattered over the sequence: a gather, not a
// dense tile.  One warp owns one (token, group).  The group's G query heads are the
// 16 rows of the MMA tile (G = 8 leaves rows 8..15 zero).  The tokens of the
// selected blocks (rows of the block-sorted K_s / V_s) are gathered 32 at a time
// into padded shared memory and read back with ldmatrix.  Products of a probability
// (P, dS) with an operand use bf16 high + low parts, as in the other branches.
//
//   slc_fwd_mma:  S = Q K^T, online softmax over the chunks, O += P V.
//   slc_bwd_mma:  S, dP = dO V^T; dS = P (w dP - D); dQ += dS K (registers);
//                 dK += dS^T Q, dV += (P w)^T dO per chunk, added to the key
//                 tokens' rows with vector atomics.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tc_host.cuh"

namespace ssa {
namespace {

using tc::ex2;
using tc::fmul2;
using tc::ffma2;
using tc::smem_u32;
using tc::split2;

constexpr int kChunk = 32;     // keys gathered per step
constexpr int kRowB = 144;     // bytes per staged K/V/Q row: 64 bf16 + 16 pad (conflict-free ldmatrix)
constexpr int kPRowB = 80;     // bytes per staged P/dS row: 32 bf16 + 16 pad
constexpr int kSlcWarps = 4;   // warps per CTA, one (token, group) each
constexpr int kSlcTopkMax = 32;

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// four 8x8 b16 matrices; lane l gives the address of row l % 8 of matrix l / 8
__device__ __forceinline__ void ldsm4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// The key list of a (token, group): the selected blocks' token ranges in K_s order.
// Lane i < topk holds block i's start row and the exclusive prefix of the sizes.
struct KeyList {
  int start, pre, total;
};
__device__ __forceinline__ KeyList key_list(const int32_t* srow, const int32_t* bptr, int topk, int lane) {
  int b = lane < topk ? srow[lane] : -1;
  const int start = b >= 0 ? bptr[b] : 0;
  const int n = b >= 0 ? bptr[b + 1] - start : 0;
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  KeyList kl;
  kl.start = start;
  kl.pre = incl - n;
  kl.total = __shfl_sync(0xffffffffu, incl, 31);
  return kl;
}
// K_s row (within the group) of key k of the list: the block of the last lane whose
// prefix is <= k (prefixes ascend; lanes past topk hold the total); every lane
// searches for its own k.
__device__ __forceinline__ int key_row(const KeyList& kl, int k) {
  int lo = 0;
#pragma unroll
  for (int step = 16; step >= 1; step >>= 1) {
    const int cand = lo + step;
    if (__shfl_sync(0xffffffffu, kl.pre, cand & 31) <= k && cand < 32) lo = cand;
  }
  const int st = __shfl_sync(0xffffffffu, kl.start, lo);
  const int pr = __shfl_sync(0xffffffffu, kl.pre, lo);
  return st + (k - pr);
}

// Copy 128-byte rows (64 bf16) into a staged tile with kRowB stride; lanes past
// `n` write zeros.  `src_row(i)` is the element offset of row i.
template <typename F>
__device__ __forceinline__ void stage_rows(uint8_t* dst, const __nv_bfloat16* base, int n, int lane, F src_row) {
  if (lane < kChunk) {
    uint4* d = reinterpret_cast<uint4*>(dst + lane * kRowB);
    if (lane < n) {
      const uint4* s = reinterpret_cast<const uint4*>(base + src_row(lane));
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = s[i];
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = make_uint4(0, 0, 0, 0);
    }
  }
}
// the G head rows of one token (rows >= G zero), 16 rows of kRowB
__device__ __forceinline__ void stage_heads(uint8_t* dst, const __nv_bfloat16* rows, int G, int lane) {
  // 16 rows x 8 uint4 = 128 copies, 4 per lane
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = lane + 32 * i;
    const int r = idx / 8, c = idx % 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < G) v = reinterpret_cast<const uint4*>(rows + (int64_t)r * 64)[c];
    *reinterpret_cast<uint4*>(dst + r * kRowB + c * 16) = v;
  }
}

// A fragments (16 rows x 64) of a staged 16-row tile, k-steps of 16
__device__ __forceinline__ void load_a64(uint32_t (*a)[4], const uint8_t* tile, int lane) {
  const int mi = lane / 8, ri = lane % 8;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm4(a[ks], smem_u32(tile + ((mi & 1) * 8 + ri) * kRowB + (16 * ks + (mi >> 1) * 8) * 2));
}
// S[16 x 32] = A[16 x 64] B^T with B = 32 staged rows (keys)
__device__ __forceinline__ void mma_rows_keys(float (*s)[4], const uint32_t (*a)[4], const uint8_t* keys, int lane) {
  const int mi = lane / 8, ri = lane % 8;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) {
      uint32_t b[4];
      ldsm4(b, smem_u32(keys + (8 * nt + ri) * kRowB + (32 * kp + 8 * mi) * 2));
      mma16816(s[nt], a[2 * kp], b[0], b[1]);
      mma16816(s[nt], a[2 * kp + 1], b[2], b[3]);
    }
  }
}
// A fragment (16 rows x 16 keys) of k-step kk from the C fragments of n-tiles 2kk, 2kk+1
__device__ __forceinline__ void c_to_a(const float (*p)[4], int kk, uint32_t* hi, uint32_t* lo) {
  split2(make_float2(p[2 * kk][0], p[2 * kk][1]), hi[0], lo[0]);
  split2(make_float2(p[2 * kk][2], p[2 * kk][3]), hi[1], lo[1]);
  split2(make_float2(p[2 * kk + 1][0], p[2 * kk + 1][1]), hi[2], lo[2]);
  split2(make_float2(p[2 * kk + 1][2], p[2 * kk + 1][3]), hi[3], lo[3]);
}
// acc[16 x 64] += A[16 x 32] X with X = 32 staged rows (keys) x 64, A given as hi + lo
__device__ __forceinline__ void mma_keys_dims(float (*acc)[4], const float (*p)[4], const uint8_t* rows, int lane) {
  const int mi = lane / 8, ri = lane % 8;
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    uint32_t ahi[4], alo[4];
    c_to_a(p, kk, ahi, alo);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      ldsm4t(b, smem_u32(rows + (16 * kk + (mi & 1) * 8 + ri) * kRowB + (16 * np + (mi >> 1) * 8) * 2));
      mma16816(acc[2 * np], ahi, b[0], b[1]);
      mma16816(acc[2 * np], alo, b[0], b[1]);
      mma16816(acc[2 * np + 1], ahi, b[2], b[3]);
      mma16816(acc[2 * np + 1], alo, b[2], b[3]);
    }
  }
}

struct SlcFwdSmem {
  __align__(16) uint8_t q[kSlcWarps][16 * kRowB];
  __align__(16) uint8_t k[kSlcWarps][kChunk * kRowB];
  __align__(16) uint8_t v[kSlcWarps][kChunk * kRowB];
};

template <int G>
__global__ void __launch_bounds__(32 * kSlcWarps) slc_fwd_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ ks, const __nv_bfloat16* __restrict__ vs,
    const int32_t* __restrict__ bptr, const int32_t* __restrict__ sel, int64_t N, int64_t ldk, int hq, int hkv,
    int topk, float qs2, float* __restrict__ o_out, float* __restrict__ lse_out) {
  __shared__ SlcFwdSmem sm;
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  uint8_t* qs_t = sm.q[w];
  uint8_t* ks_t = sm.k[w];
  uint8_t* vs_t = sm.v[w];
  const int64_t npairs = N * hkv;
  for (int64_t pair = (int64_t)blockIdx.x * kSlcWarps + w; pair < npairs; pair += (int64_t)gridDim.x * kSlcWarps) {
    const int64_t t = pair / hkv;
    const int g = (int)(pair % hkv);
    const __nv_bfloat16* kg = ks + (int64_t)g * ldk * 64;
    const __nv_bfloat16* vg = vs + (int64_t)g * ldk * 64;
    stage_heads(qs_t, q + (t * hq + (int64_t)g * G) * 64, G, lane);
    const KeyList kl = key_list(sel + pair * topk, bptr, topk, lane);
    __syncwarp();
    uint32_t qa[4][4];
    load_a64(qa, qs_t, lane);
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;  // rows gid, gid + 8
    for (int c0 = 0; c0 < kl.total; c0 += kChunk) {
      const int nk = min(kChunk, kl.total - c0);
      const int myrow = key_row(kl, c0 + lane);
      __syncwarp();  // the previous chunk's ldmatrix reads are done
      stage_rows(ks_t, kg, nk, lane, [&](int) { return (int64_t)myrow * 64; });
      stage_rows(vs_t, vg, nk, lane, [&](int) { return (int64_t)myrow * 64; });
      __syncwarp();
      float s[4][4];
      mma_rows_keys(s, qa, ks_t, lane);
      // scores in log2 units; keys past the list masked
      float cm0 = -CUDART_INF_F, cm1 = -CUDART_INF_F;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool valid = 8 * nt + 2 * tig + e < nk;
          s[nt][e] = valid ? s[nt][e] * qs2 : -CUDART_INF_F;
          s[nt][2 + e] = valid ? s[nt][2 + e] * qs2 : -CUDART_INF_F;
          cm0 = fmaxf(cm0, s[nt][e]);
          cm1 = fmaxf(cm1, s[nt][2 + e]);
        }
      }
      cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 1));
      cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 2));
      cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 1));
      cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 2));
      const float n0 = fmaxf(m0, cm0), n1 = fmaxf(m1, cm1);
      const float r0 = ex2(m0 - n0), r1 = ex2(m1 - n1);
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        s[nt][0] = ex2(s[nt][0] - n0);
        s[nt][1] = ex2(s[nt][1] - n0);
        s[nt][2] = ex2(s[nt][2] - n1);
        s[nt][3] = ex2(s[nt][3] - n1);
        ps0 += s[nt][0] + s[nt][1];
        ps1 += s[nt][2] + s[nt][3];
      }
      l0 = l0 * r0 + ps0;
      l1 = l1 * r1 + ps1;
      m0 = n0;
      m1 = n1;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i][0] *= r0;
        o[i][1] *= r0;
        o[i][2] *= r1;
        o[i][3] *= r1;
      }
      mma_keys_dims(o, s, vs_t, lane);
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = gid + 8 * half;
      if (r < G) {
        const int64_t row = t * hq + (int64_t)g * G + r;
        const float inv = half ? i1 : i0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float2*>(o_out + row * 64 + 8 * i + 2 * tig) =
              make_float2(o[i][2 * half] * inv, o[i][2 * half + 1] * inv);
        if (tig == 0) lse_out[row] = ((half ? m1 : m0) + log2f(half ? l1 : l0)) * kLn2;
      }
    }
  }
}

struct SlcBwdSmem {
  __align__(16) uint8_t q[kSlcWarps][16 * kRowB];
  __align__(16) uint8_t d[kSlcWarps][16 * kRowB];
  __align__(16) uint8_t k[kSlcWarps][kChunk * kRowB];
  __align__(16) uint8_t v[kSlcWarps][kChunk * kRowB];
  __align__(16) uint8_t ph[kSlcWarps][16 * kPRowB];  // (P w), hi and lo, [head][key]
  __align__(16) uint8_t pl[kSlcWarps][16 * kPRowB];
  __align__(16) uint8_t dh[kSlcWarps][16 * kPRowB];  // dS, hi and lo
  __align__(16) uint8_t dl[kSlcWarps][16 * kPRowB];
  int tok[kSlcWarps][kChunk];
};

// acc[16 keys x 64] = X^T Y for m-tile mt: X = staged [16 heads][32 keys] (hi + lo), Y = staged 16 head rows x 64
__device__ __forceinline__ void mma_keys_heads(float (*acc)[4], const uint8_t* xh, const uint8_t* xl,
                                               const uint8_t* y, int mt, int lane) {
  const int mi = lane / 8, ri = lane % 8;
  uint32_t ahi[4], alo[4];
  const uint32_t off = ((mi >> 1) * 8 + ri) * kPRowB + (16 * mt + (mi & 1) * 8) * 2;
  ldsm4t(ahi, smem_u32(xh + off));
  ldsm4t(alo, smem_u32(xl + off));
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    uint32_t b[4];
    ldsm4t(b, smem_u32(y + ((mi & 1) * 8 + ri) * kRowB + (16 * np + (mi >> 1) * 8) * 2));
    mma16816(acc[2 * np], ahi, b[0], b[1]);
    mma16816(acc[2 * np], alo, b[0], b[1]);
    mma16816(acc[2 * np + 1], ahi, b[2], b[3]);
    mma16816(acc[2 * np + 1], alo, b[2], b[3]);
  }
}

template <int G>
__global__ void __launch_bounds__(32 * kSlcWarps) slc_bwd_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ ks, const __nv_bfloat16* __restrict__ vs,
    const __nv_bfloat16* __restrict__ dout, const float* __restrict__ gates, int mode,
    const int32_t* __restrict__ bptr, const int32_t* __restrict__ bperm, const int32_t* __restrict__ sel, int64_t N,
    int64_t ldk, int hq, int hkv, int topk, float qs2, float scale, const float* __restrict__ lse_in,
    const float* __restrict__ Dc, float* __restrict__ dq_out, float* __restrict__ dk_out,
    float* __restrict__ dv_out, unsigned long long* __restrict__ fk, unsigned long long* __restrict__ fv) {
  extern __shared__ uint8_t smem_raw[];
  SlcBwdSmem& sm = *reinterpret_cast<SlcBwdSmem*>(smem_raw);
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  uint8_t *qs_t = sm.q[w], *ds_t = sm.d[w], *ks_t = sm.k[w], *vs_t = sm.v[w];
  const int64_t npairs = N * hkv;
  for (int64_t pair = (int64_t)blockIdx.x * kSlcWarps + w; pair < npairs; pair += (int64_t)gridDim.x * kSlcWarps) {
    const int64_t t = pair / hkv;
    const int g = (int)(pair % hkv);
    const __nv_bfloat16* kg = ks + (int64_t)g * ldk * 64;
    const __nv_bfloat16* vg = vs + (int64_t)g * ldk * 64;
    const int64_t row0 = t * hq + (int64_t)g * G;
    __syncwarp();  // the previous pair's reads of the staged tiles are done
    stage_heads(qs_t, q + row0 * 64, G, lane);
    stage_heads(ds_t, dout + row0 * 64, G, lane);
    const KeyList kl = key_list(sel + pair * topk, bptr, topk, lane);
    // row constants of rows gid, gid + 8: -lse log2(e), w, D (padded rows: p = 0)
    float nl[2], wr[2], dr[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = gid + 8 * half;
      if (r < G) {
        const int64_t row = row0 + r;
        nl[half] = -lse_in[row] * kLog2e;
        const float x = gates[row * 3 + 1];
        wr[half] = mode == SSA_GATE_LOGITS ? 1.f / (1.f + expf(-x)) : x;
        dr[half] = Dc[row];
      } else {
        nl[half] = -CUDART_INF_F;
        wr[half] = 0.f;
        dr[half] = 0.f;
      }
    }
    __syncwarp();
    uint32_t qa[4][4], da[4][4];
    load_a64(qa, qs_t, lane);
    load_a64(da, ds_t, lane);
    float dq[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
    for (int c0 = 0; c0 < kl.total; c0 += kChunk) {
      const int nk = min(kChunk, kl.total - c0);
      const int myrow = key_row(kl, c0 + lane);
      __syncwarp();
      stage_rows(ks_t, kg, nk, lane, [&](int) { return (int64_t)myrow * 64; });
      stage_rows(vs_t, vg, nk, lane, [&](int) { return (int64_t)myrow * 64; });
      sm.tok[w][lane] = lane < nk ? bperm[myrow] : -1;
      __syncwarp();
      float s[4][4], dp[4][4];
      mma_rows_keys(s, qa, ks_t, lane);
      mma_rows_keys(dp, da, vs_t, lane);
      // P = 2^(s qs2 - lse log2 e), masked past the list; P w and dS = P (w dP - D)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int half = e >> 1;
          const bool valid = 8 * nt + 2 * tig + (e & 1) < nk;
          const float p = valid ? ex2(fmaf(s[nt][e], qs2, nl[half])) : 0.f;
          s[nt][e] = p * wr[half];                                // P w
          dp[nt][e] = p * fmaf(wr[half], dp[nt][e], -dr[half]);  // dS
        }
      }
      // dQ += dS K
      mma_keys_dims(dq, dp, ks_t, lane);
      // stage P w and dS as [head][key] (hi + lo) for the transposed products
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int r = gid + 8 * half;
          const uint32_t off = r * kPRowB + (8 * nt + 2 * tig) * 2;
          uint32_t hi, lo;
          split2(make_float2(s[nt][2 * half], s[nt][2 * half + 1]), hi, lo);
          *reinterpret_cast<uint32_t*>(sm.ph[w] + off) = hi;
          *reinterpret_cast<uint32_t*>(sm.pl[w] + off) = lo;
          split2(make_float2(dp[nt][2 * half], dp[nt][2 * half + 1]), hi, lo);
          *reinterpret_cast<uint32_t*>(sm.dh[w] + off) = hi;
          *reinterpret_cast<uint32_t*>(sm.dl[w] + off) = lo;
        }
      }
      __syncwarp();
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        if (16 * mt >= nk) break;
        float acc[8][4];
#pragma unroll
        for (int which = 0; which < 2; ++which) {  // 0: dK = dS^T Q, 1: dV = (P w)^T dO
          if (which == 0)
            mma_keys_heads(acc, sm.dh[w], sm.dl[w], qs_t, mt, lane);
          else
            mma_keys_heads(acc, sm.ph[w], sm.pl[w], ds_t, mt, lane);
          float* dst = which == 0 ? dk_out : dv_out;
          unsigned long long* fdst = which == 0 ? fk : fv;
          const float mul = which == 0 ? scale : 1.f;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int kk = 16 * mt + gid + 8 * half;
            const int tok = sm.tok[w][kk];
            if (kk < nk) {
              const int64_t off = ((int64_t)tok * hkv + g) * 64 + 2 * tig;
              if (fdst) {  // deterministic: 64-bit fixed-point sums
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  atomicAdd(fdst + off + 8 * i, (unsigned long long)__float2ll_rn(acc[i][2 * half] * mul * kFixScale));
                  atomicAdd(fdst + off + 8 * i + 1,
                            (unsigned long long)__float2ll_rn(acc[i][2 * half + 1] * mul * kFixScale));
                }
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  atomicAdd(reinterpret_cast<float2*>(dst + off + 8 * i),
                            make_float2(acc[i][2 * half] * mul, acc[i][2 * half + 1] * mul));
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = gid + 8 * half;
      if (r < G) {
        float* rowp = dq_out + (row0 + r) * 64 + 2 * tig;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float2 cur = *reinterpret_cast<float2*>(rowp + 8 * i);
          cur.x += dq[i][2 * half] * scale;
          cur.y += dq[i][2 * half + 1] * scale;
          *reinterpret_cast<float2*>(rowp + 8 * i) = cur;
        }
      }
    }
  }
}

int slc_grid(int64_t npairs) {
  const int64_t ctas = (npairs + kSlcWarps - 1) / kSlcWarps;
  const int64_t cap = (int64_t)tch::num_sms() * 16;
  return (int)(ctas < cap ? (ctas > 0 ? ctas : 1) : cap);
}

}  // namespace

bool slc_mma_supported(int dtype, int d, int hq, int hkv, int topk) {
  const int G = hkv > 0 ? hq / hkv : 0;
  return dtype == SSA_DTYPE_BF16 && d == 64 && (G == 8 || G == 16) && topk >= 1 && topk <= kSlcTopkMax;
}

cudaError_t slc_fwd_mma(const FwdArgs& a, cudaStream_t st) {
  const int G = a.hq / a.hkv;
  const int64_t rows = a.N * a.hq;
  const auto* q = static_cast<const __nv_bfloat16*>(a.q);
  const auto* ksp = static_cast<const __nv_bfloat16*>(a.ks);
  const auto* vsp = static_cast<const __nv_bfloat16*>(a.vs);
  float* o = static_cast<float*>(a.o_branch) + rows * 64;
  const int grid = slc_grid(a.N * a.hkv);
  const float qs2 = a.scale * kLog2e;
  if (G == 16)
    SSA_LAUNCH("slc_fwd_mma_kernel", slc_fwd_mma_kernel<16>, grid, 32 * kSlcWarps, 0, st, q, ksp, vsp, a.blk->ptr,
               a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, o, a.lse + rows);
  else
    SSA_LAUNCH("slc_fwd_mma_kernel", slc_fwd_mma_kernel<8>, grid, 32 * kSlcWarps, 0, st, q, ksp, vsp, a.blk->ptr,
               a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, o, a.lse + rows);
  return cudaGetLastError();
}

cudaError_t slc_bwd_mma(const BwdArgs& a, cudaStream_t st) {
  const int G = a.hq / a.hkv;
  const int64_t rows = a.N * a.hq;
  const auto* q = static_cast<const __nv_bfloat16*>(a.q);
  const auto* ksp = static_cast<const __nv_bfloat16*>(a.ks);
  const auto* vsp = static_cast<const __nv_bfloat16*>(a.vs);
  const auto* dO = static_cast<const __nv_bfloat16*>(a.dout);
  const int grid = slc_grid(a.N * a.hkv);
  const float qs2 = a.scale * kLog2e;
  const size_t smem = sizeof(SlcBwdSmem);
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(slc_bwd_mma_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(slc_bwd_mma_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr = true;
  }
  if (G == 16)
    SSA_LAUNCH("slc_bwd_mma_kernel", slc_bwd_mma_kernel<16>, grid, 32 * kSlcWarps, smem, st, q, ksp, vsp, dO,
               a.gates, a.gate_mode, a.blk->ptr, a.blk->perm, a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, a.scale,
               a.lse + rows, a.Dc + rows, a.dq, a.dk, a.dv, a.fx_k, a.fx_v);
  else
    SSA_LAUNCH("slc_bwd_mma_kernel", slc_bwd_mma_kernel<8>, grid, 32 * kSlcWarps, smem, st, q, ksp, vsp, dO,
               a.gates, a.gate_mode, a.blk->ptr, a.blk->perm, a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, a.scale,
               a.lse + rows, a.Dc + rows, a.dq, a.dk, a.dv, a.fx_k, a.fx_v);
  return cudaGetLastError();
}

}  // namespace ssa
