// Steps 3-7 of SSA as fp32 SIMT kernels (FFMA): compressed attention + top-k
// selection, selected-block attention, window attention, gated combine and the
// backward of all three branches.
//
// Direct3D-S2 (hyper.ai, "方法"): queries attend to the compressed blocks; the
// top-k blocks by that attention score get a second, full attention over their
// tokens; a third attention runs inside non-overlapping m_win^3 windows; the
// three outputs are summed with predicted gate weights.  The selection score of
// a block is its softmax probability summed over the query heads of a GQA group
// (LSRM, shuwu5.cn, "阶段一": grouped-query attention with 2 KV heads).
//
// These kernels serve the fp32 configuration (which needs true fp32 math) and
// every shape the tensor-core kernels do not cover.  Layout: NT = D/32 adjacent
// lanes own one query row (32 dims each); keys/values are staged in shared
// memory as fp32 with a 4-float pad between 32-dim sub-rows (no bank conflicts
// between the NT sub-lanes).  Softmax runs in the log2 domain (q pre-scaled by
// scale * log2(e)); stored lse values are natural logs.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

template <int D>
struct Cfg {
  static constexpr int NT = D / 32;          // lanes per row
  static constexpr int THREADS = 128;
  static constexpr int ROWS = THREADS / NT;  // rows per CTA
  static constexpr int KSTR = NT * 36;       // floats per staged row
};

__device__ __forceinline__ float4 load4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
}

// Stage n rows of D elements into shared memory (fp32, padded sub-rows).
template <typename T, int D, typename F>
__device__ __forceinline__ void stage_rows(float* dst, int n, F src, float mul = 1.f) {
  constexpr int QPR = D / 4;
  for (int idx = threadIdx.x; idx < n * QPR; idx += blockDim.x) {
    const int j = idx / QPR, qd = idx % QPR;
    float4 v = load4(src(j) + qd * 4);
    v.x *= mul;
    v.y *= mul;
    v.z *= mul;
    v.w *= mul;
    *reinterpret_cast<float4*>(dst + j * Cfg<D>::KSTR + (qd >> 3) * 36 + (qd & 7) * 4) = v;
  }
}

__device__ __forceinline__ float dot32(const float* a, const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 k = r4[i];
    acc = fmaf(a[4 * i + 0], k.x, acc);
    acc = fmaf(a[4 * i + 1], k.y, acc);
    acc = fmaf(a[4 * i + 2], k.z, acc);
    acc = fmaf(a[4 * i + 3], k.w, acc);
  }
  return acc;
}

__device__ __forceinline__ float dot32r(const float* a, const float* b) {
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) acc = fmaf(a[i], b[i], acc);
  return acc;
}

__device__ __forceinline__ void axpy32(float* y, float a, const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 k = r4[i];
    y[4 * i + 0] = fmaf(a, k.x, y[4 * i + 0]);
    y[4 * i + 1] = fmaf(a, k.y, y[4 * i + 1]);
    y[4 * i + 2] = fmaf(a, k.z, y[4 * i + 2]);
    y[4 * i + 3] = fmaf(a, k.w, y[4 * i + 3]);
  }
}

template <int NT>
__device__ __forceinline__ float row_sum(float x, unsigned mask) {
  if (NT >= 2) x += __shfl_xor_sync(mask, x, 1);
  if (NT >= 4) x += __shfl_xor_sync(mask, x, 2);
  return x;
}

__device__ __forceinline__ float gate_weight(const float* gates, int64_t idx, int mode) {
  const float x = gates[idx];
  return mode == SSA_GATE_LOGITS ? 1.f / (1.f + expf(-x)) : x;
}

// ---------------------------------------------------------------------------
// compressed branch, pass 1: lse over all blocks of the query's sequence
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) cmp_lse_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                                                      const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu,
                                                      const int32_t* __restrict__ tpre, int S, int hq, int hkv,
                                                      int64_t btot, float qs2, float* __restrict__ lse_out) {
  using C = Cfg<D>;
  constexpr int KT = 64;
  __shared__ __align__(16) float sk[KT * C::KSTR];
  const int g = blockIdx.y, G = hq / hkv;
  const int r = threadIdx.x / C::NT, sub = threadIdx.x % C::NT;
  const int ntiles = tpre[S];
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int s = find_segment(tpre, S, tile);
    const int64_t nrows = (int64_t)(cu[s + 1] - cu[s]) * G;
    const int64_t gr = (int64_t)(tile - tpre[s]) * C::ROWS + r;
    const bool valid = gr < nrows;
    const int64_t t = cu[s] + (valid ? gr / G : 0);
    const int h = g * G + (valid ? (int)(gr % G) : 0);
    float qv[32];
    load32(q + (t * hq + h) * D + sub * 32, qv);
#pragma unroll
    for (int i = 0; i < 32; ++i) qv[i] *= qs2;
    float m = -CUDART_INF_F, l = 0.f;
    const int b0 = bcu[s], nb = bcu[s + 1] - b0;
    for (int c0 = 0; c0 < nb; c0 += KT) {
      const int kn = min(KT, nb - c0);
      __syncthreads();
      stage_rows<T, D>(sk, kn, [&](int j) { return kc + ((int64_t)g * btot + b0 + c0 + j) * D; });
      __syncthreads();
      for (int j0 = 0; j0 < kn; j0 += 16) {
        float sc[16];
        float cm = -CUDART_INF_F;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          float x = -CUDART_INF_F;
          if (j0 + jj < kn) x = row_sum<C::NT>(dot32(qv, sk + (j0 + jj) * C::KSTR + sub * 36), 0xffffffffu);
          sc[jj] = x;
          cm = fmaxf(cm, x);
        }
        const float mn = fmaxf(m, cm);
        l *= exp2f(m - mn);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) l += exp2f(sc[jj] - mn);
        m = mn;
      }
    }
    if (valid && sub == 0) lse_out[t * hq + h] = (m + log2f(l)) * kLn2;
  }
}

// ---------------------------------------------------------------------------
// compressed branch, pass 2: output with the final lse + top-k block selection
// ---------------------------------------------------------------------------
constexpr int kTopkMax = 32;

__device__ __forceinline__ int find_worst(const float* v, const int* id, int n) {
  int w = 0;
  for (int i = 1; i < n; ++i)
    if (v[i] < v[w] || (v[i] == v[w] && id[i] > id[w])) w = i;
  return w;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) cmp_out_topk_kernel(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc, const int32_t* __restrict__ cu,
    const int32_t* __restrict__ bcu, const int32_t* __restrict__ tpre, int S, int hq, int hkv, int64_t btot,
    float qs2, const float* __restrict__ lse_in, float* __restrict__ o_out, int topk, int32_t* __restrict__ sel) {
  using C = Cfg<D>;
  constexpr int KT = 32;
  __shared__ __align__(16) float sk[KT * C::KSTR];
  __shared__ __align__(16) float sv[KT * C::KSTR];
  __shared__ float tv[C::ROWS][kTopkMax];
  __shared__ int ti[C::ROWS][kTopkMax];
  const int g = blockIdx.y, G = hq / hkv;
  const int r = threadIdx.x / C::NT, sub = threadIdx.x % C::NT;
  const int tok = r / G;
  const bool leader = (r % G == 0) && sub == 0;
  const int ntiles = tpre[S];
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int s = find_segment(tpre, S, tile);
    const int64_t nrows = (int64_t)(cu[s + 1] - cu[s]) * G;
    const int64_t gr = (int64_t)(tile - tpre[s]) * C::ROWS + r;
    const bool valid = gr < nrows;
    const int64_t t = cu[s] + (valid ? gr / G : 0);
    const int h = g * G + (valid ? (int)(gr % G) : 0);
    float qv[32], o[32];
    load32(q + (t * hq + h) * D + sub * 32, qv);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      qv[i] *= qs2;
      o[i] = 0.f;
    }
    const float lse2 = lse_in[t * hq + h] * kLog2e;
    const int b0 = bcu[s], nb = bcu[s + 1] - b0;
    const int keff = min(topk, nb);
    int cnt = 0, worst = 0;
    for (int c0 = 0; c0 < nb; c0 += KT) {
      const int kn = min(KT, nb - c0);
      __syncthreads();
      stage_rows<T, D>(sk, kn, [&](int j) { return kc + ((int64_t)g * btot + b0 + c0 + j) * D; });
      stage_rows<T, D>(sv, kn, [&](int j) { return vc + ((int64_t)g * btot + b0 + c0 + j) * D; });
      __syncthreads();
      for (int j = 0; j < kn; ++j) {
        const float s2 = row_sum<C::NT>(dot32(qv, sk + j * C::KSTR + sub * 36), 0xffffffffu);
        const float p = exp2f(s2 - lse2);
        axpy32(o, p, sv + j * C::KSTR + sub * 36);
        float imp = p;
        for (int off = C::NT; off < G * C::NT; off <<= 1) imp += __shfl_xor_sync(0xffffffffu, imp, off);
        if (leader && valid && sel) {
          const int bid = b0 + c0 + j;
          if (cnt < keff) {
            tv[tok][cnt] = imp;
            ti[tok][cnt] = bid;
            ++cnt;
            if (cnt == keff) worst = find_worst(tv[tok], ti[tok], keff);
          } else if (imp > tv[tok][worst]) {
            tv[tok][worst] = imp;
            ti[tok][worst] = bid;
            worst = find_worst(tv[tok], ti[tok], keff);
          }
        }
      }
    }
    if (valid) {
      store32(o_out + (t * hq + h) * D + sub * 32, o);
      if (leader && sel) {
        int* ids = ti[tok];
        for (int i = 1; i < keff; ++i) {  // insertion sort, ascending ids
          const int x = ids[i];
          int j = i - 1;
          while (j >= 0 && ids[j] > x) {
            ids[j + 1] = ids[j];
            --j;
          }
          ids[j + 1] = x;
        }
        int32_t* out = sel + (t * hkv + g) * topk;
        for (int i = 0; i < topk; ++i) out[i] = i < keff ? ids[i] : -1;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// selected-block attention: per (token, group), all tokens of the selected blocks
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) slc_fwd_kernel(const T* __restrict__ q, const T* __restrict__ ks,
                                                      const T* __restrict__ vs, const int32_t* __restrict__ bptr,
                                                      const int32_t* __restrict__ sel, int64_t N, int64_t ldk,
                                                      int hq, int hkv, int topk, float qs2, float* __restrict__ o_out,
                                                      float* __restrict__ lse_out) {
  constexpr int NT = D / 32;
  const int G = hq / hkv, GT = G * NT, PPC = 128 / GT;
  const int lane = threadIdx.x & 31;
  const unsigned gmask = GT >= 32 ? 0xffffffffu : (((1u << GT) - 1u) << (lane & ~(GT - 1)));
  const int r = (threadIdx.x % GT) / NT, sub = threadIdx.x % NT;
  const int64_t npairs = N * hkv;
  for (int64_t pair = (int64_t)blockIdx.x * PPC + threadIdx.x / GT; pair < npairs; pair += (int64_t)gridDim.x * PPC) {
    const int64_t t = pair / hkv;
    const int g = (int)(pair % hkv), h = g * G + r;
    float qv[32], o[32];
    load32(q + (t * hq + h) * D + sub * 32, qv);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      qv[i] *= qs2;
      o[i] = 0.f;
    }
    float m = -CUDART_INF_F, l = 0.f;
    const int32_t* srow = sel + pair * topk;
    for (int si = 0; si < topk; ++si) {
      const int b = srow[si];
      if (b < 0) continue;
      const int p1 = bptr[b + 1];
      for (int j0 = bptr[b]; j0 < p1; j0 += 8) {
        float sc[8];
        float cm = -CUDART_INF_F;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          float x = -CUDART_INF_F;
          if (j0 + jj < p1) {
            float kv[32];
            load32(ks + ((int64_t)g * ldk + j0 + jj) * D + sub * 32, kv);
            x = row_sum<NT>(dot32r(qv, kv), gmask);
          }
          sc[jj] = x;
          cm = fmaxf(cm, x);
        }
        const float mn = fmaxf(m, cm);
        const float corr = exp2f(m - mn);
        l *= corr;
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= corr;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          if (j0 + jj < p1) {
            const float p = exp2f(sc[jj] - mn);
            l += p;
            float vv[32];
            load32(vs + ((int64_t)g * ldk + j0 + jj) * D + sub * 32, vv);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = fmaf(p, vv[i], o[i]);
          }
        }
        m = mn;
      }
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] *= inv;
    store32(o_out + (t * hq + h) * D + sub * 32, o);
    if (sub == 0) lse_out[t * hq + h] = (m + log2f(l)) * kLn2;
  }
}

// ---------------------------------------------------------------------------
// window attention: per (window, group), every token of the window
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) win_fwd_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                      const T* __restrict__ v, const int32_t* __restrict__ wperm,
                                                      const int32_t* __restrict__ wptr, int64_t wtot, int hq, int hkv,
                                                      float qs2, float* __restrict__ o_out, float* __restrict__ lse_out) {
  using C = Cfg<D>;
  constexpr int KT = D >= 128 ? 32 : 64;  // staged keys per chunk (two chunks of K and V fit 48 KB)
  __shared__ __align__(16) float sk[KT * C::KSTR];
  __shared__ __align__(16) float sv[KT * C::KSTR];
  const int g = blockIdx.y, G = hq / hkv;
  const int r = threadIdx.x / C::NT, sub = threadIdx.x % C::NT;
  for (int64_t w = blockIdx.x; w < wtot; w += gridDim.x) {
    const int p0 = wptr[w], nw = wptr[w + 1] - p0;
    const int nrows = nw * G;
    const int nchunks = (nw + KT - 1) / KT;
    for (int row0 = 0; row0 < nrows; row0 += C::ROWS) {
      const int rr = row0 + r;
      const bool valid = rr < nrows;
      const int64_t t = wperm[p0 + (valid ? rr / G : 0)];
      const int h = g * G + (valid ? rr % G : 0);
      float qv[32], o[32];
      load32(q + (t * hq + h) * D + sub * 32, qv);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        qv[i] *= qs2;
        o[i] = 0.f;
      }
      float m = -CUDART_INF_F, l = 0.f;
      for (int c = 0; c < nchunks; ++c) {
        const int kn = min(KT, nw - c * KT);
        if (nchunks > 1 || row0 == 0) {
          __syncthreads();
          stage_rows<T, D>(sk, kn, [&](int j) { return k + ((int64_t)wperm[p0 + c * KT + j] * hkv + g) * D; });
          stage_rows<T, D>(sv, kn, [&](int j) { return v + ((int64_t)wperm[p0 + c * KT + j] * hkv + g) * D; });
          __syncthreads();
        }
        for (int j0 = 0; j0 < kn; j0 += 16) {
          float sc[16];
          float cm = -CUDART_INF_F;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            float x = -CUDART_INF_F;
            if (j0 + jj < kn) x = row_sum<C::NT>(dot32(qv, sk + (j0 + jj) * C::KSTR + sub * 36), 0xffffffffu);
            sc[jj] = x;
            cm = fmaxf(cm, x);
          }
          const float mn = fmaxf(m, cm);
          const float corr = exp2f(m - mn);
          l *= corr;
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            if (j0 + jj < kn) {
              const float p = exp2f(sc[jj] - mn);
              l += p;
              axpy32(o, p, sv + (j0 + jj) * C::KSTR + sub * 36);
            }
          }
          m = mn;
        }
      }
      if (valid) {
        const float inv = 1.f / l;
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= inv;
        store32(o_out + (t * hq + h) * D + sub * 32, o);
        if (sub == 0) lse_out[t * hq + h] = (m + log2f(l)) * kLn2;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// gated combine: out = sum_c w_c * o_c
// ---------------------------------------------------------------------------
// The combine streams the [3, rows, D] branch outputs as one contiguous range: a warp
// takes 256 consecutive float4 slots (16 rows of 64 or 32 rows of 32), lane t the
// slots t, t + 32, ..., so each load instruction of the warp reads 512 contiguous
// bytes (a lane owning 128 contiguous bytes instead makes every instruction touch 32
// lines, and the L1 wavefront rate, not HBM, sets the pace).  The branch outputs are
// read once: streaming loads.
constexpr int kSlotsPerWarp = 256;

__device__ __forceinline__ float4 ldcs4(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void store4(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// out = sum_c w_c o_c over the nbr branches (per row; w = gate weights)
template <typename T, int D>
__global__ void combine_kernel(const float* __restrict__ ob, const float* __restrict__ gates, int64_t rows, int mode,
                               int nbr, T* __restrict__ out) {
  const int64_t total4 = rows * (D / 4);
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t chunk = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; chunk * kSlotsPerWarp < total4;
       chunk += nwarps) {
    float4 x[3][8];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      if (c >= nbr) break;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t sl = chunk * kSlotsPerWarp + i * 32 + lane;
        x[c][i] = sl < total4 ? ldcs4(ob + ((int64_t)c * total4 + sl) * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t sl = chunk * kSlotsPerWarp + i * 32 + lane;
      if (sl >= total4) continue;
      const int64_t row = sl / (D / 4);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (c >= nbr) break;
        const float w = gate_weight(gates, row * 3 + c, mode);
        acc[0] = fmaf(w, x[c][i].x, acc[0]);
        acc[1] = fmaf(w, x[c][i].y, acc[1]);
        acc[2] = fmaf(w, x[c][i].z, acc[2]);
        acc[3] = fmaf(w, x[c][i].w, acc[3]);
      }
      store4(out + sl * 4, acc);
    }
  }
}

// ---------------------------------------------------------------------------
// backward: per-row dot products <dO, o_c>, the softmax correction D_c and dgates
// ---------------------------------------------------------------------------
// Also writes the per-row constants of the tensor-core kernels (rc, [2][3][rows]):
// for the compressed (c = 0) and window (c = 2) branches, -lse * log2(e), w and -D.
// Access as in the combine, with 128 float4 slots per warp pass (4 per lane, to keep
// the live registers low enough for 16+ warps per SM): a row's D / 4 slots sit in D / 4
// consecutive lanes; their partial dot products are summed across those lanes, and
// then lane L collects row L of the pass so that the per-row outputs are contiguous.
constexpr int kPreSlots = 4;  // float4 slots per lane per pass

__device__ __forceinline__ void load4s(const float* p, float* o) {
  const float4 v = __ldcs(reinterpret_cast<const float4*>(p));
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4s(const __nv_bfloat16* p, float* o) {
  const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
  o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
  o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
}

template <typename T, int D>
__global__ void bwd_pre_kernel(const float* __restrict__ ob, const T* __restrict__ dout, const float* __restrict__ gates,
                               const float* __restrict__ lse, int64_t rows, int mode, int nbr, float* __restrict__ Dc,
                               float* __restrict__ dgates, float* __restrict__ rc) {
  constexpr int LPR = D / 4;      // lanes per row
  constexpr int RPI = 32 / LPR;   // rows per slot index
  constexpr int SPW = 32 * kPreSlots;  // slots per warp pass
  const int64_t total4 = rows * LPR;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t chunk = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; chunk * SPW < total4; chunk += nwarps) {
    float dov[kPreSlots][4];
    float4 x[3][kPreSlots];
#pragma unroll
    for (int i = 0; i < kPreSlots; ++i) {
      const int64_t sl = chunk * SPW + i * 32 + lane;
      if (sl < total4) {
        load4s(dout + sl * 4, dov[i]);
      } else {
        dov[i][0] = dov[i][1] = dov[i][2] = dov[i][3] = 0.f;
      }
    }
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      if (c >= nbr) break;
#pragma unroll
      for (int i = 0; i < kPreSlots; ++i) {
        const int64_t sl = chunk * SPW + i * 32 + lane;
        x[c][i] = sl < total4 ? __ldcs(reinterpret_cast<const float4*>(ob + ((int64_t)c * total4 + sl) * 4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const int my_i = lane / RPI, src = LPR * (lane % RPI);
    float mine[3] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 3; ++c) {
#pragma unroll
      for (int i = 0; i < kPreSlots; ++i) {
        float dot = 0.f;
        if (c < nbr)
          dot = dov[i][0] * x[c][i].x + dov[i][1] * x[c][i].y + dov[i][2] * x[c][i].z + dov[i][3] * x[c][i].w;
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float t = __shfl_sync(0xffffffffu, dot, src);
        if (i == my_i) mine[c] = t;
      }
    }
    const int64_t row = chunk * (SPW / LPR) + lane;
    if (lane < kPreSlots * RPI && row < rows) {
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (c >= nbr) break;
        const float w = gate_weight(gates, row * 3 + c, mode);
        const float dot = mine[c];
        Dc[(int64_t)c * rows + row] = w * dot;
        dgates[row * nbr + c] = mode == SSA_GATE_LOGITS ? dot * w * (1.f - w) : dot;
        if (c != 1) {
          float* r = rc + (c == 0 ? 0 : 3 * rows);
          r[row] = -lse[(int64_t)c * rows + row] * kLog2e;
          r[rows + row] = w;
          r[2 * rows + row] = -(w * dot);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// compressed branch backward: dQ (query-major)
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) cmp_bwd_dq_kernel(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu,
    const int32_t* __restrict__ tpre, int S, int hq, int hkv, int64_t btot, float qs2, float scale,
    const float* __restrict__ lse_in, const float* __restrict__ Dc, float* __restrict__ dq_out) {
  using C = Cfg<D>;
  constexpr int KT = 32;
  __shared__ __align__(16) float sk[KT * C::KSTR];
  __shared__ __align__(16) float sv[KT * C::KSTR];
  const int g = blockIdx.y, G = hq / hkv;
  const int r = threadIdx.x / C::NT, sub = threadIdx.x % C::NT;
  const int ntiles = tpre[S];
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int s = find_segment(tpre, S, tile);
    const int64_t nrows = (int64_t)(cu[s + 1] - cu[s]) * G;
    const int64_t gr = (int64_t)(tile - tpre[s]) * C::ROWS + r;
    const bool valid = gr < nrows;
    const int64_t t = cu[s] + (valid ? gr / G : 0);
    const int h = g * G + (valid ? (int)(gr % G) : 0);
    const int64_t row = t * hq + h;
    float qv[32], dov[32], dq[32];
    load32(q + row * D + sub * 32, qv);
    load32(dout + row * D + sub * 32, dov);
    const float wg = gate_weight(gates, row * 3 + 0, mode);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      qv[i] *= qs2;
      dov[i] *= wg;
      dq[i] = 0.f;
    }
    const float lse2 = lse_in[row] * kLog2e;
    const float Dr = Dc[row];
    const int b0 = bcu[s], nb = bcu[s + 1] - b0;
    for (int c0 = 0; c0 < nb; c0 += KT) {
      const int kn = min(KT, nb - c0);
      __syncthreads();
      stage_rows<T, D>(sk, kn, [&](int j) { return kc + ((int64_t)g * btot + b0 + c0 + j) * D; });
      stage_rows<T, D>(sv, kn, [&](int j) { return vc + ((int64_t)g * btot + b0 + c0 + j) * D; });
      __syncthreads();
      for (int j = 0; j < kn; ++j) {
        const float* krow = sk + j * C::KSTR + sub * 36;
        const float s2 = row_sum<C::NT>(dot32(qv, krow), 0xffffffffu);
        const float p = exp2f(s2 - lse2);
        const float dp = row_sum<C::NT>(dot32(dov, sv + j * C::KSTR + sub * 36), 0xffffffffu);
        axpy32(dq, p * (dp - Dr), krow);
      }
    }
    if (valid) {
#pragma unroll
      for (int i = 0; i < 32; ++i) dq[i] *= scale;
      store32(dq_out + row * D + sub * 32, dq);
    }
  }
}

// ---------------------------------------------------------------------------
// Shared key-major backward core: a CTA owns KPC keys (k, v rows in registers)
// and streams query rows through shared memory, accumulating dk, dv.
// ---------------------------------------------------------------------------
template <typename T, int D>
struct RowStage {
  static constexpr int RT = 16;  // rows per stage
  float q[RT * Cfg<D>::KSTR];
  float dO[RT * Cfg<D>::KSTR];
  float lse2[RT];
  float Dr[RT];
};

// Stage rows [r0, r0+n) where row index -> (global q/dO row, lse index) via `map`.
// map(i, &row, &ok): row = token*hq + head of staged row i.
template <typename T, int D, typename MAP>
__device__ __forceinline__ void stage_query_rows(RowStage<T, D>& st, int n, MAP map, const T* q, const T* dout,
                                                 const float* gates, int mode, int branch, const float* lse_b,
                                                 const float* Dc_b) {
  constexpr int QPR = D / 4;
  for (int idx = threadIdx.x; idx < RowStage<T, D>::RT * QPR; idx += blockDim.x) {
    const int i = idx / QPR, qd = idx % QPR;
    int64_t row = 0;
    bool ok = i < n && map(i, &row);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (ok) {
      a = load4(q + row * D + qd * 4);
      b = load4(dout + row * D + qd * 4);
      const float w = gate_weight(gates, row * 3 + branch, mode);
      b.x *= w;
      b.y *= w;
      b.z *= w;
      b.w *= w;
    }
    const int off = i * Cfg<D>::KSTR + (qd >> 3) * 36 + (qd & 7) * 4;
    *reinterpret_cast<float4*>(st.q + off) = a;
    *reinterpret_cast<float4*>(st.dO + off) = b;
    if (qd == 0) {
      st.lse2[i] = ok ? lse_b[row] * kLog2e : CUDART_INF_F;
      st.Dr[i] = ok ? Dc_b[row] : 0.f;
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void accumulate_rows(const RowStage<T, D>& st, const float* kv, const float* vv, float qs2,
                                                float* dk, float* dv) {
  constexpr int NT = D / 32;
  const int sub = threadIdx.x % NT;
#pragma unroll 2
  for (int i = 0; i < RowStage<T, D>::RT; ++i) {
    const float* qrow = st.q + i * Cfg<D>::KSTR + sub * 36;
    const float* drow = st.dO + i * Cfg<D>::KSTR + sub * 36;
    const float s2 = row_sum<NT>(dot32(kv, qrow), 0xffffffffu) * qs2;
    const float p = exp2f(s2 - st.lse2[i]);
    const float dp = row_sum<NT>(dot32(vv, drow), 0xffffffffu);
    const float ds = p * (dp - st.Dr[i]);
    axpy32(dk, ds, qrow);
    axpy32(dv, p, drow);
  }
}

// compressed branch: dKc, dVc (atomic fp32 accumulation across row chunks)
template <typename T, int D>
__global__ void __launch_bounds__(128) cmp_bwd_dkv_kernel(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu,
    const int32_t* __restrict__ ipre, int S, int hq, int hkv, int64_t btot, float qs2, float scale, int rc_rows,
    const float* __restrict__ lse_in, const float* __restrict__ Dc, float* __restrict__ dkc, float* __restrict__ dvc) {
  using C = Cfg<D>;
  __shared__ __align__(16) RowStage<T, D> st;
  const int g = blockIdx.y, G = hq / hkv;
  const int sub = threadIdx.x % C::NT;
  const int nitems = ipre[S];
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int s = find_segment(ipre, S, item);
    const int b0 = bcu[s], nb = bcu[s + 1] - b0;
    const int nbt = (nb + C::ROWS - 1) / C::ROWS;
    const int local = item - ipre[s];
    const int bt = local % nbt, rc = local / nbt;
    const int j = bt * C::ROWS + threadIdx.x / C::NT;
    const bool validb = j < nb;
    const int64_t bidx = (int64_t)g * btot + b0 + (validb ? j : 0);
    float kv[32], vv[32], dk[32], dv[32];
    load32(kc + bidx * D + sub * 32, kv);
    load32(vc + bidx * D + sub * 32, vv);
#pragma unroll
    for (int i = 0; i < 32; ++i) dk[i] = dv[i] = 0.f;
    const int64_t nrows = (int64_t)(cu[s + 1] - cu[s]) * G;
    const int64_t r0 = (int64_t)rc * rc_rows;
    const int64_t r1 = min(nrows, r0 + rc_rows);
    for (int64_t rs = r0; rs < r1; rs += RowStage<T, D>::RT) {
      const int n = (int)min((int64_t)RowStage<T, D>::RT, r1 - rs);
      __syncthreads();
      stage_query_rows<T, D>(
          st, n,
          [&](int i, int64_t* row) {
            const int64_t gr = rs + i;
            *row = (cu[s] + gr / G) * hq + g * G + gr % G;
            return true;
          },
          q, dout, gates, mode, 0, lse_in, Dc);
      __syncthreads();
      accumulate_rows<T, D>(st, kv, vv, qs2, dk, dv);
    }
    if (validb) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        atomicAdd(dkc + bidx * D + sub * 32 + i, dk[i] * scale);
        atomicAdd(dvc + bidx * D + sub * 32 + i, dv[i]);
      }
    }
  }
}

// selected branch: dQ (query-major, like the forward)
template <typename T, int D>
__global__ void __launch_bounds__(128) slc_bwd_dq_kernel(
    const T* __restrict__ q, const T* __restrict__ ks, const T* __restrict__ vs, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ bptr, const int32_t* __restrict__ sel,
    int64_t N, int64_t ldk, int hq, int hkv, int topk, float qs2, float scale, const float* __restrict__ lse_in,
    const float* __restrict__ Dc, float* __restrict__ dq_out) {
  constexpr int NT = D / 32;
  const int G = hq / hkv, GT = G * NT, PPC = 128 / GT;
  const int lane = threadIdx.x & 31;
  const unsigned gmask = GT >= 32 ? 0xffffffffu : (((1u << GT) - 1u) << (lane & ~(GT - 1)));
  const int r = (threadIdx.x % GT) / NT, sub = threadIdx.x % NT;
  const int64_t npairs = N * hkv;
  for (int64_t pair = (int64_t)blockIdx.x * PPC + threadIdx.x / GT; pair < npairs; pair += (int64_t)gridDim.x * PPC) {
    const int64_t t = pair / hkv;
    const int g = (int)(pair % hkv), h = g * G + r;
    const int64_t row = t * hq + h;
    float qv[32], dov[32], dq[32];
    load32(q + row * D + sub * 32, qv);
    load32(dout + row * D + sub * 32, dov);
    const float wg = gate_weight(gates, row * 3 + 1, mode);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      qv[i] *= qs2;
      dov[i] *= wg;
      dq[i] = 0.f;
    }
    const float lse2 = lse_in[row] * kLog2e;
    const float Dr = Dc[row];
    const int32_t* srow = sel + pair * topk;
    for (int si = 0; si < topk; ++si) {
      const int b = srow[si];
      if (b < 0) continue;
      const int p1 = bptr[b + 1];
      for (int j = bptr[b]; j < p1; ++j) {
        float kv[32], vv[32];
        load32(ks + ((int64_t)g * ldk + j) * D + sub * 32, kv);
        load32(vs + ((int64_t)g * ldk + j) * D + sub * 32, vv);
        const float s2 = row_sum<NT>(dot32r(qv, kv), gmask);
        const float p = exp2f(s2 - lse2);
        const float dp = row_sum<NT>(dot32r(dov, vv), gmask);
        const float ds = p * (dp - Dr);
#pragma unroll
        for (int i = 0; i < 32; ++i) dq[i] = fmaf(ds, kv[i], dq[i]);
      }
    }
    float* dst = dq_out + row * D + sub * 32;
#pragma unroll
    for (int i = 0; i < 32; ++i) dst[i] += dq[i] * scale;
  }
}

// selected branch: dK, dV per block, over the (token, group) pairs that selected it.
// A work item is (group g, block b, chunk of kSlcRowChunk rows of the pairs that
// selected b).  Threads split as (key slot, row slice): small blocks (the common
// case, 1-2 tokens) use many row slices, large blocks many key slots.  Partial
// dk/dv are reduced over row slices in shared memory and added to dK/dV (zeroed
// beforehand) with fp32 atomics.
constexpr int kSlcRowChunk = 1024;
// staged query rows per pass (the q / dO stages of head dim 128 would not fit 48 KB at 64)
template <int D>
constexpr int slc_stage_rows() { return D >= 128 ? 32 : 64; }

template <typename T, int D>
struct SlcStage {
  float q[slc_stage_rows<D>() * Cfg<D>::KSTR];
  float dO[slc_stage_rows<D>() * Cfg<D>::KSTR];
  float lse2[slc_stage_rows<D>()];
  float Dr[slc_stage_rows<D>()];
};

__global__ void slc_items_kernel(const int32_t* __restrict__ inv_ptr, int64_t nkeys, int G, int32_t* __restrict__ cnt) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i <= nkeys; i += (int64_t)gridDim.x * blockDim.x) {
    if (i == nkeys) {
      cnt[i] = 0;
      continue;
    }
    const int64_t rows = (int64_t)(inv_ptr[i + 1] - inv_ptr[i]) * G;
    cnt[i] = (int32_t)((rows + kSlcRowChunk - 1) / kSlcRowChunk);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(128) slc_bwd_dkv_kernel(
    const T* __restrict__ q, const T* __restrict__ ks, const T* __restrict__ vs, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ bptr, const int32_t* __restrict__ bperm,
    const int32_t* __restrict__ inv_ptr, const int32_t* __restrict__ inv_tok, const int32_t* __restrict__ ipre,
    int64_t ldk, int64_t btot, int hq, int hkv, float qs2, float scale, const float* __restrict__ lse_in,
    const float* __restrict__ Dc, float* __restrict__ dk_out, float* __restrict__ dv_out) {
  constexpr int NT = D / 32;
  constexpr int SLOTS = 128 / NT;  // (key slot, row slice) pairs
  __shared__ __align__(16) SlcStage<T, D> st;
  constexpr int kSlcStageRows = slc_stage_rows<D>();
  constexpr int KMAX = D >= 128 ? 32 : 64;  // key slots per pass (the reduction buffers hold KMAX * D floats each)
  static_assert(kSlcStageRows * Cfg<D>::KSTR >= KMAX * D, "reduction buffers must fit in the staging area");
  const int G = hq / hkv;
  const int sub = threadIdx.x % NT;
  const int pair_id = threadIdx.x / NT;
  const int64_t nkeys = (int64_t)hkv * btot;
  const int nitems = ipre[nkeys];
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int64_t key = find_segment(ipre, (int)nkeys, item);  // g * btot + b
    const int g = (int)(key / btot);
    const int64_t b = key % btot;
    const int chunk = item - ipre[key];
    const int l0 = inv_ptr[key];
    const int64_t nrows_all = (int64_t)(inv_ptr[key + 1] - l0) * G;
    const int64_t r0 = (int64_t)chunk * kSlcRowChunk;
    const int64_t r1 = min(nrows_all, r0 + kSlcRowChunk);
    const int p0 = bptr[b], nb = bptr[b + 1] - p0;
    int kpc = 1;
    while (kpc < nb && kpc < KMAX) kpc <<= 1;
    const int rs = SLOTS / kpc;
    const int kslot = pair_id % kpc, rslice = pair_id / kpc;
    for (int kp = 0; kp < nb; kp += kpc) {
      const int j = kp + kslot;
      const bool validk = j < nb;
      const int64_t kidx = (int64_t)g * ldk + p0 + (validk ? j : 0);
      float kv[32], vv[32], dk[32], dv[32];
      load32(ks + kidx * D + sub * 32, kv);
      load32(vs + kidx * D + sub * 32, vv);
#pragma unroll
      for (int i = 0; i < 32; ++i) dk[i] = dv[i] = 0.f;
      for (int64_t rsb = r0; rsb < r1; rsb += kSlcStageRows) {
        const int n = (int)min((int64_t)kSlcStageRows, r1 - rsb);
        __syncthreads();
        constexpr int QPR = D / 4;
        for (int idx = threadIdx.x; idx < kSlcStageRows * QPR; idx += blockDim.x) {
          const int i = idx / QPR, qd = idx % QPR;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
          int64_t row = 0;
          const bool ok = i < n;
          if (ok) {
            const int64_t gr = rsb + i;
            row = (int64_t)inv_tok[l0 + gr / G] * hq + g * G + gr % G;
            a = load4(q + row * D + qd * 4);
            c = load4(dout + row * D + qd * 4);
            const float w = gate_weight(gates, row * 3 + 1, mode);
            c.x *= w;
            c.y *= w;
            c.z *= w;
            c.w *= w;
          }
          const int off = i * Cfg<D>::KSTR + (qd >> 3) * 36 + (qd & 7) * 4;
          *reinterpret_cast<float4*>(st.q + off) = a;
          *reinterpret_cast<float4*>(st.dO + off) = c;
          if (qd == 0) {
            st.lse2[i] = ok ? lse_in[row] * kLog2e : CUDART_INF_F;
            st.Dr[i] = ok ? Dc[row] : 0.f;
          }
        }
        __syncthreads();
        for (int i = rslice; i < kSlcStageRows; i += rs) {
          const float* qrow = st.q + i * Cfg<D>::KSTR + sub * 36;
          const float* drow = st.dO + i * Cfg<D>::KSTR + sub * 36;
          const float s2 = row_sum<NT>(dot32(kv, qrow), 0xffffffffu) * qs2;
          const float p = exp2f(s2 - st.lse2[i]);
          const float dp = row_sum<NT>(dot32(vv, drow), 0xffffffffu);
          const float ds = p * (dp - st.Dr[i]);
          axpy32(dk, ds, qrow);
          axpy32(dv, p, drow);
        }
      }
      // reduce over row slices (in the staging area, now free), then one atomic
      // add per (key, dim)
      float* red_k = st.q;
      float* red_v = st.dO;
      __syncthreads();
      for (int i = threadIdx.x; i < kpc * D; i += blockDim.x) {
        red_k[i] = 0.f;
        red_v[i] = 0.f;
      }
      __syncthreads();
      if (validk) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          atomicAdd(&red_k[kslot * D + sub * 32 + i], dk[i]);
          atomicAdd(&red_v[kslot * D + sub * 32 + i], dv[i]);
        }
      }
      __syncthreads();
      for (int i = threadIdx.x; i < kpc * D; i += blockDim.x) {
        const int jj = kp + i / D;
        if (jj < nb) {
          const int64_t tok = bperm[p0 + jj];
          atomicAdd(dk_out + (tok * hkv + g) * D + i % D, red_k[i] * scale);
          atomicAdd(dv_out + (tok * hkv + g) * D + i % D, red_v[i]);
        }
      }
    }
  }
}

// selected branch backward, query-centric and fused (head dim 64, G in {8, 16}):
// one warp per (token, group); lane l owns dims {2l, 2l+1} of every head of the
// group.  For each key of the selected blocks the per-head dot products are
// reduced across the warp by a transpose-reduction (G values, G shuffles), each
// lane finishes the softmax gradient of its head, the results are broadcast,
// and the warp accumulates dQ in registers and adds dK, dV rows of the key with
// fp32 vector atomics.  Q and dO are read once per pair.
template <typename T>
__device__ __forceinline__ float2 load2(const T* p);
template <>
__device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
template <>
__device__ __forceinline__ float2 load2<float>(const float* p) {
  return __ldg(reinterpret_cast<const float2*>(p));
}

// Sum over the 32 lanes of each of the G values a[0..G); on return the 32/G
// lanes [h * 32/G, (h+1) * 32/G) hold the total of value h (G in {8, 16}).
template <int G>
__device__ __forceinline__ float warp_transpose_reduce(float (&a)[G]) {
  const int lane = threadIdx.x & 31;
  float v[G];
#pragma unroll
  for (int i = 0; i < G; ++i) v[i] = a[i];
  // offsets 16, 8, 4, 2 halve the number of values per lane (head bits 3..0 <- lane bits 4..1)
  int n = G;
#pragma unroll
  for (int off = 16; off >= 2; off >>= 1) {
    if (n == 1) {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
      continue;
    }
    const bool up = (lane & off) != 0;
    const int h = n / 2;
#pragma unroll
    for (int i = 0; i < G / 2; ++i) {
      if (i < h) {
        const float send = up ? v[i] : v[i + h];
        const float keep = up ? v[i + h] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    n = h;
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

template <typename T, int G>
__global__ void __launch_bounds__(256) slc_bwd_fused_kernel(
    const T* __restrict__ q, const T* __restrict__ ks, const T* __restrict__ vs, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ bptr, const int32_t* __restrict__ bperm,
    const int32_t* __restrict__ sel, int64_t N, int64_t ldk, int hq, int hkv, int topk, float qs2, float scale,
    const float* __restrict__ lse_in, const float* __restrict__ Dc, float* __restrict__ dq_out,
    float* __restrict__ dk_out, float* __restrict__ dv_out) {
  constexpr int D = 64;
  const int lane = threadIdx.x & 31;
  const int wpc = blockDim.x / 32;
  const int64_t npairs = N * hkv;
  // head whose softmax this lane finishes after the reduction: lanes [h LPH, (h+1) LPH) -> head h
  constexpr int LPH = 32 / G;
  const int myh = lane / LPH;
  for (int64_t pair = (int64_t)blockIdx.x * wpc + threadIdx.x / 32; pair < npairs; pair += (int64_t)gridDim.x * wpc) {
    const int64_t t = pair / hkv;
    const int g = (int)(pair % hkv);
    float q2[G][2], d2[G][2], dq2[G][2];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const int64_t row = t * hq + g * G + h;
      const float2 a = load2<T>(q + row * D + 2 * lane);
      const float2 b = load2<T>(dout + row * D + 2 * lane);
      const float w = gate_weight(gates, row * 3 + 1, mode);
      q2[h][0] = a.x;
      q2[h][1] = a.y;
      d2[h][0] = b.x * w;
      d2[h][1] = b.y * w;
      dq2[h][0] = dq2[h][1] = 0.f;
    }
    const int64_t my_row = t * hq + g * G + myh;
    const float lse2 = lse_in[my_row] * kLog2e;
    const float Dm = Dc[my_row];
    const int32_t* srow = sel + pair * topk;
    for (int si = 0; si < topk; ++si) {
      const int b = srow[si];
      if (b < 0) continue;
      const int p1 = bptr[b + 1];
      for (int j = bptr[b]; j < p1; ++j) {
        const int64_t kidx = (int64_t)g * ldk + j;
        const float2 kk = load2<T>(ks + kidx * D + 2 * lane);
        const float2 vv = load2<T>(vs + kidx * D + 2 * lane);
        float ps[G], pd[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          ps[h] = q2[h][0] * kk.x + q2[h][1] * kk.y;
          pd[h] = d2[h][0] * vv.x + d2[h][1] * vv.y;
        }
        const float s2 = warp_transpose_reduce<G>(ps) * qs2;
        const float dp = warp_transpose_reduce<G>(pd);
        const float pm = exp2f(s2 - lse2);
        const float dsm = pm * (dp - Dm);
        float dk0 = 0.f, dk1 = 0.f, dv0 = 0.f, dv1 = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float ph = __shfl_sync(0xffffffffu, pm, h * LPH);
          const float dsh = __shfl_sync(0xffffffffu, dsm, h * LPH);
          dq2[h][0] = fmaf(dsh, kk.x, dq2[h][0]);
          dq2[h][1] = fmaf(dsh, kk.y, dq2[h][1]);
          dk0 = fmaf(dsh, q2[h][0], dk0);
          dk1 = fmaf(dsh, q2[h][1], dk1);
          dv0 = fmaf(ph, d2[h][0], dv0);
          dv1 = fmaf(ph, d2[h][1], dv1);
        }
        const int64_t tok = bperm[j];
        atomicAdd(reinterpret_cast<float2*>(dk_out + (tok * hkv + g) * D + 2 * lane), make_float2(dk0 * scale, dk1 * scale));
        atomicAdd(reinterpret_cast<float2*>(dv_out + (tok * hkv + g) * D + 2 * lane), make_float2(dv0, dv1));
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float2* dst = reinterpret_cast<float2*>(dq_out + (t * hq + g * G + h) * D + 2 * lane);
      float2 cur = *dst;
      cur.x += dq2[h][0] * scale;
      cur.y += dq2[h][1] * scale;
      *dst = cur;
    }
  }
}

// window branch: dQ
template <typename T, int D>
__global__ void __launch_bounds__(128) win_bwd_dq_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ wperm, const int32_t* __restrict__ wptr,
    int64_t wtot, int hq, int hkv, float qs2, float scale, const float* __restrict__ lse_in,
    const float* __restrict__ Dc, float* __restrict__ dq_out) {
  using C = Cfg<D>;
  constexpr int KT = 32;
  __shared__ __align__(16) float sk[KT * C::KSTR];
  __shared__ __align__(16) float sv[KT * C::KSTR];
  const int g = blockIdx.y, G = hq / hkv;
  const int r = threadIdx.x / C::NT, sub = threadIdx.x % C::NT;
  for (int64_t w = blockIdx.x; w < wtot; w += gridDim.x) {
    const int p0 = wptr[w], nw = wptr[w + 1] - p0;
    const int nrows = nw * G;
    const int nchunks = (nw + KT - 1) / KT;
    for (int row0 = 0; row0 < nrows; row0 += C::ROWS) {
      const int rr = row0 + r;
      const bool valid = rr < nrows;
      const int64_t t = wperm[p0 + (valid ? rr / G : 0)];
      const int h = g * G + (valid ? rr % G : 0);
      const int64_t row = t * hq + h;
      float qv[32], dov[32], dq[32];
      load32(q + row * D + sub * 32, qv);
      load32(dout + row * D + sub * 32, dov);
      const float wg = gate_weight(gates, row * 3 + 2, mode);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        qv[i] *= qs2;
        dov[i] *= wg;
        dq[i] = 0.f;
      }
      const float lse2 = lse_in[row] * kLog2e;
      const float Dr = Dc[row];
      for (int c = 0; c < nchunks; ++c) {
        const int kn = min(KT, nw - c * KT);
        if (nchunks > 1 || row0 == 0) {
          __syncthreads();
          stage_rows<T, D>(sk, kn, [&](int j) { return k + ((int64_t)wperm[p0 + c * KT + j] * hkv + g) * D; });
          stage_rows<T, D>(sv, kn, [&](int j) { return v + ((int64_t)wperm[p0 + c * KT + j] * hkv + g) * D; });
          __syncthreads();
        }
        for (int j = 0; j < kn; ++j) {
          const float* krow = sk + j * C::KSTR + sub * 36;
          const float s2 = row_sum<C::NT>(dot32(qv, krow), 0xffffffffu);
          const float p = exp2f(s2 - lse2);
          const float dp = row_sum<C::NT>(dot32(dov, sv + j * C::KSTR + sub * 36), 0xffffffffu);
          axpy32(dq, p * (dp - Dr), krow);
        }
      }
      if (valid) {
        float* dst = dq_out + row * D + sub * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[i] += dq[i] * scale;
      }
    }
  }
}

// window branch: dK, dV (added onto the selected branch's values)
template <typename T, int D>
__global__ void __launch_bounds__(128) win_bwd_dkv_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dout,
    const float* __restrict__ gates, int mode, const int32_t* __restrict__ wperm, const int32_t* __restrict__ wptr,
    int64_t wtot, int hq, int hkv, float qs2, float scale, const float* __restrict__ lse_in,
    const float* __restrict__ Dc, float* __restrict__ dk_out, float* __restrict__ dv_out) {
  using C = Cfg<D>;
  __shared__ __align__(16) RowStage<T, D> st;
  const int g = blockIdx.y, G = hq / hkv;
  const int sub = threadIdx.x % C::NT;
  for (int64_t w = blockIdx.x; w < wtot; w += gridDim.x) {
    const int p0 = wptr[w], nw = wptr[w + 1] - p0;
    const int64_t nrows = (int64_t)nw * G;
    for (int kp = 0; kp < nw; kp += C::ROWS) {
      const int j = kp + threadIdx.x / C::NT;
      const bool validk = j < nw;
      const int64_t tok = wperm[p0 + (validk ? j : 0)];
      float kv[32], vv[32], dk[32], dv[32];
      load32(k + (tok * hkv + g) * D + sub * 32, kv);
      load32(v + (tok * hkv + g) * D + sub * 32, vv);
#pragma unroll
      for (int i = 0; i < 32; ++i) dk[i] = dv[i] = 0.f;
      for (int64_t rs = 0; rs < nrows; rs += RowStage<T, D>::RT) {
        const int n = (int)min((int64_t)RowStage<T, D>::RT, nrows - rs);
        __syncthreads();
        stage_query_rows<T, D>(
            st, n,
            [&](int i, int64_t* row) {
              const int64_t gr = rs + i;
              *row = (int64_t)wperm[p0 + gr / G] * hq + g * G + gr % G;
              return true;
            },
            q, dout, gates, mode, 2, lse_in, Dc);
        __syncthreads();
        accumulate_rows<T, D>(st, kv, vv, qs2, dk, dv);
      }
      if (validk) {
        float* a = dk_out + (tok * hkv + g) * D + sub * 32;
        float* c = dv_out + (tok * hkv + g) * D + sub * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          a[i] += dk[i] * scale;
          c[i] += dv[i];
        }
      }
    }
  }
}

// compression gradient back to tokens: dK_i += dKc_b / n_b (likewise V)
__global__ void cmp_scatter_kernel(const float* __restrict__ dkc, const float* __restrict__ dvc,
                                   const int32_t* __restrict__ bid, const int32_t* __restrict__ bptr, int64_t N,
                                   int64_t btot, int hkv, int d, float* __restrict__ dk, float* __restrict__ dv) {
  const int q4 = d / 4;
  const int64_t total = N * hkv * q4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int qd = (int)(i % q4);
    const int64_t tg = i / q4;
    const int g = (int)(tg % hkv);
    const int64_t t = tg / hkv;
    const int b = bid[t];
    const float n = (float)(bptr[b + 1] - bptr[b]);
    const int64_t src = ((int64_t)g * btot + b) * d + qd * 4;
    const float4 a = *reinterpret_cast<const float4*>(dkc + src);
    const float4 c = *reinterpret_cast<const float4*>(dvc + src);
    float4* pk = reinterpret_cast<float4*>(dk + tg * d + qd * 4);
    float4* pv = reinterpret_cast<float4*>(dv + tg * d + qd * 4);
    float4 x = *pk, y = *pv;
    x.x += __fdiv_rn(a.x, n);
    x.y += __fdiv_rn(a.y, n);
    x.z += __fdiv_rn(a.z, n);
    x.w += __fdiv_rn(a.w, n);
    y.x += __fdiv_rn(c.x, n);
    y.y += __fdiv_rn(c.y, n);
    y.z += __fdiv_rn(c.z, n);
    y.w += __fdiv_rn(c.w, n);
    *pk = x;
    *pv = y;
  }
}

// inverted selection: key (g * btot + b) per (token, group, slot), sentinel for -1
// A selection given by the caller: every entry must be -1 or a block of the token's
// own sequence; anything else becomes -1 and is reported in the device check word.
__global__ void sel_check_kernel(int32_t* __restrict__ sel, int64_t N, int hkv, int topk,
                                 const int32_t* __restrict__ cu, int S, const int32_t* __restrict__ bcu,
                                 int* __restrict__ status) {
  const int64_t total = N * hkv * topk;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t b = sel[i];
    if (b == -1) continue;
    const int s = find_segment(cu, S, i / ((int64_t)hkv * topk));
    if (b < bcu[s] || b >= bcu[s + 1]) {
      sel[i] = -1;
      bad = true;
    }
  }
  if (bad) atomicOr(status, kStatusSelection);
}

// Cross attention: gates [rows, 2] widened to the [rows, 3] layout the kernels read
// (column 2 unused), and a check that every sequence with queries has blocks.
__global__ void cross_prep_kernel(const float* __restrict__ g2, int64_t rows, float* __restrict__ g3,
                                  const int32_t* __restrict__ q_cu, const int32_t* __restrict__ bcu, int S,
                                  int* __restrict__ bad) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows; r += stride) {
    g3[3 * r] = g2[2 * r];
    g3[3 * r + 1] = g2[2 * r + 1];
    g3[3 * r + 2] = 0.f;
  }
  for (int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; s < S; s += stride)
    if (q_cu[s + 1] > q_cu[s] && bcu[s + 1] == bcu[s]) atomicOr(bad, 1);
}

__global__ void sel_keys_kernel(const int32_t* __restrict__ sel, int64_t N, int hkv, int topk, int64_t btot,
                                uint64_t* __restrict__ keys, int32_t* __restrict__ vals) {
  const int64_t total = N * hkv * topk;
  const uint64_t sentinel = (uint64_t)hkv * btot;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t pair = i / topk;
    const int g = (int)(pair % hkv);
    const int b = sel[i];
    keys[i] = b >= 0 ? (uint64_t)g * btot + b : sentinel;
    vals[i] = (int32_t)(pair / hkv);
  }
}

// CSR pointers from sorted keys: ptr[key] = first position with that key (or later)
__global__ void keys_to_ptr_kernel(const uint64_t* __restrict__ keys, int64_t n, int64_t nkeys,
                                   int32_t* __restrict__ ptr) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i <= n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t lo = i == 0 ? 0 : (int64_t)keys[i - 1] + 1;
    const int64_t hi = i == n ? nkeys : (int64_t)keys[i];
    for (int64_t k = lo; k <= hi && k <= nkeys; ++k) ptr[k] = (int32_t)i;
  }
}

// per-sequence work counts for the tiled kernels
// dst[i] = src[i] * 2^-32: the deterministic fixed-point sums back to fp32 (through
// fp64, which holds the 64-bit integer's leading bits exactly enough for one rounding).
__global__ void fix_to_float_kernel(const unsigned long long* __restrict__ src, float* __restrict__ dst, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = (float)((double)(long long)src[i] * (1.0 / 4294967296.0));
}

// dst[rows[i]] += src[i] for rows of `w4` float4 (dK and dV at once); the rows are distinct.
__global__ void rows_add_kernel(const float* __restrict__ srck, const float* __restrict__ srcv,
                                const int32_t* __restrict__ rows, int64_t n, int w4, float* __restrict__ dstk,
                                float* __restrict__ dstv) {
  const int64_t total = n * w4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / w4, c = i % w4;
    const int64_t d = (int64_t)rows[r] * w4 + c;
    const float4 a = reinterpret_cast<const float4*>(srck)[i], b = reinterpret_cast<const float4*>(srcv)[i];
    float4 x = reinterpret_cast<float4*>(dstk)[d], y = reinterpret_cast<float4*>(dstv)[d];
    x.x += a.x; x.y += a.y; x.z += a.z; x.w += a.w;
    y.x += b.x; y.y += b.y; y.z += b.z; y.w += b.w;
    reinterpret_cast<float4*>(dstk)[d] = x;
    reinterpret_cast<float4*>(dstv)[d] = y;
  }
}

__global__ void plan_counts_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ bcu, int S, int G,
                                   int rows_per_tile, int blocks_per_item, int rc_rows, int32_t* __restrict__ tiles,
                                   int32_t* __restrict__ items) {
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s <= S; s += gridDim.x * blockDim.x) {
    if (s == S) {
      tiles[s] = 0;
      items[s] = 0;
      continue;
    }
    const int64_t nrows = (int64_t)(cu[s + 1] - cu[s]) * G;
    const int nb = bcu[s + 1] - bcu[s];
    tiles[s] = (int32_t)((nrows + rows_per_tile - 1) / rows_per_tile);
    items[s] = (int32_t)(((nb + blocks_per_item - 1) / blocks_per_item) * ((nrows + rc_rows - 1) / rc_rows));
  }
}

inline int grid_1d(int64_t n, int threads, int cap = 148 * 16) {
  int64_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return (int)b;
}

template <typename T, int D>
cudaError_t forward_impl(const FwdArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  const int G = a.hq / a.hkv;
  const float qs2 = a.scale * kLog2e;
  const int64_t rows = a.N * a.hq;
  const T* q = static_cast<const T*>(a.q);
  const T* kc = static_cast<const T*>(a.kc);
  const T* vc = static_cast<const T*>(a.vc);
  float* ob = static_cast<float*>(a.o_branch);
  if (a.sel_given)
    SSA_LAUNCH("sel_check_kernel", sel_check_kernel, grid_1d(a.N * a.hkv * a.topk, 256, 148 * 32), 256, 0, st, a.sel,
               a.N, a.hkv, a.topk, a.cu_seqlens, a.S, a.blk->cu, a.status);
  // plan
  SSA_LAUNCH("plan_counts_kernel", plan_counts_kernel, grid_1d(a.S + 1, 256), 256, 0, st, a.cu_seqlens, a.blk->cu, a.S, G, C::ROWS, C::ROWS,
                                                            kCmpRowChunk, a.tiles_cnt, a.items_cnt);
  cudaError_t e = exclusive_scan(a.tiles_cnt, a.tiles_pre, a.S + 1, a.scan_tmp, st);
  if (e != cudaSuccess) return e;
  if (a.use_tc && D == 64 && cmp_tc_supported(a.dtype, D, a.hq, a.hkv, a.topk)) {
    // 128-row tiles for the tensor-core kernels
    SSA_LAUNCH("plan_counts_kernel", plan_counts_kernel, grid_1d(a.S + 1, 256), 256, 0, st, a.cu_seqlens, a.blk->cu,
               a.S, G, 128, 128, kCmpRowChunk, a.items_cnt, a.tiles_cnt);
    e = exclusive_scan(a.items_cnt, a.items_pre, a.S + 1, a.scan_tmp, st);
    if (e != cudaSuccess) return e;
    e = cmp_fwd_tc(a, a.items_pre, (a.N * G + 127) / 128 + a.S, st);
    if (e != cudaSuccess) return e;
  } else {
    const int tile_grid = grid_1d(rows, C::ROWS, 148 * 8);
    const dim3 g2(tile_grid, a.hkv);
    SSA_LAUNCH("cmp_lse_kernel", (cmp_lse_kernel<T, D>), g2, 128, 0, st, q, kc, a.cu_seqlens, a.blk->cu, a.tiles_pre, a.S, a.hq, a.hkv,
                                             a.blk->count, qs2, a.lse);
    SSA_LAUNCH("cmp_out_topk_kernel", (cmp_out_topk_kernel<T, D>), g2, 128, 0, st, q, kc, vc, a.cu_seqlens, a.blk->cu, a.tiles_pre, a.S, a.hq, a.hkv,
                                                  a.blk->count, qs2, a.lse, ob, a.topk,
                                                  a.sel_given ? nullptr : a.sel);
  }
  if (a.use_tc && D == 64 && slc_mma_supported(a.dtype, D, a.hq, a.hkv, a.topk)) {
    e = slc_fwd_mma(a, st);
    if (e != cudaSuccess) return e;
  } else {
    const int pairs_per_cta = 128 / (G * C::NT);
    SSA_LAUNCH("slc_fwd_kernel", (slc_fwd_kernel<T, D>), grid_1d(a.N * a.hkv, pairs_per_cta, 148 * 16), 128, 0, st,
               q, static_cast<const T*>(a.ks), static_cast<const T*>(a.vs), a.blk->ptr, a.sel, a.N, a.Nkv, a.hq,
               a.hkv, a.topk, qs2, ob + rows * D, a.lse + rows);
  }
  if (a.has_win) {  // cross attention has no window branch (the queries have no voxel)
    const dim3 gw(grid_1d(a.win->count, 1, 148 * 16), a.hkv);
    if (a.use_tc && D == 64 && win_tc_supported(a.dtype, D, a.hq, a.hkv, a.m_cmp, a.m_win)) {
      e = win_fwd_tc(a, a.win_cnt, a.win_pre, a.win_scan, st);
      if (e != cudaSuccess) return e;
    } else
      SSA_LAUNCH("win_fwd_kernel", (win_fwd_kernel<T, D>), gw, 128, 0, st, q, static_cast<const T*>(a.wk),
                 static_cast<const T*>(a.wv), a.win->perm, a.win->ptr, a.win->count, a.hq, a.hkv, qs2,
                 ob + 2 * rows * D, a.lse + 2 * rows);
  }
  SSA_LAUNCH("combine_kernel", (combine_kernel<T, D>), grid_1d(rows * C::NT, 256, 148 * 32), 256, 0, st, ob, a.gates,
             rows, a.gate_mode, a.has_win ? 3 : 2, static_cast<T*>(a.out));
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t backward_impl(const BwdArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  const int G = a.hq / a.hkv;
  const float qs2 = a.scale * kLog2e;
  const int64_t rows = a.N * a.hq;
  const int64_t btot = a.blk->count;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* kc = static_cast<const T*>(a.kc);
  const T* vc = static_cast<const T*>(a.vc);
  const T* ks = static_cast<const T*>(a.ks);
  const T* vs = static_cast<const T*>(a.vs);
  const float* ob = static_cast<const float*>(a.o_branch);
  const T* dout = static_cast<const T*>(a.dout);

  SSA_LAUNCH("plan_counts_kernel", plan_counts_kernel, grid_1d(a.S + 1, 256), 256, 0, st, a.cu_seqlens, a.blk->cu, a.S, G, C::ROWS, C::ROWS,
                                                            kCmpRowChunk, a.tiles_cnt, a.items_cnt);
  cudaError_t e = exclusive_scan(a.tiles_cnt, a.tiles_pre, a.S + 1, a.scan_tmp, st);
  if (e != cudaSuccess) return e;
  e = exclusive_scan(a.items_cnt, a.items_pre, a.S + 1, a.scan_tmp, st);
  if (e != cudaSuccess) return e;

  const bool cmp_tc = a.use_tc && D == 64 && cmp_tc_supported(a.dtype, D, a.hq, a.hkv, a.topk) && a.q16;
  SSA_LAUNCH("bwd_pre_kernel", (bwd_pre_kernel<T, D>), grid_1d(rows * C::NT, 256, 148 * 32), 256, 0, st, ob, dout,
             a.gates, a.lse, rows, a.gate_mode, a.has_win ? 3 : 2, a.Dc, a.dgates, a.rc);
  if (cmp_tc) {
    // 128-row tiles for the tensor-core kernels (tiles_cnt / tiles_pre are free again here)
    SSA_LAUNCH("plan_counts_kernel", plan_counts_kernel, grid_1d(a.S + 1, 256), 256, 0, st, a.cu_seqlens, a.blk->cu,
               a.S, G, 128, 128, kCmpRowChunk, a.tiles_cnt, a.items_cnt);
    e = exclusive_scan(a.tiles_cnt, a.tiles_pre, a.S + 1, a.scan_tmp, st);
    if (e != cudaSuccess) return e;
    e = cmp_bwd_tc(a, a.tiles_pre, a.items_cnt, a.items_pre, a.scan_tmp, (a.N * G + 127) / 128 + a.S, st);
    if (e != cudaSuccess) return e;
  } else {
    const dim3 g2(grid_1d(rows, C::ROWS, 148 * 8), a.hkv);
    SSA_LAUNCH("cmp_bwd_dq_kernel", (cmp_bwd_dq_kernel<T, D>), g2, 128, 0, st, q, kc, vc, dout, a.gates, a.gate_mode, a.cu_seqlens, a.blk->cu,
                                                a.tiles_pre, a.S, a.hq, a.hkv, btot, qs2, a.scale, a.lse, a.Dc, a.dq);
    cudaMemsetAsync(a.dkc, 0, sizeof(float) * a.hkv * btot * D, st);
    cudaMemsetAsync(a.dvc, 0, sizeof(float) * a.hkv * btot * D, st);
    SSA_LAUNCH("cmp_bwd_dkv_kernel", (cmp_bwd_dkv_kernel<T, D>), dim3(148 * 8, a.hkv), 128, 0, st, 
        q, kc, vc, dout, a.gates, a.gate_mode, a.cu_seqlens, a.blk->cu, a.items_pre, a.S, a.hq, a.hkv, btot, qs2,
        a.scale, kCmpRowChunk, a.lse, a.Dc, a.dkc, a.dvc);
  }
  if (D == 64 && (G == 8 || G == 16)) {
    const int g_slc = grid_1d(a.N * a.hkv, 8, 148 * 16);
    if (a.use_tc && slc_mma_supported(a.dtype, D, a.hq, a.hkv, a.topk)) {
      if (a.fx_k) {  // deterministic: fixed-point sums of the selected branch, then dK / dV = them
        cudaMemsetAsync(a.fx_k, 0, sizeof(unsigned long long) * a.Nkv * a.hkv * D, st);
        cudaMemsetAsync(a.fx_v, 0, sizeof(unsigned long long) * a.Nkv * a.hkv * D, st);
      } else {
        cudaMemsetAsync(a.dk, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
        cudaMemsetAsync(a.dv, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
      }
      e = slc_bwd_mma(a, st);
      if (e == cudaSuccess && a.fx_k) {
        e = fix_to_float(a.fx_k, a.dk, a.Nkv * a.hkv * D, st);
        if (e == cudaSuccess) e = fix_to_float(a.fx_v, a.dv, a.Nkv * a.hkv * D, st);
      }
      if (e != cudaSuccess) return e;
    } else if (G == 16) {
      cudaMemsetAsync(a.dk, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
      cudaMemsetAsync(a.dv, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
      SSA_LAUNCH("slc_bwd_fused_kernel", (slc_bwd_fused_kernel<T, 16>), g_slc, 256, 0, st, q, ks, vs, dout, a.gates,
                 a.gate_mode, a.blk->ptr, a.blk->perm, a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, a.scale,
                 a.lse + rows,
                 a.Dc + rows, a.dq, a.dk, a.dv);
    } else {
      cudaMemsetAsync(a.dk, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
      cudaMemsetAsync(a.dv, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
      SSA_LAUNCH("slc_bwd_fused_kernel", (slc_bwd_fused_kernel<T, 8>), g_slc, 256, 0, st, q, ks, vs, dout, a.gates,
                 a.gate_mode, a.blk->ptr, a.blk->perm, a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, a.scale,
                 a.lse + rows,
                 a.Dc + rows, a.dq, a.dk, a.dv);
    }
  } else {
    const int pairs_per_cta = 128 / (G * C::NT);
    SSA_LAUNCH("slc_bwd_dq_kernel", (slc_bwd_dq_kernel<T, D>), grid_1d(a.N * a.hkv, pairs_per_cta, 148 * 16), 128, 0, st, 
        q, ks, vs, dout, a.gates, a.gate_mode, a.blk->ptr, a.sel, a.N, a.Nkv, a.hq, a.hkv, a.topk, qs2, a.scale,
        a.lse + rows,
        a.Dc + rows, a.dq);
    // inverted selection CSR: for (g, b), the tokens whose group g selected b, ascending
    const int64_t nsel = a.N * a.hkv * a.topk;
    const int64_t nkeys = a.hkv * btot;
    SSA_LAUNCH("sel_keys_kernel", sel_keys_kernel, grid_1d(nsel, 256, 148 * 32), 256, 0, st, a.sel, a.N, a.hkv, a.topk, btot, a.inv_keys_a,
                                                                  a.inv_vals_a);
    int bits = 1;
    while ((1ll << bits) <= nkeys) ++bits;
    bool in_b = false;
    e = radix_sort_pairs(a.inv_keys_a, a.inv_vals_a, a.inv_keys_b, a.inv_vals_b, nsel, bits, a.radix_tmp, &in_b, st);
    if (e != cudaSuccess) return e;
    const uint64_t* sk = in_b ? a.inv_keys_b : a.inv_keys_a;
    const int32_t* sv = in_b ? a.inv_vals_b : a.inv_vals_a;
    SSA_LAUNCH("keys_to_ptr_kernel", keys_to_ptr_kernel, grid_1d(nsel + 1, 256, 148 * 32), 256, 0, st, sk, nsel, nkeys, a.inv_ptr);
    SSA_LAUNCH("slc_items_kernel", slc_items_kernel, grid_1d(nkeys + 1, 256, 148 * 32), 256, 0, st, a.inv_ptr, nkeys,
               G, a.slc_cnt);
    e = exclusive_scan(a.slc_cnt, a.slc_pre, nkeys + 1, a.scan_tmp, st);
    if (e != cudaSuccess) return e;
    cudaMemsetAsync(a.dk, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
    cudaMemsetAsync(a.dv, 0, sizeof(float) * a.Nkv * a.hkv * D, st);
    SSA_LAUNCH("slc_bwd_dkv_kernel", (slc_bwd_dkv_kernel<T, D>), 148 * 8, 128, 0, st, q, ks, vs, dout, a.gates,
               a.gate_mode, a.blk->ptr, a.blk->perm, a.inv_ptr, sv, a.slc_pre, a.Nkv, btot, a.hq, a.hkv, qs2, a.scale,
               a.lse + rows, a.Dc + rows, a.dk, a.dv);
  }
  if (a.has_win) {
    if (a.wtok) {  // a rank's window gradients go to a local buffer first
      cudaMemsetAsync(a.wdk, 0, sizeof(float) * a.N * a.hkv * D, st);
      cudaMemsetAsync(a.wdv, 0, sizeof(float) * a.N * a.hkv * D, st);
    }
    if (a.use_tc && D == 64 && win_tc_supported(a.dtype, D, a.hq, a.hkv, a.m_cmp, a.m_win)) {
      e = win_bwd_tc(a, a.win_cnt, a.win_pre, a.scan_tmp, st);
      if (e != cudaSuccess) return e;
    } else {
      const T* wk = static_cast<const T*>(a.wk);
      const T* wv = static_cast<const T*>(a.wv);
      const dim3 gw(grid_1d(a.win->count, 1, 148 * 16), a.hkv);
      SSA_LAUNCH("win_bwd_dq_kernel", (win_bwd_dq_kernel<T, D>), gw, 128, 0, st, q, wk, wv, dout, a.gates,
                 a.gate_mode, a.win->perm, a.win->ptr, a.win->count, a.hq, a.hkv, qs2, a.scale, a.lse + 2 * rows,
                 a.Dc + 2 * rows, a.dq);
      SSA_LAUNCH("win_bwd_dkv_kernel", (win_bwd_dkv_kernel<T, D>), gw, 128, 0, st, q, wk, wv, dout, a.gates,
                 a.gate_mode, a.win->perm, a.win->ptr, a.win->count, a.hq, a.hkv, qs2, a.scale, a.lse + 2 * rows,
                 a.Dc + 2 * rows, a.wdk, a.wdv);
    }
  }
  if (a.conv)  // the learned compression: dK, dV through the convolution, dW, db
    return conv_backward(*a.conv, a.dtype, a.k, a.v, a.dkc, a.dvc, a.dk, a.dv, st);
  SSA_LAUNCH("cmp_scatter_kernel", cmp_scatter_kernel, grid_1d(a.Nkv * a.hkv * D / 4, 256, 148 * 32), 256, 0, st,
             a.dkc, a.dvc, a.blk->id, a.blk->ptr, a.Nkv, btot, a.hkv, D, a.dk, a.dv);
  if (a.has_win && a.wtok)  // a rank's window gradients into the rows of its tokens
    SSA_LAUNCH("rows_add_kernel", rows_add_kernel, grid_1d(a.N * a.hkv * D / 4, 256, 148 * 32), 256, 0, st, a.wdk,
               a.wdv, a.wtok, a.N, a.hkv * D / 4, a.dk, a.dv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t cross_prep(const float* gates2, int64_t rows, float* gates3, const int32_t* q_cu, const int32_t* bcu,
                       int S, int* bad, cudaStream_t st) {
  SSA_LAUNCH("cross_prep_kernel", cross_prep_kernel, grid_1d(rows > S ? rows : S, 256, 148 * 32), 256, 0, st, gates2,
             rows, gates3, q_cu, bcu, S, bad);
  return cudaGetLastError();
}

cudaError_t simt_forward(const FwdArgs& a, cudaStream_t st) {
  if (a.dtype == SSA_DTYPE_BF16) {
    if (a.d == 32) return forward_impl<__nv_bfloat16, 32>(a, st);
    if (a.d == 64) return forward_impl<__nv_bfloat16, 64>(a, st);
    if (a.d == 128) return forward_impl<__nv_bfloat16, 128>(a, st);
  } else {
    if (a.d == 32) return forward_impl<float, 32>(a, st);
    if (a.d == 64) return forward_impl<float, 64>(a, st);
    if (a.d == 128) return forward_impl<float, 128>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t fix_to_float(const unsigned long long* src, float* dst, int64_t n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  SSA_LAUNCH("fix_to_float_kernel", fix_to_float_kernel, grid_1d(n, 256, 148 * 32), 256, 0, st, src, dst, n);
  return cudaGetLastError();
}

cudaError_t simt_backward(const BwdArgs& a, cudaStream_t st) {
  if (a.dtype == SSA_DTYPE_BF16) {
    if (a.d == 32) return backward_impl<__nv_bfloat16, 32>(a, st);
    if (a.d == 64) return backward_impl<__nv_bfloat16, 64>(a, st);
    if (a.d == 128) return backward_impl<__nv_bfloat16, 128>(a, st);
  } else {
    if (a.d == 32) return backward_impl<float, 32>(a, st);
    if (a.d == 64) return backward_impl<float, 64>(a, st);
    if (a.d == 128) return backward_impl<float, 128>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ssa
