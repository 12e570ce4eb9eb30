// Window branch of SSA on the tcgen05 tensor cores (bf16, head dim 64), for
// window edge == block edge, so that a window's keys are one contiguous range
// of the block-sorted copies K_s / V_s [Hkv, N, 64].
//
// Direct3D-S2 (hyper.ai, "方法"): the sparse 3D window module splits the tokens
// into non-overlapping m_win^3 windows and runs self-attention only inside each.
//
// A row tile is 128 query rows = (128/G tokens of one window) x (G heads of a KV
// group); the tokens' Q (and dO) rows and per-row scalars are gathered by
// per-token TMA boxes.  Key tiles are 128 rows of K_s / V_s.
//   win_fwd_tc:     thread = row; S = Q K^T, online softmax across key tiles
//                   (O in TMEM rescaled when the row max grows), P (one bf16 per
//                   key: a row's sum over its own window's keys) as the TMEM A
//                   operand of O += P V.
//   win_bwd_dq_tc:  thread = row; S, dP = dO V^T; dS (bf16) -> dQ += dS K.
//   win_bwd_dkv_tc: thread = key; S^T = K Q^T, dP^T = V dO^T over the window's
//                   row tiles; dV += (P^T w) dO, dK += dS^T Q; adds into dK/dV.
// Roles: compute warps (thread <-> TMEM lane), one TMA warp, one MMA warp.
// Every wait is bounded; a timeout records kStatusTimeout and the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tc_host.cuh"

namespace ssa {
namespace {

using namespace tc;
using namespace tch;

constexpr int kTile = 128 * 128;  // bytes of a 128 x 64 bf16 tile
constexpr int kKT = 128;          // keys per key tile
constexpr int kWStages = 2;

__device__ __forceinline__ void timeout_exit(int* status, int* abort_flag) {
  atomicOr(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(abort_flag) = 1;
}
__device__ __forceinline__ bool is_aborted(const int* f) { return *reinterpret_cast<const volatile int*>(f) != 0; }

// item -> (group, window, row tile): items of a group are the row tiles of all windows
struct WinItem {
  int g, w, rt, p0, nw;
};
__device__ __forceinline__ WinItem win_item(int it, int nitems_g, const int32_t* wpre, int64_t W,
                                            const int32_t* wptr) {
  WinItem x;
  x.g = it / nitems_g;
  const int local = it % nitems_g;
  x.w = find_segment(wpre, (int)W, local);
  x.rt = local - wpre[x.w];
  x.p0 = wptr[x.w];
  x.nw = wptr[x.w + 1] - x.p0;
  return x;
}

// Gather the G head rows of each of the tile's tokens (slots past the window
// load an out-of-range token: zeros) into a 128-row SW128 tile, using lanes
// 0..TPT-1 of the calling warp.  `bytes` are added to `bar` by the caller.
template <int G>
__device__ __forceinline__ void gather_rows(void* dst, const CUtensorMap* map, uint64_t* bar, const int32_t* wperm,
                                            int p, int nvalid, int g, int64_t N, int lane) {
  constexpr int TPT = 128 / G;
  if (lane < TPT) {
    const int tok = lane < nvalid ? wperm[p + lane] : (int)N;
    tma_load_3d(static_cast<uint8_t*>(dst) + lane * G * 128, map, bar, 0, g * G, tok);
  }
}
// Row scalars of token slot i land in a 128-byte slot (TMA destinations must be
// 128-byte aligned): row r of the tile is at dst[(r / G) * kSlot + r % G].
constexpr int kSlot = 32;
constexpr int kScalarFloats = 16 * kSlot;  // up to 16 token slots (G >= 8)
__device__ __forceinline__ int scalar_idx(int r, int G) { return (r / G) * kSlot + r % G; }

template <int G>
__device__ __forceinline__ void gather_scalars(float* dst, const CUtensorMap* map, uint64_t* bar,
                                               const int32_t* wperm, int p, int nvalid, int g, int64_t N, int lane) {
  constexpr int TPT = 128 / G;
  if (lane < TPT) {
    const int tok = lane < nvalid ? wperm[p + lane] : (int)N;
    tma_load_2d(dst + lane * kSlot, map, bar, g * G, tok);
  }
}

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
struct WinFwdSmem {
  uint8_t q[2][kTile];
  uint8_t k[kWStages][kTile];
  uint8_t v[kWStages][kTile];
  uint64_t q_full[2], q_empty[2], kv_full[kWStages], kv_empty[kWStages];
  uint64_t s_full, s_empty, p_full, pv_done, o_empty, mma_done;
  uint32_t tmem;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(192, 1) win_fwd_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, const int32_t* __restrict__ wperm, const int32_t* __restrict__ wptr,
    const int32_t* __restrict__ wpre, int64_t W, int64_t N, int hq, int hkv, float qs2, float* __restrict__ o_out,
    float* __restrict__ lse_out, int* status) {
  constexpr int TPT = 128 / G;
  extern __shared__ uint8_t smem_raw[];
  WinFwdSmem& sm =
      *reinterpret_cast<WinFwdSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nitems_g = wpre[W];
  const int total = nitems_g * hkv;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
    }
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_empty, 4);
    mbar_init(&sm.p_full, 4);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_empty, 4);
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
  // TMEM columns: S [0,128), P [128,192), O [256,320)
  const uint32_t tm_s = tmem, tm_ph = tmem + 128, tm_o = tmem + 256;

  if (warp == 4) {
    // ---------------- producer: gathered Q per item; (K, V) per key tile
    uint32_t q_count = 0, kv_count = 0;
    int last_par[kWStages];
    for (int i = 0; i < kWStages; ++i) last_par[i] = -1;
    for (int it = blockIdx.x; it < total && !is_aborted(&sm.abort_flag); it += gridDim.x) {
      const WinItem x = win_item(it, nitems_g, wpre, W, wptr);
      const int qb = q_count % 2;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&sm.q_empty[qb], ((q_count / 2) & 1) ^ 1);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { timeout_exit(status, &sm.abort_flag); break; }
      if (lane == 0) mbar_expect_tx_only(&sm.q_full[qb], kTile);
      __syncwarp();
      gather_rows<G>(sm.q[qb], &qmap, &sm.q_full[qb], wperm, x.p0 + x.rt * TPT, x.nw - x.rt * TPT, x.g, N, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full[qb]);
      ++q_count;
      const int nkt = (x.nw + kKT - 1) / kKT;
      for (int kt = 0; kt < nkt; ++kt) {
        const int st = kv_count % kWStages;
        const uint32_t ph = (kv_count / kWStages) & 1;
        if (lane == 0) {
          ok = mbar_wait(&sm.kv_empty[st], ph ^ 1);
          if (ok) {
            mbar_expect_tx(&sm.kv_full[st], 2 * kTile);
            const int row = x.g * (int)N + x.p0 + kt * kKT;
            tma_load_2d(sm.k[st], &kmap, &sm.kv_full[st], 0, row);
            tma_load_2d(sm.v[st], &vmap, &sm.kv_full[st], 0, row);
            last_par[st] = (int)ph;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { timeout_exit(status, &sm.abort_flag); break; }
        ++kv_count;
      }
    }
    if (lane == 0)
      for (int i = 0; i < kWStages; ++i)
        if (last_par[i] >= 0) mbar_wait(&sm.kv_full[i], (uint32_t)last_par[i]);
  } else if (warp == 5) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, kKT);
      const uint32_t id_o = idesc_bf16(128, 64, false, true);
      uint32_t q_count = 0, kv_count = 0, s_count = 0, p_count = 0, o_count = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !is_aborted(&sm.abort_flag); it += gridDim.x) {
        const WinItem x = win_item(it, nitems_g, wpre, W, wptr);
        const int qb = q_count % 2;
        if (!mbar_wait(&sm.q_full[qb], (q_count / 2) & 1)) { ok = false; break; }
        ++q_count;
        const int nkt = (x.nw + kKT - 1) / kKT;
        for (int kt = 0; kt < nkt && ok; ++kt) {
          const int st = kv_count % kWStages;
          if (!mbar_wait(&sm.kv_full[st], (kv_count / kWStages) & 1) || !mbar_wait(&sm.s_empty, (s_count & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ss(tm_s, sdesc_kmajor_sw128(sm.q[qb], 32 * k), sdesc_kmajor_sw128(sm.k[st], 32 * k), id_s, k > 0);
          mma_commit(&sm.s_full);
          ++s_count;
          // O of the previous item must have been read before this item's first P V
          if ((kt == 0 && !mbar_wait(&sm.o_empty, (o_count & 1) ^ 1)) || !mbar_wait(&sm.p_full, p_count & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // only the 16-key steps that hold keys of the window (P is zero past them)
          const int nks = (min(kKT, x.nw - kt * kKT) + 15) / 16;
          for (int k = 0; k < nks; ++k) {
            const uint64_t bdesc = sdesc_mnmajor_sw128(sm.v[st], 2048 * k, kTile);
            mma_bf16_ts(tm_o, tm_ph + 8 * k, bdesc, id_o, kt > 0 || k > 0);
          }
          mma_commit(&sm.pv_done);
          mma_commit(&sm.kv_empty[st]);
          ++p_count;
          ++kv_count;
        }
        if (!ok) break;
        mma_commit(&sm.q_empty[qb]);
        ++o_count;
      }
      if (!ok) timeout_exit(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ---------------- compute warps: thread = row
    const int r = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t s_count = 0, p_count = 0, o_count = 0;
    for (int it = blockIdx.x; it < total && !is_aborted(&sm.abort_flag); it += gridDim.x) {
      const WinItem x = win_item(it, nitems_g, wpre, W, wptr);
      const int tk = x.rt * TPT + r / G;  // token position inside the window
      const bool valid = tk < x.nw;
      const int nkt = (x.nw + kKT - 1) / kKT;
      float m = -CUDART_INF_F, l = 0.f;
      bool ok = true;
      for (int kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait_warp(&sm.s_full, s_count & 1)) { ok = false; break; }
        tc_fence_after();
        // only the 32-key chunks that hold keys of the window are read and exponentiated
        // (windows average ~56 tokens); nch is the same for the whole warp
        const int vc = min(kKT, x.nw - kt * kKT);
        const int nch = (vc + 31) / 32;
        float sv[kKT];
#pragma unroll
        for (int ch = 0; ch < kKT / 32; ++ch)
          if (ch < nch) tmem_ld32(tm_s + lane_off + 32 * ch, sv + 32 * ch);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_empty);
        ++s_count;
#pragma unroll
        for (int c = 0; c < kKT; ++c) sv[c] = c < vc ? sv[c] : -CUDART_INF_F;  // keys past the window
        // row max as 8 independent chains
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = sv[c];
#pragma unroll
        for (int c = 8; c < kKT; ++c) mx8[c % 8] = fmaxf(mx8[c % 8], sv[c]);
        const float cm = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float mn = fmaxf(m, cm * qs2);  // qs2 > 0
        // the previous P V must be done before P is overwritten (and before O is rescaled)
        if (kt > 0 && !mbar_wait_warp(&sm.pv_done, (p_count - 1) & 1)) { ok = false; break; }
        // rescale the partial O by 2^(m - mn) (1 where the max did not grow); the
        // decision is the warp's, as tcgen05.ld / st are warp-collective
        if (kt > 0 && __any_sync(0xffffffffu, mn > m)) {
          tc_fence_after();
          const float corr = ex2(m - mn);
          float o[64];
          tmem_ld32(tm_o + lane_off, o);
          tmem_ld32(tm_o + lane_off + 32, o + 32);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] *= corr;
          tmem_st16(tm_o + lane_off, reinterpret_cast<const uint32_t*>(o));
          tmem_st16(tm_o + lane_off + 16, reinterpret_cast<const uint32_t*>(o + 16));
          tmem_st16(tm_o + lane_off + 32, reinterpret_cast<const uint32_t*>(o + 32));
          tmem_st16(tm_o + lane_off + 48, reinterpret_cast<const uint32_t*>(o + 48));
          l *= corr;
        }
        m = mn;
        const float2 qs = make_float2(qs2, qs2), nm = make_float2(-m, -m);
        float2 lsum = make_float2(0.f, 0.f);
        uint32_t hi[64];
#pragma unroll
        for (int ch = 0; ch < kKT / 32; ++ch) {
          if (ch < nch) {
#pragma unroll
            for (int c = 32 * ch; c < 32 * ch + 32; c += 2) {
              const float2 p = ex2x2(ffma2(make_float2(sv[c], sv[c + 1]), qs, nm));
              lsum = fadd2(lsum, p);
              hi[c / 2] = pack2(p);
            }
          }
        }
        l += lsum.x + lsum.y;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < kKT / 32; ++ch)
          if (ch < nch) tmem_st16(tm_ph + lane_off + 16 * ch, hi + 16 * ch);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
        ++p_count;
      }
      if (!ok) {
        timeout_exit(status, &sm.abort_flag);
        break;
      }
      // O = (P V) / l after the last P V
      if (!mbar_wait_warp(&sm.pv_done, (p_count - 1) & 1)) { timeout_exit(status, &sm.abort_flag); break; }
      tc_fence_after();
      float o[64];
      tmem_ld32(tm_o + lane_off, o);
      tmem_ld32(tm_o + lane_off + 32, o + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_empty);
      ++o_count;
      if (valid) {
        const int64_t t = wperm[x.p0 + tk];
        const int64_t row = t * hq + x.g * G + r % G;
        const float inv = 1.f / l;
        float4* dst = reinterpret_cast<float4*>(o_out + row * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
        lse_out[row] = (m + log2f(l)) * kLn2;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// backward dQ (thread = row)
// ---------------------------------------------------------------------------
struct WinDqSmem {
  uint8_t q[2][kTile];
  uint8_t dout[2][kTile];
  uint8_t k[kWStages][kTile];
  uint8_t v[kWStages][kTile];
  __align__(128) float lse[2][kScalarFloats];
  __align__(128) float Dr[2][kScalarFloats];
  __align__(128) float wr[2][kScalarFloats];
  uint64_t q_full[2], q_empty[2], kv_full[kWStages], kv_empty[kWStages];
  uint64_t sdp_full, sdp_empty, ds_full, ds_empty, dq_full, dq_empty, mma_done;
  uint32_t tmem;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(192, 1) win_bwd_dq_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const __grid_constant__ CUtensorMap lmap, const __grid_constant__ CUtensorMap cmap,
    const __grid_constant__ CUtensorMap wmap, const int32_t* __restrict__ wperm, const int32_t* __restrict__ wptr,
    const int32_t* __restrict__ wpre, int64_t W, int64_t N, int hq, int hkv, float qs2, float scale,
    float* __restrict__ dq_out, int* status) {
  constexpr int TPT = 128 / G;
  extern __shared__ uint8_t smem_raw[];
  WinDqSmem& sm = *reinterpret_cast<WinDqSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nitems_g = wpre[W];
  const int total = nitems_g * hkv;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
    }
    for (int i = 0; i < kWStages; ++i) {
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
    tmem_alloc(&sm.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  // TMEM columns: S [0,128), dP [128,256), dS [256,320), dQ [384,448)
  const uint32_t tm_s = tmem, tm_dp = tmem + 128, tm_dsh = tmem + 256, tm_dq = tmem + 384;

  if (warp == 4) {
    // ---------------- producer: gathered Q, dO, row scalars per item; (K, V) per key tile
    uint32_t q_count = 0, kv_count = 0;
    int last_par[kWStages];
    for (int i = 0; i < kWStages; ++i) last_par[i] = -1;
    for (int it = blockIdx.x; it < total && !is_aborted(&sm.abort_flag); it += gridDim.x) {
      const WinItem x = win_item(it, nitems_g, wpre, W, wptr);
      const int qb = q_count % 2;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&sm.q_empty[qb], ((q_count / 2) & 1) ^ 1);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { timeout_exit(status, &sm.abort_flag); break; }
      if (lane == 0) mbar_expect_tx_only(&sm.q_full[qb], 2 * kTile + 3 * 128 * 4);  // 3 scalar boxes of G floats x TPT tokens
      __syncwarp();
      const int pp = x.p0 + x.rt * TPT, nv = x.nw - x.rt * TPT;
      gather_rows<G>(sm.q[qb], &qmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
      gather_rows<G>(sm.dout[qb], &dmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
      gather_scalars<G>(sm.lse[qb], &lmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
      gather_scalars<G>(sm.Dr[qb], &cmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
      gather_scalars<G>(sm.wr[qb], &wmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full[qb]);
      ++q_count;
      const int nkt = (x.nw + kKT - 1) / kKT;
      for (int kt = 0; kt < nkt; ++kt) {
        const int st = kv_count % kWStages;
        const uint32_t ph = (kv_count / kWStages) & 1;
        if (lane == 0) {
          ok = mbar_wait(&sm.kv_empty[st], ph ^ 1);
          if (ok) {
            mbar_expect_tx(&sm.kv_full[st], 2 * kTile);
            const int row = x.g * (int)N + x.p0 + kt * kKT;
            tma_load_2d(sm.k[st], &kmap, &sm.kv_full[st], 0, row);
            tma_load_2d(sm.v[st], &vmap, &sm.kv_full[st], 0, row);
            last_par[st] = (int)ph;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { timeout_exit(status, &sm.abort_flag); break; }
        ++kv_count;
      }
    }
    if (lane == 0)
      for (int i = 0; i < kWStages; ++i)
        if (last_par[i] >= 0) mbar_wait(&sm.kv_full[i], (uint32_t)last_par[i]);
  } else if (warp == 5) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, kKT);
      const uint32_t id_q = idesc_bf16(128, 64, false, true);
      uint32_t q_count = 0, kv_count = 0, sdp_count = 0, ds_count = 0, dq_count = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !is_aborted(&sm.abort_flag); it += gridDim.x) {
        const WinItem x = win_item(it, nitems_g, wpre, W, wptr);
        const int qb = q_count % 2;
        if (!mbar_wait(&sm.q_full[qb], (q_count / 2) & 1)) { ok = false; break; }
        ++q_count;
        const int nkt = (x.nw + kKT - 1) / kKT;
        for (int kt = 0; kt < nkt; ++kt) {
          const int st = kv_count % kWStages;
          if (!mbar_wait(&sm.kv_full[st], (kv_count / kWStages) & 1) ||
              !mbar_wait(&sm.sdp_empty, (sdp_count & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mma_bf16_ss(tm_s, sdesc_kmajor_sw128(sm.q[qb], 32 * k), sdesc_kmajor_sw128(sm.k[st], 32 * k), id_s, k > 0);
            mma_bf16_ss(tm_dp, sdesc_kmajor_sw128(sm.dout[qb], 32 * k), sdesc_kmajor_sw128(sm.v[st], 32 * k), id_s,
                        k > 0);
          }
          mma_commit(&sm.sdp_full);
          ++sdp_count;
          if ((kt == 0 && !mbar_wait(&sm.dq_empty, (dq_count & 1) ^ 1)) || !mbar_wait(&sm.ds_full, ds_count & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // only the 16-key steps that hold keys of the window (dS is zero past them)
          const int nks = (min(kKT, x.nw - kt * kKT) + 15) / 16;
          for (int k = 0; k < nks; ++k) {
            const uint64_t bdesc = sdesc_mnmajor_sw128(sm.k[st], 2048 * k, kTile);
            mma_bf16_ts(tm_dq, tm_dsh + 8 * k, bdesc, id_q, kt > 0 || k > 0);
          }
          mma_commit(&sm.ds_empty);
          mma_commit(&sm.kv_empty[st]);
          ++ds_count;
          ++kv_count;
        }
        if (!ok) break;
        mma_commit(&sm.q_empty[qb]);
        mma_commit(&sm.dq_full);
        ++dq_count;
      }
      if (!ok) timeout_exit(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ---------------- compute warps: thread = row
    const int r = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t q_count = 0, sdp_count = 0, ds_count = 0, dq_count = 0;
    for (int it = blockIdx.x; it < total && !is_aborted(&sm.abort_flag); it += gridDim.x) {
      const WinItem x = win_item(it, nitems_g, wpre, W, wptr);
      const int qb = q_count % 2;
      if (!mbar_wait_warp(&sm.q_full[qb], (q_count / 2) & 1)) { timeout_exit(status, &sm.abort_flag); break; }
      ++q_count;
      // row constants: -lse log2(e), -D, w
      const float2 nl2 = make_float2(sm.lse[qb][scalar_idx(r, G)], sm.lse[qb][scalar_idx(r, G)]);
      const float2 nd2 = make_float2(sm.Dr[qb][scalar_idx(r, G)], sm.Dr[qb][scalar_idx(r, G)]);
      const float2 w2 = make_float2(sm.wr[qb][scalar_idx(r, G)], sm.wr[qb][scalar_idx(r, G)]);
      const float2 qs = make_float2(qs2, qs2);
      const int tk = x.rt * TPT + r / G;
      const bool valid = tk < x.nw;
      const int nkt = (x.nw + kKT - 1) / kKT;
      bool ok = true;
      for (int kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait_warp(&sm.sdp_full, sdp_count & 1)) { ok = false; break; }
        tc_fence_after();
        // only the 32-key chunks that hold keys of the window take part (vc keys)
        const int vc = min(kKT, x.nw - kt * kKT);
        const int nch = (vc + 31) / 32;
        uint32_t hi[64];
#pragma unroll
        for (int ch = 0; ch < kKT / 32; ++ch) {
          if (ch < nch) {
            float sv[32], dp[32];
            tmem_ld32(tm_s + lane_off + 32 * ch, sv);
            tmem_ld32(tm_dp + lane_off + 32 * ch, dp);
            tmem_ld_wait();
            const int nvh = vc - 32 * ch;
            if (nvh < 32) {  // keys past the window
#pragma unroll
              for (int c = 0; c < 32; ++c) sv[c] = c < nvh ? sv[c] : -CUDART_INF_F;
            }
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float2 p = ex2x2(ffma2(make_float2(sv[c], sv[c + 1]), qs, nl2));
              const float2 d = fmul2(p, ffma2(w2, make_float2(dp[c], dp[c + 1]), nd2));
              hi[(32 * ch + c) / 2] = pack2(d);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sdp_empty);
        ++sdp_count;
        if (!mbar_wait_warp(&sm.ds_empty, (ds_count & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < kKT / 32; ++ch) {
          if (ch < nch) {
            tmem_st16(tm_dsh + lane_off + 16 * ch, hi + 16 * ch);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ds_full);
        ++ds_count;
      }
      if (!ok) {
        timeout_exit(status, &sm.abort_flag);
        break;
      }
      if (!mbar_wait_warp(&sm.dq_full, dq_count & 1)) { timeout_exit(status, &sm.abort_flag); break; }
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
        const int64_t t = wperm[x.p0 + tk];
        float4* dst = reinterpret_cast<float4*>(dq_out + (t * hq + x.g * G + r % G) * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float4 c4 = dst[i];
          c4.x += g[4 * i] * scale;
          c4.y += g[4 * i + 1] * scale;
          c4.z += g[4 * i + 2] * scale;
          c4.w += g[4 * i + 3] * scale;
          dst[i] = c4;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// backward dK, dV (thread = key; two warpgroups split the rows of a row tile)
// ---------------------------------------------------------------------------
constexpr int kCW = 8;  // compute warps of the dK/dV kernel

struct WinDkvSmem {
  uint8_t k[kTile];
  uint8_t v[kTile];
  uint8_t q[2][kTile];
  uint8_t dout[2][kTile];
  __align__(128) float lse[2][kScalarFloats];
  __align__(128) float Dr[2][kScalarFloats];
  __align__(128) float wr[2][kScalarFloats];
  uint64_t kv_full, kv_empty, q_full[2], q_empty[2];
  uint64_t sdp_full, sdp_empty, pds_full, pds_empty, acc_full, acc_empty, mma_done;
  uint32_t tmem;
  int abort_flag;
};

// item -> (group, window, key tile)
__device__ __forceinline__ WinItem win_kitem(int it, int nitems_g, const int32_t* wkpre, int64_t W,
                                             const int32_t* wptr) {
  return win_item(it, nitems_g, wkpre, W, wptr);  // .rt is the key tile
}

template <int G>
__global__ void __launch_bounds__(32 * (kCW + 2), 1) win_bwd_dkv_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const __grid_constant__ CUtensorMap lmap, const __grid_constant__ CUtensorMap cmap,
    const __grid_constant__ CUtensorMap wmap, const int32_t* __restrict__ wperm, const int32_t* __restrict__ wptr,
    const int32_t* __restrict__ wkpre, int64_t W, int64_t N, int hq, int hkv, float qs2, float scale,
    float* __restrict__ dk_out, float* __restrict__ dv_out, int* status) {
  constexpr int TPT = 128 / G;
  extern __shared__ uint8_t smem_raw[];
  WinDkvSmem& sm =
      *reinterpret_cast<WinDkvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nitems_g = wkpre[W];
  const int total = nitems_g * hkv;
  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_empty, kCW);
    mbar_init(&sm.pds_full, kCW);
    mbar_init(&sm.pds_empty, 1);
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, kCW);
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
  // TMEM columns: S^T [0,128), dP^T [128,256), P^T w [256,320), dS^T [320,384), dK [384,448), dV [448,512)
  const uint32_t tm_s = tmem, tm_dp = tmem + 128, tm_p = tmem + 256, tm_ds = tmem + 320, tm_dk = tmem + 384,
                 tm_dv = tmem + 448;

  if (warp == kCW) {
    // ---------------- producer: (K, V) per item; gathered Q, dO, row scalars per row tile
    uint32_t kv_count = 0, q_count = 0;
    bool kv_issued = false;
    uint32_t kv_last_par = 0;
    for (int it = blockIdx.x; it < total && !is_aborted(&sm.abort_flag); it += gridDim.x) {
      const WinItem x = win_kitem(it, nitems_g, wkpre, W, wptr);
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&sm.kv_empty, (kv_count & 1) ^ 1);
        if (ok) {
          mbar_expect_tx(&sm.kv_full, 2 * kTile);
          const int row = x.g * (int)N + x.p0 + x.rt * kKT;
          tma_load_2d(sm.k, &kmap, &sm.kv_full, 0, row);
          tma_load_2d(sm.v, &vmap, &sm.kv_full, 0, row);
          kv_last_par = kv_count & 1;
          kv_issued = true;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { timeout_exit(status, &sm.abort_flag); break; }
      ++kv_count;
      const int nrt = (x.nw + TPT - 1) / TPT;
      for (int rt = 0; rt < nrt; ++rt) {
        const int qb = q_count % 2;
        if (lane == 0) ok = mbar_wait(&sm.q_empty[qb], ((q_count / 2) & 1) ^ 1);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { timeout_exit(status, &sm.abort_flag); break; }
        if (lane == 0) mbar_expect_tx_only(&sm.q_full[qb], 2 * kTile + 3 * 128 * 4);  // 3 scalar boxes of G floats x TPT tokens
        __syncwarp();
        const int pp = x.p0 + rt * TPT, nv = x.nw - rt * TPT;
        gather_rows<G>(sm.q[qb], &qmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
        gather_rows<G>(sm.dout[qb], &dmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
        gather_scalars<G>(sm.lse[qb], &lmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
        gather_scalars<G>(sm.Dr[qb], &cmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
        gather_scalars<G>(sm.wr[qb], &wmap, &sm.q_full[qb], wperm, pp, nv, x.g, N, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.q_full[qb]);
        ++q_count;
      }
    }
    if (lane == 0 && kv_issued) mbar_wait(&sm.kv_full, kv_last_par);
  } else if (warp == kCW + 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(kKT, 128);             // S^T, dP^T [keys, rows]
      const uint32_t id_a = idesc_bf16(kKT, 64, false, true);  // dK / dV [keys, 64] += X^T[keys, rows] Y
      uint32_t kv_count = 0, q_count = 0, sdp_count = 0, pds_count = 0, acc_count = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok && !is_aborted(&sm.abort_flag); it += gridDim.x) {
        const WinItem x = win_kitem(it, nitems_g, wkpre, W, wptr);
        if (!mbar_wait(&sm.kv_full, kv_count & 1)) { ok = false; break; }
        ++kv_count;
        const int nrt = (x.nw + TPT - 1) / TPT;
        for (int i = 0; i < nrt; ++i) {
          const int qb = q_count % 2;
          if (!mbar_wait(&sm.q_full[qb], (q_count / 2) & 1) || !mbar_wait(&sm.sdp_empty, (sdp_count & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mma_bf16_ss(tm_s, sdesc_kmajor_sw128(sm.k, 32 * k), sdesc_kmajor_sw128(sm.q[qb], 32 * k), id_s, k > 0);
            mma_bf16_ss(tm_dp, sdesc_kmajor_sw128(sm.v, 32 * k), sdesc_kmajor_sw128(sm.dout[qb], 32 * k), id_s,
                        k > 0);
          }
          mma_commit(&sm.sdp_full);
          ++sdp_count;
          if ((i == 0 && !mbar_wait(&sm.acc_empty, (acc_count & 1) ^ 1)) || !mbar_wait(&sm.pds_full, pds_count & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k) {
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
      if (!ok) timeout_exit(status, &sm.abort_flag);
      mma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0);
    }
  } else {
    // ---------------- compute warps: thread = key; warpgroup wg owns rows [64 wg, 64 wg + 64)
    const int b = threadIdx.x % 128;
    const int wg = warp / 4;
    const int r0 = 64 * wg;
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    uint32_t sdp_count = 0, pds_count = 0, acc_count = 0, q_count = 0;
    for (int it = blockIdx.x; it < total && !is_aborted(&sm.abort_flag); it += gridDim.x) {
      const WinItem x = win_kitem(it, nitems_g, wkpre, W, wptr);
      const int nrt = (x.nw + TPT - 1) / TPT;
      // a warp whose 32 keys all lie past the window skips the arithmetic (its rows of
      // dK / dV are discarded) but keeps the barrier protocol
      const bool active = 32 * (warp % 4) < x.nw - x.rt * kKT;
      bool ok = true;
      for (int i = 0; i < nrt; ++i) {
        const int qb = q_count % 2;
        if (!mbar_wait_warp(&sm.sdp_full, sdp_count & 1)) { ok = false; break; }
        tc_fence_after();
        if (!active) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.sdp_empty);
          ++sdp_count;
          if (!mbar_wait_warp(&sm.pds_empty, (pds_count & 1) ^ 1)) { ok = false; break; }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.pds_full);
          ++pds_count;
          ++q_count;
          continue;
        }
        float sv[64], dp[64];
        tmem_ld32(tm_s + lane_off + r0, sv);
        tmem_ld32(tm_s + lane_off + r0 + 32, sv + 32);
        tmem_ld32(tm_dp + lane_off + r0, dp);
        tmem_ld32(tm_dp + lane_off + r0 + 32, dp + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sdp_empty);
        ++sdp_count;
        if (!mbar_wait_warp(&sm.q_full[qb], (q_count / 2) & 1)) { ok = false; break; }
        const float2 qs = make_float2(qs2, qs2);
        uint32_t pw[32], dsv[32];
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          // 4 consecutive rows share a token (G >= 8): one float4 of its slot of row
          // constants (-lse log2 e, -D, w); rows of tokens past the window were loaded
          // as zeros: w = D = 0 there, so they add nothing
          const int si = scalar_idx(r0 + c, G);
          const float4 l4 = *reinterpret_cast<const float4*>(&sm.lse[qb][si]);
          const float4 d4 = *reinterpret_cast<const float4*>(&sm.Dr[qb][si]);
          const float4 w4 = *reinterpret_cast<const float4*>(&sm.wr[qb][si]);
          const float2 wa = make_float2(w4.x, w4.y), wb = make_float2(w4.z, w4.w);
          const float2 pa = ex2x2(ffma2(make_float2(sv[c], sv[c + 1]), qs, make_float2(l4.x, l4.y)));
          const float2 pb = ex2x2(ffma2(make_float2(sv[c + 2], sv[c + 3]), qs, make_float2(l4.z, l4.w)));
          pw[c / 2] = pack2(fmul2(pa, wa));
          pw[c / 2 + 1] = pack2(fmul2(pb, wb));
          dsv[c / 2] = pack2(fmul2(pa, ffma2(wa, make_float2(dp[c], dp[c + 1]), make_float2(d4.x, d4.y))));
          dsv[c / 2 + 1] = pack2(fmul2(pb, ffma2(wb, make_float2(dp[c + 2], dp[c + 3]), make_float2(d4.z, d4.w))));
        }
        if (!mbar_wait_warp(&sm.pds_empty, (pds_count & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        tmem_st16(tm_p + lane_off + 32 * wg, pw);
        tmem_st16(tm_p + lane_off + 32 * wg + 16, pw + 16);
        tmem_st16(tm_ds + lane_off + 32 * wg, dsv);
        tmem_st16(tm_ds + lane_off + 32 * wg + 16, dsv + 16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.pds_full);
        ++pds_count;
        ++q_count;
      }
      if (!ok) {
        timeout_exit(status, &sm.abort_flag);
        break;
      }
      if (!mbar_wait_warp(&sm.acc_full, acc_count & 1)) { timeout_exit(status, &sm.abort_flag); break; }
      ++acc_count;
      tc_fence_after();
      float acc[64];
      const uint32_t src = (wg == 0 ? tm_dk : tm_dv) + lane_off;
      tmem_ld32(src, acc);
      tmem_ld32(src + 32, acc + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);
      const int kj = x.rt * kKT + b;  // key position inside the window
      if (kj < x.nw) {
        const int64_t tok = wperm[x.p0 + kj];
        float* dst = (wg == 0 ? dk_out : dv_out) + (tok * hkv + x.g) * 64;
        const float mul = wg == 0 ? scale : 1.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float4 c4 = reinterpret_cast<float4*>(dst)[i];
          c4.x += acc[4 * i] * mul;
          c4.y += acc[4 * i + 1] * mul;
          c4.z += acc[4 * i + 2] * mul;
          c4.w += acc[4 * i + 3] * mul;
          reinterpret_cast<float4*>(dst)[i] = c4;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// items: row tiles (forward, dQ) or key tiles (dK/dV) of each window
__global__ void win_plan_kernel(const int32_t* __restrict__ wptr, int64_t W, int per, int32_t* __restrict__ cnt) {
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w <= W; w += (int64_t)gridDim.x * blockDim.x)
    cnt[w] = w == W ? 0 : (wptr[w + 1] - wptr[w] + per - 1) / per;
}

template <int G>
cudaError_t win_fwd_tc_g(const FwdArgs& a, int32_t* cnt, int32_t* pre, int32_t* scan_tmp, cudaStream_t st) {
  const int64_t W = a.win->count, N = a.N;
  CUtensorMap qm, km, vm;
  if (!map_q_token(&qm, a.q, N, a.hq, G) || !map_rows64(&km, a.wks, (int64_t)a.hkv * N) ||
      !map_rows64(&vm, a.wvs, (int64_t)a.hkv * N))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(win_fwd_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(sizeof(WinFwdSmem) + 1024));
    attr = true;
  }
  SSA_LAUNCH("win_plan_kernel", win_plan_kernel, (int)((W + 256) / 256), 256, 0, st, a.win->ptr, W, 128 / G, cnt);
  cudaError_t e = exclusive_scan(cnt, pre, W + 1, scan_tmp, st);
  if (e != cudaSuccess) return e;
  SSA_LAUNCH("win_fwd_tc_kernel", win_fwd_tc_kernel<G>, num_sms(), 192, sizeof(WinFwdSmem) + 1024, st, qm, km, vm,
             a.win->perm, a.win->ptr, pre, W, N, a.hq, a.hkv, a.scale * kLog2e, a.o_branch + 2 * N * a.hq * 64,
             a.lse + 2 * N * a.hq, a.status);
  return cudaGetLastError();
}

template <int G>
cudaError_t win_bwd_tc_g(const BwdArgs& a, int32_t* cnt, int32_t* pre, int32_t* scan_tmp, cudaStream_t st) {
  const int64_t W = a.win->count, N = a.N;
  const int64_t rows = N * a.hq;
  CUtensorMap qm, dm, km, vm, lm, cm, wm;
  if (!map_q_token(&qm, a.q, N, a.hq, G) || !map_q_token(&dm, a.dout, N, a.hq, G) ||
      !map_rows64(&km, a.wks, (int64_t)a.hkv * N) || !map_rows64(&vm, a.wvs, (int64_t)a.hkv * N) ||
      !map_rowscalars_token(&lm, a.rc + 3 * rows, N, a.hq, G) ||  // -lse log2(e) of the window branch
      !map_rowscalars_token(&cm, a.rc + 5 * rows, N, a.hq, G) ||  // -D
      !map_rowscalars_token(&wm, a.rc + 4 * rows, N, a.hq, G))    // w
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(win_bwd_dq_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(sizeof(WinDqSmem) + 1024));
    cudaFuncSetAttribute(win_bwd_dkv_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(sizeof(WinDkvSmem) + 1024));
    attr = true;
  }
  const float qs2 = a.scale * kLog2e;
  SSA_LAUNCH("win_plan_kernel", win_plan_kernel, (int)((W + 256) / 256), 256, 0, st, a.win->ptr, W, 128 / G, cnt);
  cudaError_t e = exclusive_scan(cnt, pre, W + 1, scan_tmp, st);
  if (e != cudaSuccess) return e;
  SSA_LAUNCH("win_bwd_dq_tc_kernel", win_bwd_dq_tc_kernel<G>, num_sms(), 192, sizeof(WinDqSmem) + 1024, st, qm, dm,
             km, vm, lm, cm, wm, a.win->perm, a.win->ptr, pre, W, N, a.hq, a.hkv, qs2, a.scale, a.dq, a.status);
  SSA_LAUNCH("win_plan_kernel", win_plan_kernel, (int)((W + 256) / 256), 256, 0, st, a.win->ptr, W, kKT, cnt);
  e = exclusive_scan(cnt, pre, W + 1, scan_tmp, st);
  if (e != cudaSuccess) return e;
  SSA_LAUNCH("win_bwd_dkv_tc_kernel", win_bwd_dkv_tc_kernel<G>, num_sms(), 32 * (kCW + 2), sizeof(WinDkvSmem) + 1024,
             st, qm, dm, km, vm, lm, cm, wm, a.win->perm, a.win->ptr, pre, W, N, a.hq, a.hkv, qs2, a.scale, a.wdk,
             a.wdv, a.status);
  return cudaGetLastError();
}

}  // namespace
}  // namespace ssa

namespace ssa {
bool win_tc_supported(int dtype, int d, int hq, int hkv, int m_cmp, int m_win) {
  const int G = hkv > 0 ? hq / hkv : 0;
  return dtype == SSA_DTYPE_BF16 && d == 64 && (G == 8 || G == 16) && m_cmp == m_win && tch::encode_fn() != nullptr;
}
cudaError_t win_fwd_tc(const FwdArgs& a, int32_t* cnt, int32_t* pre, int32_t* scan_tmp, cudaStream_t st) {
  const int G = a.hq / a.hkv;
  return G == 16 ? win_fwd_tc_g<16>(a, cnt, pre, scan_tmp, st) : win_fwd_tc_g<8>(a, cnt, pre, scan_tmp, st);
}
cudaError_t win_bwd_tc(const BwdArgs& a, int32_t* cnt, int32_t* pre, int32_t* scan_tmp, cudaStream_t st) {
  const int G = a.hq / a.hkv;
  return G == 16 ? win_bwd_tc_g<16>(a, cnt, pre, scan_tmp, st) : win_bwd_tc_g<8>(a, cnt, pre, scan_tmp, st);
}
}  // namespace ssa
