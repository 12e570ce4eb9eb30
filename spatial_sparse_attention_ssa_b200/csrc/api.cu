// C ABI of libssa: argument checks, workspace layout and launch order.
#include <math.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace {

// Device check word (or of ssa::kStatus* bits), read and cleared by the host.
__device__ int g_ssa_status;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Carver {
  char* p;
  size_t used = 0;
  explicit Carver(void* base) : p(static_cast<char*>(base)) {}
  template <typename T>
  T* take(size_t count) {
    T* r = reinterpret_cast<T*>(p ? p + used : nullptr);
    used += align256(sizeof(T) * (count > 0 ? count : 1));
    return r;
  }
};

int* status_ptr() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_ssa_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(ptr);
}

ssa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA; }

// SSA_DISABLE_TC=1 selects the fp32 SIMT kernels for every shape (cross-checks).
bool tc_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("SSA_DISABLE_TC");
    v = (e && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}

ssa_status check_params(const ssa_params* p) {
  if (!p) return SSA_ERR_INVALID_ARG;
  if (p->hq < 1 || p->hkv < 1 || p->hq % p->hkv != 0) return SSA_ERR_INVALID_ARG;
  if (p->m_cmp < 1 || p->m_win < 1 || p->topk < 1) return SSA_ERR_INVALID_ARG;
  if (p->dtype != SSA_DTYPE_BF16 && p->dtype != SSA_DTYPE_F32) return SSA_ERR_INVALID_ARG;
  if (p->gate_mode != SSA_GATE_WEIGHTS && p->gate_mode != SSA_GATE_LOGITS) return SSA_ERR_INVALID_ARG;
  if (p->selection != SSA_SEL_SCORES && p->selection != SSA_SEL_GIVEN) return SSA_ERR_INVALID_ARG;
  if (p->conv && (!p->conv->coords || !p->conv->wk || !p->conv->bk || !p->conv->wv || !p->conv->bv))
    return SSA_ERR_INVALID_ARG;
  if (!(p->scale >= 0.f) || isinf(p->scale)) return SSA_ERR_INVALID_ARG;
  if (p->d != 32 && p->d != 64 && p->d != 128) return SSA_ERR_UNSUPPORTED;
  if (p->topk > 32) return SSA_ERR_UNSUPPORTED;
  const int G = p->hq / p->hkv;
  if (G & (G - 1)) return SSA_ERR_UNSUPPORTED;  // power of two
  if (G * (p->d / 32) > 32) return SSA_ERR_UNSUPPORTED;
  if (p->conv && p->hkv * p->d > 256) return SSA_ERR_UNSUPPORTED;
  if (!ssa::pool_supported(p->dtype, p->hkv, p->d)) return SSA_ERR_UNSUPPORTED;
  if (p->deterministic != 0 && p->deterministic != 1) return SSA_ERR_INVALID_ARG;
  if (p->deterministic &&
      (p->conv || !tc_enabled() || !ssa::cmp_tc_supported(p->dtype, p->d, p->hq, p->hkv, p->topk) ||
       !ssa::slc_mma_supported(p->dtype, p->d, p->hq, p->hkv, p->topk)))
    return SSA_ERR_UNSUPPORTED;  // the fixed-point sums are built into the tensor-core backward
  return SSA_OK;
}

// The per-token arrays (id, perm) and the cell keys may be null when there are no
// tokens: nothing is written to them then.  ptr and cu are always written.
bool partition_ok(const ssa_partition* x, int64_t n) {
  return x && x->ptr && x->cu && x->count >= 0 && (n == 0 || (x->id && x->perm && x->key));
}

float eff_scale(const ssa_params* p) { return p->scale > 0.f ? p->scale : 1.f / sqrtf((float)p->d); }

// Workspace of the forward (after `ws` base): plan arrays.
void carve_plan(Carver& c, int32_t S, int32_t** tc, int32_t** tp, int32_t** ic, int32_t** ip, int32_t** st) {
  *tc = c.take<int32_t>(S + 1);
  *tp = c.take<int32_t>(S + 1);
  *ic = c.take<int32_t>(S + 1);
  *ip = c.take<int32_t>(S + 1);
  *st = c.take<int32_t>(ssa::scan_tmp_ints(S + 1));
}

size_t bin_bytes(int32_t S, int64_t N) { return ssa::bin_ws_bytes(S, N) + 256; }

size_t fwd_bytes(const ssa_params* p, int32_t S, int64_t N, int64_t B, int64_t W, float** imp = nullptr,
                 int32_t** wc = nullptr, int32_t** wp = nullptr, int32_t** wst = nullptr, void* base = nullptr) {
  (void)N;
  Carver c(base);
  int32_t *a, *b, *d, *e, *f;
  carve_plan(c, S, &a, &b, &d, &e, &f);
  float* x = c.take<float>(ssa::cmp_tc_scratch_floats(p->hq, p->hkv, B));
  int32_t* y0 = c.take<int32_t>(W + 1);
  int32_t* y1 = c.take<int32_t>(W + 1);
  int32_t* y2 = c.take<int32_t>(ssa::scan_tmp_ints(W + 1));
  if (imp) *imp = x;
  if (wc) *wc = y0;
  if (wp) *wp = y1;
  if (wst) *wst = y2;
  return c.used;
}

// Learned-compression region after the regular workspace (0 without it).
size_t conv_bytes(const ssa_params* p, int64_t N, int64_t B) {
  return p->conv ? align256(sizeof(float) * ssa::conv_ws_floats(N, B, p->hkv, p->d, p->m_cmp)) + 256 : 0;
}

// Learned-compression arguments over the region at `base`.
ssa::ConvArgs conv_args(const ssa_params* p, const ssa_partition* blk, int32_t S, int64_t N, void* base) {
  ssa::ConvArgs c;
  const ssa_conv* cv = p->conv;
  c.coords = cv->coords;
  c.blk = blk;
  c.S = S;
  c.N = N;
  c.hkv = p->hkv;
  c.d = p->d;
  c.m = p->m_cmp;
  c.wk = cv->wk;
  c.bk = cv->bk;
  c.wv = cv->wv;
  c.bv = cv->bv;
  c.dwk = cv->dwk;
  c.dbk = cv->dbk;
  c.dwv = cv->dwv;
  c.dbv = cv->dbv;
  char* b = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(base) + 255) & ~uintptr_t(255));
  c.cs = reinterpret_cast<int4*>(b);
  c.M = reinterpret_cast<float*>(b + align256(sizeof(int4) * (size_t)N));
  c.dM = c.M + 2 * (size_t)blk->count * p->hkv * 27 * p->d;
  c.table = reinterpret_cast<int*>(c.dM + 2 * (size_t)blk->count * p->hkv * 27 * p->d);
  return c;
}

// Cross-attention extras after the regular workspace: the gates widened to three
// columns (the kernels read gates with a row stride of 3) and one check word.
size_t cross_extra_bytes(int64_t Nq, int hq) { return align256(sizeof(float) * 3 * (size_t)Nq * hq) + 256; }

// Sequence-parallel extras after the regular workspace: the rank's window means
// (forward; [Hkv, W, d] each for K and V) or its window key gradients (backward;
// [Nr, Hkv, d] fp32 each).
size_t sp_fwd_extra(const ssa_params* p, int64_t W) {
  return 2 * align256((size_t)p->hkv * (W > 0 ? W : 1) * p->d * (p->dtype == SSA_DTYPE_BF16 ? 2 : 4)) + 256;
}
size_t sp_bwd_extra(const ssa_params* p, int64_t Nr) {
  return 2 * align256(sizeof(float) * (size_t)(Nr > 0 ? Nr : 1) * p->hkv * p->d) + 256;
}

struct BwdWs {
  unsigned long long *fx_kc, *fx_vc, *fx_k, *fx_v;
  void *q16, *do16, *kc16, *vc16;
  float* Dc;
  float* rc;
  float *dkc, *dvc;
  uint64_t *ka, *kb;
  int32_t *va, *vb, *inv_ptr, *radix_tmp, *slc_cnt, *slc_pre, *win_cnt, *win_pre;
  int32_t *tc, *tp, *ic, *ip, *st;
};

size_t carve_bwd(void* base, const ssa_params* p, int32_t S, int64_t N, int64_t B, int64_t W, BwdWs* w) {
  Carver c(base);
  const int64_t nsel = N * p->hkv * p->topk;
  w->Dc = c.take<float>(3 * N * p->hq);
  w->rc = c.take<float>(6 * N * p->hq);
  w->dkc = c.take<float>(p->hkv * B * p->d);
  w->dvc = c.take<float>(p->hkv * B * p->d);
  w->ka = c.take<uint64_t>(nsel);
  w->kb = c.take<uint64_t>(nsel);
  w->va = c.take<int32_t>(nsel);
  w->vb = c.take<int32_t>(nsel);
  w->inv_ptr = c.take<int32_t>(p->hkv * B + 1);
  w->radix_tmp = c.take<int32_t>(ssa::radix_tmp_ints(nsel));
  w->slc_cnt = c.take<int32_t>(p->hkv * B + 1);
  w->slc_pre = c.take<int32_t>(p->hkv * B + 1);
  w->win_cnt = c.take<int32_t>(W + 1);
  w->win_pre = c.take<int32_t>(W + 1);
  int64_t mx = p->hkv * B + 1 > S + 1 ? p->hkv * B + 1 : S + 1;
  mx = mx > W + 1 ? mx : W + 1;
  w->st = c.take<int32_t>(ssa::scan_tmp_ints(mx));
  int32_t* unused_st;
  carve_plan(c, S, &w->tc, &w->tp, &w->ic, &w->ip, &unused_st);
  if (p->deterministic) {  // 64-bit fixed-point sums: dKc / dVc [Hkv, B, d], dK / dV [N, Hkv, d]
    w->fx_kc = c.take<unsigned long long>(p->hkv * B * p->d);
    w->fx_vc = c.take<unsigned long long>(p->hkv * B * p->d);
    w->fx_k = c.take<unsigned long long>(N * p->hkv * p->d);
    w->fx_v = c.take<unsigned long long>(N * p->hkv * p->d);
  } else {
    w->fx_kc = w->fx_vc = w->fx_k = w->fx_v = nullptr;
  }
  if (ssa::cmp_tc_supported(p->dtype, p->d, p->hq, p->hkv, p->topk)) {
    // fp16 operands of the tensor-core dKc / dVc kernel: Q, dO [N, Hq, d], Kc, Vc [Hkv, B, d]
    w->q16 = c.take<uint16_t>(N * p->hq * p->d);
    w->do16 = c.take<uint16_t>(N * p->hq * p->d);
    w->kc16 = c.take<uint16_t>(p->hkv * B * p->d);
    w->vc16 = c.take<uint16_t>(p->hkv * B * p->d);
  } else {
    w->q16 = w->do16 = w->kc16 = w->vc16 = nullptr;
  }
  return c.used;
}

}  // namespace

extern "C" {

SSA_API int32_t ssa_version(void) { return 100; }

SSA_API const char* ssa_error_string(ssa_status s) {
  switch (s) {
    case SSA_OK: return "ok";
    case SSA_ERR_INVALID_ARG: return "invalid argument";
    case SSA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case SSA_ERR_WORKSPACE: return "workspace too small";
    case SSA_ERR_COORD_RANGE: return "coordinate outside [0, R) or malformed cu_seqlens";
    case SSA_ERR_CUDA: return "CUDA error";
    case SSA_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

SSA_API size_t ssa_workspace_size(int32_t op, const ssa_params* p, int32_t S, int64_t N, int64_t B_tot,
                                  int64_t W_tot) {
  if (S < 0 || N < 0 || B_tot < 0 || W_tot < 0) return 0;
  if (op == SSA_OP_BIN) return bin_bytes(S, N);
  if (op == SSA_OP_GEO_SELECT) return ssa::geo_ws_bytes(N);
  if (check_params(p) != SSA_OK) return 0;
  if (op == SSA_OP_FORWARD) return fwd_bytes(p, S, N, B_tot, W_tot) + conv_bytes(p, N, B_tot);
  if (op == SSA_OP_BACKWARD) {
    BwdWs w;
    return carve_bwd(nullptr, p, S, N, B_tot, W_tot, &w) + conv_bytes(p, N, B_tot);
  }
  // a sequence-parallel rank: N = its tokens, W_tot = its windows
  if (op == SSA_OP_SP_FORWARD) return fwd_bytes(p, S, N, B_tot, W_tot) + sp_fwd_extra(p, W_tot);
  if (op == SSA_OP_SP_BACKWARD) {
    BwdWs w;
    return carve_bwd(nullptr, p, S, N, B_tot, W_tot, &w) + sp_bwd_extra(p, N);
  }
  // cross attention: N = query tokens, W_tot unused (no window branch)
  if (op == SSA_OP_CROSS_FORWARD) return fwd_bytes(p, S, N, B_tot, 0) + cross_extra_bytes(N, p->hq);
  if (op == SSA_OP_CROSS_BACKWARD) {
    BwdWs w;
    return carve_bwd(nullptr, p, S, N, B_tot, 0, &w) + cross_extra_bytes(N, p->hq);
  }
  return 0;
}

SSA_API ssa_status ssa_geo_select(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N, int32_t R,
                                  const ssa_partition* blk, int32_t m_cmp, int32_t topk, int32_t hkv, int32_t* sel,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (S < 1 || N < 0 || N > INT32_MAX - 1 || R < 1 || m_cmp < 1 || topk < 1 || topk > 32 || hkv < 1)
    return SSA_ERR_INVALID_ARG;
  if (R > 32768) return SSA_ERR_UNSUPPORTED;  // squared distances must fit 32 bits
  if (N == 0) return SSA_OK;
  if (!coords || !cu_seqlens || !partition_ok(blk, N) || !sel || !ws) return SSA_ERR_INVALID_ARG;
  if (blk->count < 1 || blk->count > N) return SSA_ERR_INVALID_ARG;
  if (ws_bytes < ssa::geo_ws_bytes(N)) return SSA_ERR_WORKSPACE;
  return cuda_status(ssa::geo_select(coords, cu_seqlens, S, N, blk, m_cmp, topk, hkv, sel, ws,
                                     static_cast<cudaStream_t>(stream)));
}

SSA_API ssa_status ssa_diag_wait_timeout(int32_t* gave_up, void* stream) {
  if (!gave_up) return SSA_ERR_INVALID_ARG;
  int* sp = status_ptr();
  if (!sp) return SSA_ERR_CUDA;
  return cuda_status(ssa::diag_wait_timeout(sp, gave_up, static_cast<cudaStream_t>(stream)));
}

SSA_API ssa_status ssa_diag_ex2(const float* x, float* y_poly, float* y_mufu, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_mufu))) return SSA_ERR_INVALID_ARG;
  return cuda_status(ssa::diag_ex2(x, y_poly, y_mufu, n, static_cast<cudaStream_t>(stream)));
}

SSA_API ssa_status ssa_get_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* sp = status_ptr();
  if (!sp) return SSA_ERR_CUDA;
  int32_t hv[3];
  if (ssa::read_ints_to_host(sp, nullptr, nullptr, hv, st) != cudaSuccess) return SSA_ERR_CUDA;
  const int h = hv[0];
  if (h) {
    cudaMemsetAsync(sp, 0, sizeof(int), st);
    cudaStreamSynchronize(st);
  }
  if (h & ssa::kStatusTimeout) return SSA_ERR_TIMEOUT;
  if (h & (ssa::kStatusCoordRange | ssa::kStatusSeqlens)) return SSA_ERR_COORD_RANGE;
  if (h & ssa::kStatusSelection) return SSA_ERR_INVALID_ARG;
  return SSA_OK;
}

SSA_API ssa_status ssa_pool(int32_t dtype, int32_t hkv, int32_t d, int64_t N, const ssa_partition* blk,
                            const void* k, const void* v, void* ks, void* vs, void* kc, void* vc, void* stream) {
  if ((dtype != SSA_DTYPE_BF16 && dtype != SSA_DTYPE_F32) || hkv < 1 || d < 1 || N < 0 || N > INT32_MAX - 1)
    return SSA_ERR_INVALID_ARG;
  if (!ssa::pool_supported(dtype, hkv, d)) return SSA_ERR_UNSUPPORTED;
  if (N == 0) return SSA_OK;
  if (!partition_ok(blk, N) || blk->count < 1 || blk->count > N || !k || !v || !ks || !vs || !kc || !vc)
    return SSA_ERR_INVALID_ARG;
  for (const void* x : {k, v, (const void*)ks, (const void*)vs, (const void*)kc, (const void*)vc})
    if (reinterpret_cast<uintptr_t>(x) % 16 != 0) return SSA_ERR_INVALID_ARG;
  return cuda_status(ssa::launch_pool(dtype, k, v, blk, N, hkv, d, ks, vs, kc, vc, static_cast<cudaStream_t>(stream)));
}

SSA_API ssa_status ssa_bin(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N, int32_t R,
                           int32_t m_cmp, int32_t m_win, ssa_partition* blk, ssa_partition* win, void* ws,
                           size_t ws_bytes, void* stream) {
  if (S < 1 || N < 0 || N > INT32_MAX - 1 || R < 1 || R > (1 << 20) || m_cmp < 1 || m_win < 1)
    return SSA_ERR_INVALID_ARG;
  if (!cu_seqlens || (N > 0 && !coords) || !partition_ok(blk, N) || !partition_ok(win, N) || !ws)
    return SSA_ERR_INVALID_ARG;
  if (ws_bytes < bin_bytes(S, N)) return SSA_ERR_WORKSPACE;
  int sbits = 0;
  while ((1ll << sbits) < S) ++sbits;
  for (int m : {m_cmp, m_win}) {
    int cbits = 1;
    while ((1ll << cbits) < (R + m - 1) / m) ++cbits;
    if (sbits + 3 * cbits > 64) return SSA_ERR_UNSUPPORTED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* sp = status_ptr();
  if (!sp) return SSA_ERR_CUDA;
  int32_t* d_counts = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + ssa::bin_ws_bytes(S, N));
  cudaError_t e = ssa::bin_partition(coords, cu_seqlens, S, N, R, m_cmp, blk, d_counts, ws, sp, st);
  if (e != cudaSuccess) return SSA_ERR_CUDA;
  if (m_win == m_cmp) {
    e = cudaMemcpyAsync(win->id, blk->id, sizeof(int32_t) * N, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(win->perm, blk->perm, sizeof(int32_t) * N, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(win->ptr, blk->ptr, sizeof(int32_t) * (N + 1), cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(win->cu, blk->cu, sizeof(int32_t) * (S + 1), cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && N > 0)
      e = cudaMemcpyAsync(win->key, blk->key, sizeof(int32_t) * 3 * N, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_counts + 1, d_counts, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
  } else {
    e = ssa::bin_partition(coords, cu_seqlens, S, N, R, m_win, win, d_counts + 1, ws, sp, st);
  }
  if (e != cudaSuccess) return SSA_ERR_CUDA;
  int32_t hv[3];
  if (ssa::read_ints_to_host(d_counts, d_counts + 1, sp, hv, st) != cudaSuccess) return SSA_ERR_CUDA;
  blk->count = hv[0];
  win->count = hv[1];
  const int h_status = hv[2];
  if (h_status) {
    cudaMemsetAsync(sp, 0, sizeof(int), st);
    cudaStreamSynchronize(st);
    return (h_status & ssa::kStatusTimeout) ? SSA_ERR_TIMEOUT : SSA_ERR_COORD_RANGE;
  }
  return SSA_OK;
}

}  // extern "C"

namespace {

// The forward of the self-attention path (cross == 0: queries are the voxel tokens,
// Nkv == N, three branches) and of the cross-attention path (cross == 1: queries of
// another token set, keys / values the Nkv voxel tokens, no window branch, gates
// already widened to 3 columns).
ssa_status forward_common(const ssa_params* p, const int32_t* cu, int32_t S, int64_t N, int64_t Nkv, int cross,
                          const ssa_partition* blk, const ssa_partition* win, const void* q, const void* k,
                          const void* v, const float* gates, void* out, const ssa_saved* saved, void* ws,
                          cudaStream_t st, const ssa_sp_local* sp = nullptr) {
  cudaError_t e = ssa::launch_pool(p->dtype, k, v, blk, Nkv, p->hkv, p->d, saved->ks, saved->vs, saved->kc,
                                   saved->vc, st);
  if (e != cudaSuccess) return SSA_ERR_CUDA;
  if (p->conv) {  // learned compression: Kc / Vc from the convolution instead of the plain mean
    const ssa::ConvArgs c = conv_args(p, blk, S, Nkv, static_cast<char*>(ws) + fwd_bytes(p, S, N, blk->count,
                                                                                           win ? win->count : 0));
    if (ssa::conv_forward(c, p->dtype, k, v, saved->kc, saved->vc, st) != cudaSuccess) return SSA_ERR_CUDA;
  }
  ssa::FwdArgs a;
  a.dtype = p->dtype;
  a.d = p->d;
  a.hq = p->hq;
  a.hkv = p->hkv;
  a.topk = p->topk;
  a.gate_mode = p->gate_mode;
  a.sel_given = p->selection == SSA_SEL_GIVEN;
  a.cross = cross;
  a.Nkv = Nkv;
  a.m_cmp = p->m_cmp;
  a.m_win = p->m_win;
  a.use_tc = tc_enabled();
  a.status = status_ptr();
  if (!a.status) return SSA_ERR_CUDA;
  a.scale = eff_scale(p);
  a.S = S;
  a.N = N;
  a.cu_seqlens = cu;
  a.blk = blk;
  a.win = win;
  a.q = q;
  a.k = k;
  a.v = v;
  a.gates = gates;
  a.out = out;
  a.kc = saved->kc;
  a.vc = saved->vc;
  a.ks = saved->ks;
  a.vs = saved->vs;
  a.o_branch = saved->o_branch;
  a.lse = saved->lse;
  a.sel = saved->sel;
  a.has_win = !cross;
  a.wk = k;
  a.wv = v;
  a.wks = saved->ks;
  a.wvs = saved->vs;
  Carver c(ws);
  carve_plan(c, S, &a.tiles_cnt, &a.tiles_pre, &a.items_cnt, &a.items_pre, &a.scan_tmp);
  int32_t* win_scan = nullptr;
  fwd_bytes(p, S, N, blk->count, win ? win->count : 0, &a.imp_scratch, &a.win_cnt, &a.win_pre, &win_scan, ws);
  a.win_scan = win_scan;
  if (sp) {  // a sequence-parallel rank: the window problem is its own tokens
    a.has_win = 1;
    a.win = sp->win;
    a.wk = sp->k;
    a.wv = sp->v;
    a.wks = sp->ks;
    a.wvs = sp->vs;
    // their window-ordered copies (the window means land in the scratch after the workspace)
    char* wsc = static_cast<char*>(ws) + fwd_bytes(p, S, N, blk->count, sp->win->count);
    void* wkc = wsc;
    void* wvc = wsc + align256((size_t)p->hkv * sp->win->count * p->d * (p->dtype == SSA_DTYPE_BF16 ? 2 : 4));
    e = ssa::launch_pool(p->dtype, sp->k, sp->v, sp->win, N, p->hkv, p->d, sp->ks, sp->vs, wkc, wvc, st);
    if (e != cudaSuccess) return SSA_ERR_CUDA;
  }
  return cuda_status(ssa::simt_forward(a, st));
}

ssa_status backward_common(const ssa_params* p, const int32_t* cu, int32_t S, int64_t N, int64_t Nkv, int cross,
                           const ssa_partition* blk, const ssa_partition* win, const void* q, const void* k,
                           const void* v, const float* gates, const ssa_saved* saved, const void* dout, float* dq,
                           float* dk, float* dv, float* dgates, void* ws, cudaStream_t st,
                           const ssa_sp_local* sp = nullptr, float* sp_wdk = nullptr, float* sp_wdv = nullptr) {
  BwdWs w;
  const size_t used = carve_bwd(ws, p, S, N, blk->count, win ? win->count : 0, &w);
  ssa::ConvArgs conv;
  if (p->conv) conv = conv_args(p, blk, S, Nkv, static_cast<char*>(ws) + used);
  ssa::BwdArgs a;
  a.conv = p->conv ? &conv : nullptr;
  a.dtype = p->dtype;
  a.d = p->d;
  a.hq = p->hq;
  a.hkv = p->hkv;
  a.topk = p->topk;
  a.gate_mode = p->gate_mode;
  a.cross = cross;
  a.Nkv = Nkv;
  a.m_cmp = p->m_cmp;
  a.m_win = p->m_win;
  a.use_tc = tc_enabled();
  a.status = status_ptr();
  if (!a.status) return SSA_ERR_CUDA;
  a.scale = eff_scale(p);
  a.S = S;
  a.N = N;
  a.cu_seqlens = cu;
  a.blk = blk;
  a.win = win;
  a.q = q;
  a.k = k;
  a.v = v;
  a.gates = gates;
  a.kc = saved->kc;
  a.vc = saved->vc;
  a.ks = saved->ks;
  a.vs = saved->vs;
  a.o_branch = saved->o_branch;
  a.lse = saved->lse;
  a.sel = saved->sel;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dgates = dgates;
  a.Dc = w.Dc;
  a.rc = w.rc;
  a.win_cnt = w.win_cnt;
  a.win_pre = w.win_pre;
  a.dkc = w.dkc;
  a.dvc = w.dvc;
  a.inv_keys_a = w.ka;
  a.inv_keys_b = w.kb;
  a.inv_vals_a = w.va;
  a.inv_vals_b = w.vb;
  a.inv_ptr = w.inv_ptr;
  a.radix_tmp = w.radix_tmp;
  a.slc_cnt = w.slc_cnt;
  a.slc_pre = w.slc_pre;
  a.tiles_cnt = w.tc;
  a.tiles_pre = w.tp;
  a.items_cnt = w.ic;
  a.items_pre = w.ip;
  a.scan_tmp = w.st;
  a.q16 = w.q16;
  a.do16 = w.do16;
  a.kc16 = w.kc16;
  a.vc16 = w.vc16;
  a.has_win = !cross;
  a.wk = k;
  a.wv = v;
  a.wks = saved->ks;
  a.wvs = saved->vs;
  a.wdk = dk;
  a.wdv = dv;
  a.wtok = nullptr;
  a.fx_kc = w.fx_kc;
  a.fx_vc = w.fx_vc;
  a.fx_k = w.fx_k;
  a.fx_v = w.fx_v;
  if (sp) {  // a sequence-parallel rank: the window problem is its own tokens
    a.has_win = 1;
    a.wk = sp->k;
    a.wv = sp->v;
    a.wks = sp->ks;
    a.wvs = sp->vs;
    a.win = sp->win;
    a.wdk = sp_wdk;
    a.wdv = sp_wdv;
    a.wtok = sp->tokens;
  }
  return cuda_status(ssa::simt_backward(a, st));
}

bool saved_ok(const ssa_saved* s) {
  return s && s->kc && s->vc && s->ks && s->vs && s->o_branch && s->lse && s->sel;
}

// Widen the gates and check that every sequence with queries has voxel tokens;
// synchronises the stream once to read the check.
ssa_status cross_prepare(const ssa_params* p, const int32_t* q_cu, int32_t S, int64_t Nq, const ssa_partition* blk,
                         const float* gates, void* extra, float** gates3, cudaStream_t st) {
  *gates3 = static_cast<float*>(extra);
  int* bad = reinterpret_cast<int*>(static_cast<char*>(extra) + align256(sizeof(float) * 3 * (size_t)Nq * p->hq));
  if (cudaMemsetAsync(bad, 0, sizeof(int), st) != cudaSuccess) return SSA_ERR_CUDA;
  if (ssa::cross_prep(gates, Nq * p->hq, *gates3, q_cu, blk->cu, S, bad, st) != cudaSuccess) return SSA_ERR_CUDA;
  int32_t hv[3];
  if (ssa::read_ints_to_host(bad, nullptr, nullptr, hv, st) != cudaSuccess) return SSA_ERR_CUDA;
  return hv[0] ? SSA_ERR_INVALID_ARG : SSA_OK;
}

}  // namespace

extern "C" {

SSA_API ssa_status ssa_forward(const ssa_params* p, const int32_t* cu_seqlens, int32_t S, int64_t N,
                               const ssa_partition* blk, const ssa_partition* win, const void* q, const void* k,
                               const void* v, const float* gates, void* out, const ssa_saved* saved, void* ws,
                               size_t ws_bytes, void* stream) {
  ssa_status ps = check_params(p);
  if (ps != SSA_OK) return ps;
  if (S < 1 || N < 0 || N > INT32_MAX - 1 || !cu_seqlens || !partition_ok(blk, N) || !partition_ok(win, N) || !saved)
    return SSA_ERR_INVALID_ARG;
  if (N == 0) return SSA_OK;
  if (!q || !k || !v || !gates || !out || !saved_ok(saved) || !ws) return SSA_ERR_INVALID_ARG;
  if (blk->count < 1 || blk->count > N || win->count < 1 || win->count > N) return SSA_ERR_INVALID_ARG;
  if (ws_bytes < fwd_bytes(p, S, N, blk->count, win->count) + conv_bytes(p, N, blk->count)) return SSA_ERR_WORKSPACE;
  return forward_common(p, cu_seqlens, S, N, N, 0, blk, win, q, k, v, gates, out, saved, ws,
                        static_cast<cudaStream_t>(stream));
}

SSA_API ssa_status ssa_backward(const ssa_params* p, const int32_t* cu_seqlens, int32_t S, int64_t N,
                                const ssa_partition* blk, const ssa_partition* win, const void* q, const void* k,
                                const void* v, const float* gates, const ssa_saved* saved, const void* dout,
                                float* dq, float* dk, float* dv, float* dgates, void* ws, size_t ws_bytes,
                                void* stream) {
  ssa_status ps = check_params(p);
  if (ps != SSA_OK) return ps;
  if (S < 1 || N < 0 || N > INT32_MAX - 1 || !cu_seqlens || !partition_ok(blk, N) || !partition_ok(win, N) || !saved)
    return SSA_ERR_INVALID_ARG;
  if (N == 0) return SSA_OK;
  if (!q || !k || !v || !gates || !dout || !dq || !dk || !dv || !dgates || !saved_ok(saved) || !ws)
    return SSA_ERR_INVALID_ARG;
  if (blk->count < 1 || blk->count > N || win->count < 1 || win->count > N) return SSA_ERR_INVALID_ARG;
  if ((int64_t)N * p->hkv * p->topk > INT32_MAX) return SSA_ERR_UNSUPPORTED;
  BwdWs w;
  if (ws_bytes < carve_bwd(nullptr, p, S, N, blk->count, win->count, &w) + conv_bytes(p, N, blk->count))
    return SSA_ERR_WORKSPACE;
  if (p->conv && (!p->conv->dwk || !p->conv->dbk || !p->conv->dwv || !p->conv->dbv)) return SSA_ERR_INVALID_ARG;
  return backward_common(p, cu_seqlens, S, N, N, 0, blk, win, q, k, v, gates, saved, dout, dq, dk, dv, dgates, ws,
                         static_cast<cudaStream_t>(stream));
}

SSA_API ssa_status ssa_cross_forward(const ssa_params* p, const int32_t* q_cu, int32_t S, int64_t Nq, int64_t Nkv,
                                     const ssa_partition* blk, const void* q, const void* k, const void* v,
                                     const float* gates, void* out, const ssa_saved* saved, void* ws,
                                     size_t ws_bytes, void* stream) {
  ssa_status ps = check_params(p);
  if (ps != SSA_OK) return ps;
  if (S < 1 || Nq < 0 || Nq > INT32_MAX - 1 || Nkv < 0 || Nkv > INT32_MAX - 1 || !q_cu || !partition_ok(blk, Nkv) ||
      !saved)
    return SSA_ERR_INVALID_ARG;
  if (p->conv) return SSA_ERR_UNSUPPORTED;  // the learned compression is built for self attention
  if (Nq == 0) return SSA_OK;
  if (Nkv < 1 || !q || !k || !v || !gates || !out || !saved_ok(saved) || !ws) return SSA_ERR_INVALID_ARG;
  if (blk->count < 1 || blk->count > Nkv) return SSA_ERR_INVALID_ARG;
  const size_t base = fwd_bytes(p, S, Nq, blk->count, 0);
  if (ws_bytes < base + cross_extra_bytes(Nq, p->hq)) return SSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* gates3 = nullptr;
  ps = cross_prepare(p, q_cu, S, Nq, blk, gates, static_cast<char*>(ws) + base, &gates3, st);
  if (ps != SSA_OK) return ps;
  return forward_common(p, q_cu, S, Nq, Nkv, 1, blk, nullptr, q, k, v, gates3, out, saved, ws, st);
}

SSA_API ssa_status ssa_cross_backward(const ssa_params* p, const int32_t* q_cu, int32_t S, int64_t Nq, int64_t Nkv,
                                      const ssa_partition* blk, const void* q, const void* k, const void* v,
                                      const float* gates, const ssa_saved* saved, const void* dout, float* dq,
                                      float* dk, float* dv, float* dgates, void* ws, size_t ws_bytes,
                                      void* stream) {
  ssa_status ps = check_params(p);
  if (ps != SSA_OK) return ps;
  if (S < 1 || Nq < 0 || Nq > INT32_MAX - 1 || Nkv < 0 || Nkv > INT32_MAX - 1 || !q_cu || !partition_ok(blk, Nkv) ||
      !saved)
    return SSA_ERR_INVALID_ARG;
  if (p->conv || p->deterministic) return SSA_ERR_UNSUPPORTED;  // both are built for ssa_backward
  if (Nkv > 0 && dk && dv && Nq == 0) {  // no queries: the key gradients are zero
    cudaStream_t st0 = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(dk, 0, sizeof(float) * Nkv * p->hkv * p->d, st0) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, sizeof(float) * Nkv * p->hkv * p->d, st0) != cudaSuccess)
      return SSA_ERR_CUDA;
    return SSA_OK;
  }
  if (Nq == 0) return SSA_OK;
  if (Nkv < 1 || !q || !k || !v || !gates || !dout || !dq || !dk || !dv || !dgates || !saved_ok(saved) || !ws)
    return SSA_ERR_INVALID_ARG;
  if (blk->count < 1 || blk->count > Nkv) return SSA_ERR_INVALID_ARG;
  if ((int64_t)Nq * p->hkv * p->topk > INT32_MAX) return SSA_ERR_UNSUPPORTED;
  BwdWs w;
  const size_t base = carve_bwd(nullptr, p, S, Nq, blk->count, 0, &w);
  if (ws_bytes < base + cross_extra_bytes(Nq, p->hq)) return SSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* gates3 = nullptr;
  ps = cross_prepare(p, q_cu, S, Nq, blk, gates, static_cast<char*>(ws) + base, &gates3, st);
  if (ps != SSA_OK) return ps;
  return backward_common(p, q_cu, S, Nq, Nkv, 1, blk, nullptr, q, k, v, gates3, saved, dout, dq, dk, dv, dgates,
                         ws, st);
}


}  // extern "C"

namespace {

ssa_status sp_check(const ssa_params* p, int32_t S, int64_t N, const ssa_partition* blk, const ssa_sp_local* loc) {
  ssa_status ps = check_params(p);
  if (ps != SSA_OK) return ps;
  if (p->conv) return SSA_ERR_INVALID_ARG;  // the learned compression is built for the whole-sequence call
  if (p->deterministic) return SSA_ERR_UNSUPPORTED;  // the fixed-point sums are built for ssa_backward
  if (p->m_cmp % p->m_win != 0) return SSA_ERR_INVALID_ARG;  // a window must lie inside one block
  if (S < 1 || N < 1 || N > INT32_MAX - 1 || !loc || loc->n < 0 || loc->n > N || !partition_ok(blk, N))
    return SSA_ERR_INVALID_ARG;
  if (!loc->cu_seqlens || !partition_ok(loc->win, loc->n)) return SSA_ERR_INVALID_ARG;
  if (loc->n > 0 && (!loc->tokens || !loc->k || !loc->v || !loc->ks || !loc->vs)) return SSA_ERR_INVALID_ARG;
  if (blk->count < 1 || blk->count > N || loc->win->count > loc->n) return SSA_ERR_INVALID_ARG;
  return SSA_OK;
}

}  // namespace

extern "C" {

SSA_API ssa_status ssa_sp_forward(const ssa_params* p, int32_t S, int64_t N, const ssa_partition* blk,
                                  const ssa_sp_local* loc, const void* q, const void* k, const void* v,
                                  const float* gates, void* out, const ssa_saved* saved, void* ws, size_t ws_bytes,
                                  void* stream) {
  ssa_status ps = sp_check(p, S, N, blk, loc);
  if (ps != SSA_OK) return ps;
  const int64_t nr = loc->n;
  if (nr == 0) return SSA_OK;
  if (!q || !k || !v || !gates || !out || !saved_ok(saved) || !ws) return SSA_ERR_INVALID_ARG;
  if (ws_bytes < fwd_bytes(p, S, nr, blk->count, loc->win->count) + sp_fwd_extra(p, loc->win->count))
    return SSA_ERR_WORKSPACE;
  return forward_common(p, loc->cu_seqlens, S, nr, N, 1, blk, nullptr, q, k, v, gates, out, saved, ws,
                        static_cast<cudaStream_t>(stream), loc);
}

SSA_API ssa_status ssa_sp_backward(const ssa_params* p, int32_t S, int64_t N, const ssa_partition* blk,
                                   const ssa_sp_local* loc, const void* q, const void* k, const void* v,
                                   const float* gates, const ssa_saved* saved, const void* dout, float* dq,
                                   float* dk, float* dv, float* dgates, void* ws, size_t ws_bytes, void* stream) {
  ssa_status ps = sp_check(p, S, N, blk, loc);
  if (ps != SSA_OK) return ps;
  const int64_t nr = loc->n;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (nr == 0) {  // no query rows here: this rank contributes nothing to any key gradient
    if (!dk || !dv) return SSA_ERR_INVALID_ARG;
    if (cudaMemsetAsync(dk, 0, sizeof(float) * N * p->hkv * p->d, st) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, sizeof(float) * N * p->hkv * p->d, st) != cudaSuccess)
      return SSA_ERR_CUDA;
    return SSA_OK;
  }
  if (!q || !k || !v || !gates || !dout || !dq || !dk || !dv || !dgates || !saved_ok(saved) || !ws)
    return SSA_ERR_INVALID_ARG;
  if (nr * p->hkv * p->topk > INT32_MAX) return SSA_ERR_UNSUPPORTED;
  BwdWs w;
  const size_t base = carve_bwd(nullptr, p, S, nr, blk->count, loc->win->count, &w);
  if (ws_bytes < base + sp_bwd_extra(p, nr)) return SSA_ERR_WORKSPACE;
  char* extra = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + base + 255) & ~uintptr_t(255));
  float* wdk = reinterpret_cast<float*>(extra);
  float* wdv = reinterpret_cast<float*>(extra + align256(sizeof(float) * (size_t)nr * p->hkv * p->d));
  return backward_common(p, loc->cu_seqlens, S, nr, N, 1, blk, nullptr, q, k, v, gates, saved, dout, dq, dk, dv,
                         dgates, ws, st, loc, wdk, wdv);
}

}  // extern "C"
