// Argument bundles passed from the C ABI layer to the kernel launchers (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ssa.h"

namespace ssa {

// Query rows per work item of the compressed-branch dKc/dVc kernel.
constexpr int kCmpRowChunk = 2048;
// Upper bound on the CTAs of the tensor-core compressed-output kernel (sizes its score scratch).
constexpr int kCmpOutCtas = 160;

struct FwdArgs {
  int dtype, d, hq, hkv, topk, gate_mode, m_cmp, m_win;
  int sel_given;  // sel is an input (checked, not computed)
  int cross;      // queries from another token set: no window branch, gates hold 2 live columns
  int64_t Nkv;    // key / value tokens (= N unless cross)
  int use_tc;   // run the tensor-core kernels where they cover the shape
  int* status;  // device check word
  float scale;
  int32_t S;
  int64_t N;
  const int32_t* cu_seqlens;
  const ssa_partition* blk;
  const ssa_partition* win;
  const void *q, *k, *v;
  const float* gates;
  void* out;
  // saved
  void *kc, *vc, *ks, *vs;
  float* o_branch;
  float* lse;
  int32_t* sel;
  // workspace
  int32_t *tiles_cnt, *tiles_pre, *items_cnt, *items_pre, *scan_tmp;
  float* imp_scratch;  // [kCmpOutCtas, 128/G, B] selection scores (tensor-core path)
  int32_t *win_cnt, *win_pre, *win_scan;  // [W + 1] window work plan
  // The window branch's problem: the queries' own tokens.  Self attention: has_win = 1,
  // wk/wv = k/v, wks/wvs = ks/vs.  Cross attention: has_win = 0.  A sequence-parallel
  // rank: its own tokens' K / V and their window-ordered copies.
  int has_win;
  const void *wk, *wv;  // [N, Hkv, d] K / V of the query tokens (SIMT window kernels)
  void *wks, *wvs;      // [Hkv, N, d] the same in window order (tensor-core window kernels)
};

// Learned compression (sparse 3D convolution before the block mean), see conv.cu.
struct ConvArgs {
  const int32_t* coords;      // [N, 3] voxel coordinates
  const ssa_partition* blk;
  int S;
  int64_t N;
  int hkv, d, m;
  const float *wk, *bk, *wv, *bv;  // [Hkv, 27, d, d], [Hkv, d]
  float *dwk, *dbk, *dwv, *dbv;    // backward outputs
  int4* cs;                   // workspace: [N] coordinates in block order
  float* M;                   // workspace: [2][B][Hkv][27][d]
  float* dM;                  // workspace: [2][B][Hkv][27][d] (backward)
  int* table;                 // workspace: [B][m^3] voxel -> token (m <= 8)
};
size_t conv_ws_floats(int64_t N, int64_t B, int hkv, int d, int m);
cudaError_t conv_forward(const ConvArgs& c, int dtype, const void* k, const void* v, void* kc, void* vc,
                         cudaStream_t st);
cudaError_t conv_backward(const ConvArgs& c, int dtype, const void* k, const void* v, const float* dkc,
                          const float* dvc, float* dk, float* dv, cudaStream_t st);

struct BwdArgs {
  int dtype, d, hq, hkv, topk, gate_mode, m_cmp, m_win;
  int cross;    // as in FwdArgs
  int64_t Nkv;  // key / value tokens (= N unless cross)
  const ConvArgs* conv;  // learned compression, or null (mean pool)
  int use_tc;
  int* status;
  float scale;
  int32_t S;
  int64_t N;
  const int32_t* cu_seqlens;
  const ssa_partition* blk;
  const ssa_partition* win;
  const void *q, *k, *v;
  const float* gates;
  const void *kc, *vc, *ks, *vs;
  const float* o_branch;
  const float* lse;
  const int32_t* sel;
  const void* dout;
  float *dq, *dk, *dv, *dgates;
  // workspace
  float* Dc;          // [3, N, Hq]
  // per-row constants of the tensor-core backward kernels, [2 branches (cmp, win)]
  // x [3][N, Hq]: -lse * log2(e), the gate weight w, and -D (D = w <dO, o>)
  float* rc;
  int32_t *win_cnt, *win_pre;  // [W + 1] window work plan
  float *dkc, *dvc;   // [Hkv, B, d]
  uint64_t *inv_keys_a, *inv_keys_b;
  int32_t *inv_vals_a, *inv_vals_b;
  int32_t* inv_ptr;   // [Hkv * B + 1]
  int32_t* radix_tmp;
  int32_t *slc_cnt, *slc_pre;  // [Hkv * B + 1] work items of the selected-branch dK/dV kernel
  int32_t *tiles_cnt, *tiles_pre, *items_cnt, *items_pre, *scan_tmp;
  // the window branch's problem, as in FwdArgs; its key gradients go to wdk / wdv
  // ([N, Hkv, d]: dk / dv themselves unless the query rows are a rank's tokens, whose
  // window gradients are then scatter-added into dk / dv at rows wtok[i])
  int has_win;
  const void *wk, *wv, *wks, *wvs;
  float *wdk, *wdv;
  const int32_t* wtok;
  // deterministic mode: 64-bit fixed-point accumulators (2^-32 units) of the compressed
  // dKc / dVc [Hkv, B, d] and of the selected branch's dK / dV [Nkv, Hkv, d]; null otherwise
  unsigned long long *fx_kc, *fx_vc, *fx_k, *fx_v;
  // fp16 copies of Q, dO [N, Hq, d] and Kc, Vc [Hkv, B, d] for the tensor-core dKc / dVc
  // kernel (written by the backward preamble); null where that kernel does not run
  void *q16, *do16, *kc16, *vc16;
};

// Fixed-point unit of the deterministic accumulations: values are added as
// round(x * 2^32) into 64-bit integers.
constexpr float kFixScale = 4294967296.f;

bool pool_supported(int dtype, int hkv, int d);
cudaError_t launch_pool(int dtype, const void* k, const void* v, const ssa_partition* blk, int64_t N, int hkv,
                        int d, void* ks, void* vs, void* kc, void* vc, cudaStream_t st);
cudaError_t simt_forward(const FwdArgs& a, cudaStream_t st);
cudaError_t cross_prep(const float* gates2, int64_t rows, float* gates3, const int32_t* q_cu, const int32_t* bcu,
                       int S, int* bad, cudaStream_t st);

// Tensor-core (tcgen05) kernels of the compressed branch, bf16, head dim 64.
bool cmp_tc_supported(int dtype, int d, int hq, int hkv, int topk);
size_t cmp_tc_scratch_floats(int hq, int hkv, int64_t btot);
cudaError_t cmp_fwd_tc(const FwdArgs& a, const int32_t* tpre, int64_t total_tiles_bound, cudaStream_t st);
bool win_tc_supported(int dtype, int d, int hq, int hkv, int m_cmp, int m_win);
cudaError_t win_fwd_tc(const FwdArgs& a, int32_t* cnt, int32_t* pre, int32_t* scan_tmp, cudaStream_t st);
cudaError_t win_bwd_tc(const BwdArgs& a, int32_t* cnt, int32_t* pre, int32_t* scan_tmp, cudaStream_t st);
cudaError_t cmp_bwd_tc(const BwdArgs& a, const int32_t* tpre, int32_t* dkv_cnt, int32_t* dkv_pre, int32_t* scan_tmp,
                       int64_t tiles_bound, cudaStream_t st);
cudaError_t simt_backward(const BwdArgs& a, cudaStream_t st);
// dst[i] = src[i] / 2^32 (the deterministic accumulators back to fp32)
cudaError_t fix_to_float(const unsigned long long* src, float* dst, int64_t n, cudaStream_t st);

// 3D-aware block routing: selection by the shortest distance to a block's voxels.
size_t geo_ws_bytes(int64_t N);
cudaError_t geo_select(const int32_t* coords, const int32_t* cu_seqlens, int S, int64_t N, const ssa_partition* blk,
                       int m, int topk, int hkv, int32_t* sel, void* ws, cudaStream_t st);

// Selected-block branch on warp-level MMAs (bf16, head dim 64, G in {8, 16}, top-k <= 32).
bool slc_mma_supported(int dtype, int d, int hq, int hkv, int topk);
cudaError_t slc_fwd_mma(const FwdArgs& a, cudaStream_t st);
cudaError_t slc_bwd_mma(const BwdArgs& a, cudaStream_t st);

// Diagnostics (diag.cu): a bounded wait that runs out; the FMA-pipe exponential.
cudaError_t diag_wait_timeout(int* status, int* out, cudaStream_t st);
cudaError_t diag_ex2(const float* x, float* y_poly, float* y_mufu, int64_t n, cudaStream_t st);

}  // namespace ssa
