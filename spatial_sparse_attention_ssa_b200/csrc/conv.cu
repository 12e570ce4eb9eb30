// Learned compression: a submanifold sparse 3D convolution (kernel 3^3) of K and V
// before the block mean (Direct3D-S2, hyper.ai, "方法": the sparse 3D compression may
// run a sparse 3D convolution before pooling; LSRM names a ResBlock there).
//
// The convolution is linear, so the block mean of its output needs no per-token
// output:   Xc_b = bias + sum_o W_o^T M_{b,o},   M_{b,o} = (1/n_b) sum_{i in b} sum_{j at c_i + o} x_j.
// M (the mean, over the block's members, of the neighbour at offset o) is gathered per
// block; the product with W is a small GEMM over (offset, channel).  The backward uses
// the same structure: dM_{b,o} = W_o dXc_b, dW_o = sum_b M_{b,o} dXc_b^T,
// db = sum_b dXc_b, and dx_j = sum_o sum_{i at c_j - o} dM_{b(i),o} / n_{b(i)} (a gather,
// no atomics).
//
// Neighbours of a token of block b lie in the 27 cells around b's cell; each CTA looks
// their block ids up once (binary search over the sequence's sorted cell keys).  For
// m <= 8 a per-block table of the m^3 voxels of the cell (token, or -1 if empty, -2 if
// several tokens share the voxel) answers a probe in one load; otherwise, and for
// shared voxels, the block's members (coordinates in block order) are scanned.
// Repeated coordinates are all matched, as a dense grid with summed duplicates would.
#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

constexpr int kConvThreads = 256;
constexpr int kConvWarps = kConvThreads / 32;

constexpr int kConvTableMaxM = 8;  // cells of up to 8^3 voxels get a lookup table

__device__ __forceinline__ int local_voxel(int x, int y, int z, int m) { return ((x % m) * m + (y % m)) * m + (z % m); }

// cs[p] = (x, y, z, token) of blk.perm[p]; with a table, table[b][voxel] = token (-2: shared)
__global__ void conv_prep_kernel(const int32_t* __restrict__ coords, const int32_t* __restrict__ perm,
                                 const int32_t* __restrict__ bid, int64_t N, int m, int4* __restrict__ cs,
                                 int* __restrict__ table) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t t = perm[i];
    const int x = coords[3 * (int64_t)t], y = coords[3 * (int64_t)t + 1], z = coords[3 * (int64_t)t + 2];
    cs[i] = make_int4(x, y, z, t);
    if (table) {
      int* slot = table + (int64_t)bid[t] * m * m * m + local_voxel(x, y, z, m);
      if (atomicCAS(slot, -1, t) != -1) atomicExch(slot, -2);
    }
  }
}

// block of [b0, b1) whose cell is (x, y, z), or -1 (keys ascend lexicographically)
__device__ int find_cell(const int32_t* __restrict__ key, int b0, int b1, int x, int y, int z) {
  int lo = b0, hi = b1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int* k = key + 3 * (int64_t)mid;
    const bool less = k[0] != x ? k[0] < x : (k[1] != y ? k[1] < y : k[2] < z);
    if (less)
      lo = mid + 1;
    else
      hi = mid;
  }
  if (lo < b1) {
    const int* k = key + 3 * (int64_t)lo;
    if (k[0] == x && k[1] == y && k[2] == z) return lo;
  }
  return -1;
}

// The 27 blocks around block b (offset index (dx+1)*9 + (dy+1)*3 + (dz+1)), -1 where
// the cell is empty or outside the grid.
__device__ void neighbour_cells(const int32_t* __restrict__ key, const int32_t* __restrict__ bcu, int S, int b,
                                int* nb) {
  const int t = threadIdx.x;
  if (t < 27) {
    const int s = find_segment(bcu, S, b);
    const int* k = key + 3 * (int64_t)b;
    const int x = k[0] + t / 9 - 1, y = k[1] + (t / 3) % 3 - 1, z = k[2] + t % 3 - 1;
    nb[t] = (x < 0 || y < 0 || z < 0) ? -1 : find_cell(key, bcu[s], bcu[s + 1], x, y, z);
  }
}

// For lane o < 27 of a warp looking at point p = c + sign * offset_o: the next token at
// p in the block that holds p, scanning from *q.  Returns the token or -1.
struct Probe {
  int px, py, pz;  // the point
  int q, qend;     // remaining members of the block to scan
  int blk;         // that block
  int direct;      // the token found in the table, returned first (-1: none)
};
__device__ __forceinline__ Probe make_probe(int4 c, int o, int sign, int m, const int* nb, const int32_t* bptr,
                                            int kx, int ky, int kz, const int* __restrict__ table) {
  Probe pr;
  pr.q = pr.qend = 0;
  pr.blk = -1;
  pr.direct = -1;
  pr.px = c.x + sign * (o / 9 - 1);
  pr.py = c.y + sign * ((o / 3) % 3 - 1);
  pr.pz = c.z + sign * (o % 3 - 1);
  if (o < 27 && pr.px >= 0 && pr.py >= 0 && pr.pz >= 0) {
    const int dx = pr.px / m - kx, dy = pr.py / m - ky, dz = pr.pz / m - kz;  // each in -1 .. 1
    const int b = nb[(dx + 1) * 9 + (dy + 1) * 3 + (dz + 1)];
    if (b >= 0) {
      pr.blk = b;
      const int tv = table ? table[(int64_t)b * m * m * m + local_voxel(pr.px, pr.py, pr.pz, m)] : -2;
      if (tv >= 0) {
        pr.direct = tv;
      } else if (tv == -2) {  // no table, or several tokens on the voxel: scan the block
        pr.q = bptr[b];
        pr.qend = bptr[b + 1];
      }
    }
  }
  return pr;
}
__device__ __forceinline__ int next_match(Probe& pr, const int4* __restrict__ cs) {
  if (pr.direct >= 0) {
    const int t = pr.direct;
    pr.direct = -1;
    return t;
  }
  for (; pr.q < pr.qend; ++pr.q) {
    const int4 r = cs[pr.q];
    if (r.x == pr.px && r.y == pr.py && r.z == pr.pz) {
      ++pr.q;
      return r.w;
    }
  }
  return -1;
}

// M[kv][b][g][o][c] = (1/n_b) sum over members i of b and tokens j at c_i + offset_o of x_j
template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv_gather_kernel(
    const T* __restrict__ k, const T* __restrict__ v, const int4* __restrict__ cs, const int32_t* __restrict__ bptr,
    const int32_t* __restrict__ key, const int32_t* __restrict__ bcu, int S, int B, int hkv, int d, int m,
    const int* __restrict__ table, float* __restrict__ M) {
  extern __shared__ float ms[];  // [2][hkv][27][d]
  __shared__ int nb[27];
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = hkv * d;
  const int per_kv = row * 27;
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    for (int i = threadIdx.x; i < 2 * per_kv; i += kConvThreads) ms[i] = 0.f;
    neighbour_cells(key, bcu, S, b, nb);
    __syncthreads();
    const int* kb = key + 3 * (int64_t)b;
    const int p0 = bptr[b], p1 = bptr[b + 1];
    for (int p = p0 + w; p < p1; p += kConvWarps) {
      Probe pr = make_probe(cs[p], lane, 1, m, nb, bptr, kb[0], kb[1], kb[2], table);
      for (;;) {
        const int j = next_match(pr, cs);
        unsigned bal = __ballot_sync(0xffffffffu, j >= 0);
        if (!bal) break;
        while (bal) {
          const int src = __ffs(bal) - 1;
          bal &= bal - 1;
          const int jj = __shfl_sync(0xffffffffu, j, src);
          for (int e = lane; e < row; e += 32) {
            const int g = e / d, c = e % d;
            atomicAdd(&ms[(g * 27 + src) * d + c], Elem<T>::to_f(k[(int64_t)jj * row + e]));
            atomicAdd(&ms[per_kv + (g * 27 + src) * d + c], Elem<T>::to_f(v[(int64_t)jj * row + e]));
          }
        }
      }
    }
    __syncthreads();
    const float inv = 1.f / (float)(p1 - p0);
    for (int i = threadIdx.x; i < 2 * per_kv; i += kConvThreads) {
      const int kv = i / per_kv, r = i % per_kv;
      M[((int64_t)kv * B + b) * per_kv + r] = ms[i] * inv;
    }
    __syncthreads();
  }
}

// dx_j += sum_o sum_{i at c_j - offset_o} dM[kv][b(i)][g][o][:] / n_{b(i)}   (dk, dv [N, hkv, d])
__global__ void __launch_bounds__(kConvThreads) conv_dx_kernel(
    const float* __restrict__ dM, const int4* __restrict__ cs, const int32_t* __restrict__ bptr,
    const int32_t* __restrict__ key, const int32_t* __restrict__ bcu, int S, int B, int hkv, int d, int m,
    const int* __restrict__ table, float* __restrict__ dk, float* __restrict__ dv) {
  __shared__ int nb[27];
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = hkv * d;
  const int per_kv = row * 27;
  constexpr int kMaxE = 8;  // row <= 256: elements per lane
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    neighbour_cells(key, bcu, S, b, nb);
    __syncthreads();
    const int* kb = key + 3 * (int64_t)b;
    const int p0 = bptr[b], p1 = bptr[b + 1];
    for (int p = p0 + w; p < p1; p += kConvWarps) {
      const int4 c = cs[p];
      float ak[kMaxE], av[kMaxE];
#pragma unroll
      for (int x = 0; x < kMaxE; ++x) ak[x] = av[x] = 0.f;
      Probe pr = make_probe(c, lane, -1, m, nb, bptr, kb[0], kb[1], kb[2], table);
      for (;;) {
        const int i = next_match(pr, cs);
        unsigned bal = __ballot_sync(0xffffffffu, i >= 0);
        if (!bal) break;
        while (bal) {
          const int src = __ffs(bal) - 1;
          bal &= bal - 1;
          const int bi = __shfl_sync(0xffffffffu, pr.blk, src);
          const float inv = 1.f / (float)(bptr[bi + 1] - bptr[bi]);
#pragma unroll
          for (int x = 0; x < kMaxE; ++x) {
            const int e = lane + 32 * x;
            if (e < row) {
              const int g = e / d, cc = e % d;
              const int64_t off = (int64_t)bi * per_kv + (g * 27 + src) * d + cc;
              ak[x] += dM[off] * inv;
              av[x] += dM[(int64_t)B * per_kv + off] * inv;
            }
          }
        }
      }
      const int64_t t = c.w;
#pragma unroll
      for (int x = 0; x < kMaxE; ++x) {
        const int e = lane + 32 * x;
        if (e < row) {
          dk[t * row + e] += ak[x];
          dv[t * row + e] += av[x];
        }
      }
    }
    __syncthreads();
  }
}

// Batched fp32 GEMM C[r][n] (+)= sum_k A[r][k] B[k][n] for batch z = kv * hkv + g; the
// operand of batch z is base[kv] + g * batch stride; element (r, k) of A sits at
// r * ar + k * ak (likewise B, C).  64 x 64 tiles, 4 x 4 per thread.  Split-K over
// gridDim.z / (2 * hkv) chunks with atomics when ATOMIC.  The non-atomic form adds
// bias[kv][g][n] and stores in T.
struct GemmOp {
  const float* a[2];
  int64_t a_g, ar, ak;
  const float* b[2];
  int64_t b_g, bk, bn;
  void* c[2];
  int64_t c_g, cr, cn;
  const float* bias[2];  // [hkv][ncols] or null
  int rows, cols, kdim, hkv;
};

template <typename T, bool ATOMIC>
__global__ void __launch_bounds__(256) conv_gemm_kernel(GemmOp op, int ksplit) {
  __shared__ float as[16][64 + 1];
  __shared__ float bs[16][64 + 1];
  const int z = blockIdx.z / ksplit, kc = blockIdx.z % ksplit;
  const int kv = z / op.hkv, g = z % op.hkv;
  const float* A = op.a[kv] + g * op.a_g;
  const float* Bm = op.b[kv] + g * op.b_g;
  const int r0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tr = threadIdx.x / 16, tn = threadIdx.x % 16;
  const int kper = (op.kdim + ksplit - 1) / ksplit;
  const int kb = kc * kper, ke = min(op.kdim, kb + kper);
  float acc[4][4] = {};
  for (int k0 = kb; k0 < ke; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i / 64, x = i % 64;
      const int k = k0 + kk;
      const int r = r0 + x, n = n0 + x;
      as[kk][x] = (k < ke && r < op.rows) ? A[r * op.ar + k * op.ak] : 0.f;
      bs[kk][x] = (k < ke && n < op.cols) ? Bm[k * op.bk + n * op.bn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float ar[4], br[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ar[i] = as[kk][tr * 4 + i];
        br[i] = bs[kk][tn * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + tr * 4 + i;
    if (r >= op.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n >= op.cols) continue;
      const int64_t off = g * op.c_g + r * op.cr + n * op.cn;
      if (ATOMIC) {
        atomicAdd(static_cast<float*>(op.c[kv]) + off, acc[i][j]);
      } else {
        const float bias = op.bias[kv] ? op.bias[kv][g * op.cols + n] : 0.f;
        static_cast<T*>(op.c[kv])[off] = Elem<T>::from_f(acc[i][j] + bias);
      }
    }
  }
}

// db[kv][g][c] = sum_b dXc[kv][g][b][c]
__global__ void conv_db_kernel(const float* __restrict__ dkc, const float* __restrict__ dvc, int B, int hkv, int d,
                               float* __restrict__ dbk, float* __restrict__ dbv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * hkv * d) return;
  const int kv = i / (hkv * d), r = i % (hkv * d);
  const int g = r / d, c = r % d;
  const float* src = (kv ? dvc : dkc) + (int64_t)g * B * d + c;
  float s = 0.f;
  for (int b = 0; b < B; ++b) s += src[(int64_t)b * d];
  (kv ? dbv : dbk)[r] = s;
}

size_t gather_smem(int hkv, int d) { return sizeof(float) * 2 * 27 * hkv * d; }

int conv_grid(int64_t B) { return (int)(B < 148 * 8 ? (B > 0 ? B : 1) : 148 * 8); }

template <typename T>
cudaError_t conv_gather(const ConvArgs& c, const void* k, const void* v, float* M, cudaStream_t st) {
  const size_t smem = gather_smem(c.hkv, c.d);
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(conv_gather_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gather_smem(4, 64));
    attr = true;
  }
  SSA_LAUNCH("conv_gather_kernel", conv_gather_kernel<T>, conv_grid(c.blk->count), kConvThreads, smem, st,
             static_cast<const T*>(k), static_cast<const T*>(v), c.cs, c.blk->ptr, c.blk->key, c.blk->cu, c.S,
             (int)c.blk->count, c.hkv, c.d, c.m, c.m <= kConvTableMaxM ? c.table : nullptr, M);
  return cudaGetLastError();
}

cudaError_t launch_prep(const ConvArgs& c, cudaStream_t st) {
  const int64_t g = (c.N + 255) / 256;
  int* table = c.m <= kConvTableMaxM ? c.table : nullptr;
  if (table && cudaMemsetAsync(table, 0xff, sizeof(int) * (size_t)c.blk->count * c.m * c.m * c.m, st) != cudaSuccess)
    return cudaErrorUnknown;
  SSA_LAUNCH("conv_prep_kernel", conv_prep_kernel, (int)(g < 148 * 32 ? (g > 0 ? g : 1) : 148 * 32), 256, 0, st,
             c.coords, c.blk->perm, c.blk->id, c.N, c.m, c.cs, table);
  return cudaGetLastError();
}

}  // namespace

size_t conv_ws_floats(int64_t N, int64_t B, int hkv, int d, int m) {
  // cs (N int4), M [2][B][hkv][27][d], dM (the same), the voxel table [B][m^3]
  const size_t table = m <= kConvTableMaxM ? (size_t)B * m * m * m : 0;
  return (size_t)N * 4 + 2 * (size_t)(2 * B * hkv * 27 * d) + table + 128;
}

cudaError_t conv_forward(const ConvArgs& c, int dtype, const void* k, const void* v, void* kc, void* vc,
                         cudaStream_t st) {
  const int64_t B = c.blk->count;
  cudaError_t e = launch_prep(c, st);
  if (e != cudaSuccess) return e;
  e = dtype == SSA_DTYPE_BF16 ? conv_gather<__nv_bfloat16>(c, k, v, c.M, st) : conv_gather<float>(c, k, v, c.M, st);
  if (e != cudaSuccess) return e;
  // Xc[g][b][n] = bias[g][n] + sum_K M[kv][b][g][K] W[g][K][n]
  const int per_g = 27 * c.d;
  GemmOp op;
  op.a[0] = c.M;
  op.a[1] = c.M + B * c.hkv * per_g;
  op.a_g = per_g;
  op.ar = (int64_t)c.hkv * per_g;
  op.ak = 1;
  op.b[0] = c.wk;
  op.b[1] = c.wv;
  op.b_g = (int64_t)per_g * c.d;
  op.bk = c.d;
  op.bn = 1;
  op.c[0] = kc;
  op.c[1] = vc;
  op.c_g = B * c.d;
  op.cr = c.d;
  op.cn = 1;
  op.bias[0] = c.bk;
  op.bias[1] = c.bv;
  op.rows = (int)B;
  op.cols = c.d;
  op.kdim = per_g;
  op.hkv = c.hkv;
  const dim3 grid((c.d + 63) / 64, (unsigned)((B + 63) / 64), 2 * c.hkv);
  if (dtype == SSA_DTYPE_BF16)
    SSA_LAUNCH("conv_gemm_kernel", (conv_gemm_kernel<__nv_bfloat16, false>), grid, 256, 0, st, op, 1);
  else
    SSA_LAUNCH("conv_gemm_kernel", (conv_gemm_kernel<float, false>), grid, 256, 0, st, op, 1);
  return cudaGetLastError();
}

cudaError_t conv_backward(const ConvArgs& c, int dtype, const void* k, const void* v, const float* dkc,
                          const float* dvc, float* dk, float* dv, cudaStream_t st) {
  const int64_t B = c.blk->count;
  const int per_g = 27 * c.d;
  const int64_t per_kv = B * c.hkv * per_g;
  cudaError_t e = launch_prep(c, st);
  if (e != cudaSuccess) return e;
  e = dtype == SSA_DTYPE_BF16 ? conv_gather<__nv_bfloat16>(c, k, v, c.M, st) : conv_gather<float>(c, k, v, c.M, st);
  if (e != cudaSuccess) return e;
  // dM[kv][b][g][K] = sum_n dXc[g][b][n] W[g][K][n]
  {
    GemmOp op;
    op.a[0] = dkc;
    op.a[1] = dvc;
    op.a_g = B * c.d;
    op.ar = c.d;
    op.ak = 1;
    op.b[0] = c.wk;
    op.b[1] = c.wv;
    op.b_g = (int64_t)per_g * c.d;
    op.bk = 1;
    op.bn = c.d;
    op.c[0] = c.dM;
    op.c[1] = c.dM + per_kv;
    op.c_g = per_g;
    op.cr = (int64_t)c.hkv * per_g;
    op.cn = 1;
    op.bias[0] = op.bias[1] = nullptr;
    op.rows = (int)B;
    op.cols = per_g;
    op.kdim = c.d;
    op.hkv = c.hkv;
    const dim3 grid((per_g + 63) / 64, (unsigned)((B + 63) / 64), 2 * c.hkv);
    SSA_LAUNCH("conv_gemm_kernel", (conv_gemm_kernel<float, false>), grid, 256, 0, st, op, 1);
  }
  // dW[g][K][n] = sum_b M[kv][b][g][K] dXc[g][b][n]  (split over b, atomics into zeroed dW)
  {
    if (cudaMemsetAsync(c.dwk, 0, sizeof(float) * c.hkv * per_g * c.d, st) != cudaSuccess ||
        cudaMemsetAsync(c.dwv, 0, sizeof(float) * c.hkv * per_g * c.d, st) != cudaSuccess)
      return cudaErrorUnknown;
    GemmOp op;
    op.a[0] = c.M;
    op.a[1] = c.M + per_kv;
    op.a_g = per_g;
    op.ar = 1;
    op.ak = (int64_t)c.hkv * per_g;
    op.b[0] = dkc;
    op.b[1] = dvc;
    op.b_g = B * c.d;
    op.bk = c.d;
    op.bn = 1;
    op.c[0] = c.dwk;
    op.c[1] = c.dwv;
    op.c_g = (int64_t)per_g * c.d;
    op.cr = c.d;
    op.cn = 1;
    op.bias[0] = op.bias[1] = nullptr;
    op.rows = per_g;
    op.cols = c.d;
    op.kdim = (int)B;
    op.hkv = c.hkv;
    const int ksplit = (int)((B + 255) / 256);
    const dim3 grid((c.d + 63) / 64, (unsigned)((per_g + 63) / 64), 2 * c.hkv * ksplit);
    SSA_LAUNCH("conv_gemm_kernel", (conv_gemm_kernel<float, true>), grid, 256, 0, st, op, ksplit);
  }
  SSA_LAUNCH("conv_db_kernel", conv_db_kernel, (2 * c.hkv * c.d + 255) / 256, 256, 0, st, dkc, dvc, (int)B, c.hkv,
             c.d, c.dbk, c.dbv);
  SSA_LAUNCH("conv_dx_kernel", conv_dx_kernel, conv_grid(B), kConvThreads, 0, st, c.dM, c.cs, c.blk->ptr,
             c.blk->key, c.blk->cu, c.S, (int)B, c.hkv, c.d, c.m, c.m <= kConvTableMaxM ? c.table : nullptr, dk, dv);
  return cudaGetLastError();
}

}  // namespace ssa
