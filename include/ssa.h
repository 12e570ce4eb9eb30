/*
 * ssa.h -- C ABI of the spatial sparse attention (SSA) library, libssa.so.
 *
 * SSA is the attention of Direct3D-S2 (hyper.ai/cn/papers/2505.17412, section
 * "方法", the SSA paragraph) over the variable-length set of occupied sparse
 * voxels near a 3D surface.  Three modules run side by side and their outputs
 * are summed with per-token gate weights:
 *   - sparse 3D compression: tokens are grouped into m_cmp^3 blocks by their
 *     integer (x, y, z) and each block's keys/values are mean-pooled;
 *   - spatial block selection: every query attends to all compressed blocks
 *     of its sequence, the top-k blocks by that attention score are picked and
 *     a second, full attention runs over every token of the picked blocks;
 *   - sparse 3D window: attention only inside non-overlapping m_win^3 windows.
 * GQA (several query heads per KV head) follows LSRM (shuwu5.cn/article/2502.html,
 * "阶段一": 32 query heads, 2 KV heads).
 *
 * Entry points: ssa_bin (step 1), ssa_pool (step 2 alone), ssa_forward (steps 2-6),
 * ssa_backward (step 7);
 * ssa_geo_select (geometric block routing) and ssa_params.selection (a given
 * selection); ssa_cross_forward / ssa_cross_backward (queries of another token
 * set); ssa_params.conv (learned compression); ssa_bin_noalloc; workspace sizes,
 * status, version and per-kernel timing.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers unless stated; the caller owns
 *     and allocates every buffer, including the workspace.  The library never
 *     allocates or frees device memory.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  Only ssa_bin, ssa_bin_noalloc, ssa_cross_forward,
 *     ssa_cross_backward and ssa_get_device_status synchronise that stream; they
 *     read their few result ints through 64 bytes of pinned, mapped host memory
 *     per calling thread (allocated on the thread's first such call, kept until
 *     exit) that a one-thread kernel writes, so the read never waits in a copy
 *     engine's queue behind other streams' bulk transfers.
 *   - Errors are returned as ssa_status codes; nothing aborts or throws across
 *     the ABI.  Argument errors are detected on the host before any launch.
 *   - N = number of tokens (all sequences), S = number of sequences,
 *     cu_seqlens = int32 [S+1] prefix offsets (cu_seqlens[0] = 0,
 *     non-decreasing, cu_seqlens[S] = N); sequence s owns tokens
 *     cu_seqlens[s] .. cu_seqlens[s+1]-1.  Tokens never attend across sequences.
 *   - Tensors are token-major and contiguous: Q, O [N, Hq, d]; K, V [N, Hkv, d];
 *     query head h belongs to KV head (group) h / (Hq/Hkv).
 *   - Results do not depend on the order of tokens inside a sequence (block,
 *     window and selected ids are functions of the coordinates only).
 */
#ifndef SSA_H
#define SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSA_API __attribute__((visibility("default")))

typedef enum ssa_status {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = 1, /* null pointer, bad size or head layout, m < 1, topk < 1 ... */
  SSA_ERR_UNSUPPORTED = 2, /* head dim / group size / key width this build does not handle */
  SSA_ERR_WORKSPACE = 3,   /* ws_bytes smaller than ssa_workspace_size() */
  SSA_ERR_COORD_RANGE = 4, /* a coordinate outside [0, R) or malformed cu_seqlens (device check) */
  SSA_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  SSA_ERR_TIMEOUT = 6      /* a bounded device wait gave up */
} ssa_status;

enum { SSA_DTYPE_BF16 = 0, SSA_DTYPE_F32 = 1 };
enum { SSA_GATE_WEIGHTS = 0, SSA_GATE_LOGITS = 1 };
/* where the selected branch's blocks come from (ssa_params.selection) */
enum { SSA_SEL_SCORES = 0, SSA_SEL_GIVEN = 1 };
enum {
  SSA_OP_BIN = 0,
  SSA_OP_FORWARD = 1,
  SSA_OP_BACKWARD = 2,
  SSA_OP_GEO_SELECT = 3,
  SSA_OP_CROSS_FORWARD = 4,
  SSA_OP_CROSS_BACKWARD = 5,
  SSA_OP_SP_FORWARD = 6,
  SSA_OP_SP_BACKWARD = 7
};

/* Shape and method parameters shared by forward and backward. */
/*
 * Learned compression (Direct3D-S2 "方法": the sparse 3D compression may apply a
 * sparse 3D convolution before pooling): Kc_b, Vc_b are the block means of a
 * submanifold sparse convolution with a 3x3x3 kernel of K and V,
 *   y_i = b + sum_o W_o^T x_j over the tokens j of i's sequence at coords_i + offset_o
 * (offset index o = (dx+1)*9 + (dy+1)*3 + (dz+1); empty voxels contribute nothing;
 * repeated coordinates all count), evaluated in fp32 and rounded once to the
 * storage type.  The selected and window branches keep the raw K and V.
 * All pointers are device pointers owned by the caller.
 */
typedef struct ssa_conv {
  const int32_t* coords; /* [N, 3] the token coordinates given to ssa_bin */
  const float* wk;       /* [Hkv, 27, d, d] (offset, in, out): the convolution of K */
  const float* bk;       /* [Hkv, d] its bias */
  const float* wv;       /* [Hkv, 27, d, d]: the convolution of V */
  const float* bv;       /* [Hkv, d] */
  float* dwk;            /* backward outputs, same shapes, written (not accumulated) */
  float* dbk;
  float* dwv;
  float* dbv;
} ssa_conv;

typedef struct ssa_params {
  int32_t hq;        /* query heads */
  int32_t hkv;       /* key/value heads; hq % hkv == 0, G = hq / hkv in {1,2,4,8,16} */
  int32_t d;         /* head dim: 32, 64 or 128 (128: G * 4 <= 32, i.e. G <= 8; the fp32 CUDA-core kernels) */
  int32_t m_cmp;     /* compression block edge (voxels), >= 1 */
  int32_t m_win;     /* window edge (voxels), >= 1 */
  int32_t topk;      /* selected blocks per (token, KV head), 1..32 */
  float scale;       /* softmax scale; 0 means 1/sqrt(d) */
  int32_t dtype;     /* SSA_DTYPE_BF16 (bf16 storage, fp32 math) or SSA_DTYPE_F32 */
  int32_t gate_mode; /* SSA_GATE_WEIGHTS: gates are the weights; SSA_GATE_LOGITS: weight = sigmoid(gate) */
  int32_t selection; /* SSA_SEL_SCORES: the forward selects by compressed-attention score (top-k) and writes
                        saved->sel; SSA_SEL_GIVEN: saved->sel is an input the caller filled (for instance by
                        ssa_geo_select), read by the selected branch and the backward, see ssa_forward */
  const ssa_conv* conv; /* NULL: mean-pool compression; else the learned compression (self attention only;
                           Hkv * d <= 256); its workspace is included by ssa_workspace_size */
  int32_t deterministic; /* 0: the backward adds key gradients with fp32 atomics (bits may vary between
                            runs); 1: it adds them as 64-bit fixed-point integers (2^-32 resolution, each
                            accumulated component below 2^31 in magnitude), so every output is bitwise
                            reproducible.  1 needs the tensor-core backward (bf16, d = 64, G in {8, 16},
                            topk <= 32) and no conv, else SSA_ERR_UNSUPPORTED; its workspace is included */
} ssa_params;

/*
 * One partition of the tokens into cells of edge m (compression blocks or
 * windows).  Direct3D-S2 "方法": the partition is by 3D coordinate, not by 1D
 * index.  Cells are numbered per sequence in lexicographic (x, y, z) order of
 * the cell coordinate floor(coord / m), offset by the cells of earlier
 * sequences.  Caller-allocated device arrays, filled by ssa_bin:
 */
typedef struct ssa_partition {
  int32_t* id;   /* [N]      cell id of every token */
  int32_t* perm; /* [N]      tokens sorted by (cell id, token index) */
  int32_t* ptr;  /* [N+1]    members of cell c are perm[ptr[c] .. ptr[c+1]-1]; count+1 entries used */
  int32_t* cu;   /* [S+1]    cells of sequence s are cu[s] .. cu[s+1]-1 */
  int32_t* key;  /* [N, 3]   cell coordinate of cell c (rows 0 .. count-1 used) */
  int64_t count; /* out: number of cells (B_tot or W_tot) */
} ssa_partition;

/*
 * Buffers the forward writes and the backward reads (caller-allocated, device).
 * B = blk.count.  Layouts are head-major so that one block's rows are contiguous.
 */
typedef struct ssa_saved {
  void* kc;       /* [Hkv, B, d] dtype: mean-pooled keys, fp32(sum)/fp32(n) rounded to dtype */
  void* vc;       /* [Hkv, B, d] dtype: mean-pooled values */
  void* ks;       /* [Hkv, N, d] dtype: keys gathered in blk.perm order */
  void* vs;       /* [Hkv, N, d] dtype: values gathered in blk.perm order */
  float* o_branch; /* [3, N, Hq, d] fp32: branch outputs (0 compressed, 1 selected, 2 window) */
  float* lse;     /* [3, N, Hq] natural-log softmax normalisers of the three branches */
  int32_t* sel;   /* [N, Hkv, topk] selected block ids (global), ascending, padded with -1 */
} ssa_saved;

/*
 * ssa_bin -- step 1, coordinate binning (Direct3D-S2 "方法": spatially coherent
 * block partition into m_cmp^3 blocks and m_win^3 windows).
 *   coords   int32 [N, 3], 0 <= x, y, z < R
 *   R        grid resolution, 1 <= R <= 2^20
 * Fills `blk` (edge m_cmp) and `win` (edge m_win), including their counts.
 * Bit-exact integer work.  Synchronises `stream` once to return the counts and
 * the device check (SSA_ERR_COORD_RANGE if a coordinate is outside [0, R) or
 * cu_seqlens is malformed; outputs are then unspecified but in bounds).
 * SSA_ERR_UNSUPPORTED if the sort key (sequence bits + 3 x cell bits) exceeds 64 bits.
 */
SSA_API ssa_status ssa_bin(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N,
                           int32_t R, int32_t m_cmp, int32_t m_win, ssa_partition* blk,
                           ssa_partition* win, void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_bin_noalloc -- ssa_bin without a workspace argument, for callers that
 * cannot allocate device memory when they bin (the pages have no counterpart:
 * this is a property of the library, not of the method).  Examples: a plugin
 * whose host application owns all device memory through its own pool, a
 * latency-critical loop where cudaMalloc / cudaFree would synchronise the
 * device, a process that reserved nearly all memory up front.
 * The scratch is a fixed array in the library's device memory (about 11 MB on
 * every GPU that loads the library, held until the process exits), so:
 *   - N must be <= SSA_BIN_NOALLOC_MAX_TOKENS, else SSA_ERR_WORKSPACE and
 *     nothing is enqueued;
 *   - every call looks up the array's address on the current device
 *     (cudaGetSymbolAddress), so call it with the device of the buffers current;
 *   - like ssa_bin, it synchronises `stream` to return the counts;
 *   - all calls on a device share the array: calls whose GPU work overlaps
 *     (other streams, other host threads) race and corrupt each other; the
 *     array keeps the last call's contents, and each call clears the parts
 *     that must start at zero.
 * Arguments, outputs, synchronisation and error codes are those of ssa_bin.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define SSA_BIN_NOALLOC_MAX_TOKENS 262144
SSA_API ssa_status ssa_bin_noalloc(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N,
                                   int32_t R, int32_t m_cmp, int32_t m_win, ssa_partition* blk,
                                   ssa_partition* win, void* stream);

/*
 * ssa_pool -- step 2 alone, the sparse 3D compression (Direct3D-S2 "方法": each
 * block's keys and values are mean-pooled; LSRM "空间块划分与键值压缩": in-block
 * average pooling).  ssa_forward runs the same kernel first; this entry point is
 * for callers that want only the compressed keys/values or time the step by itself.
 *   dtype    SSA_DTYPE_BF16 or SSA_DTYPE_F32; hkv >= 1; d a multiple of 8 with
 *            2 * hkv * d * sizeof(dtype) <= 16384 (SSA_ERR_UNSUPPORTED otherwise)
 *   blk      the block partition from ssa_bin over the same N tokens (device arrays)
 *   k, v     [N, Hkv, d] dtype, token-major
 *   ks, vs   out [Hkv, N, d] dtype: rows gathered in blk.perm order (a block's tokens
 *            are one contiguous range per head)
 *   kc, vc   out [Hkv, blk.count, d] dtype: fp32(exact sum) / fp32(n), rounded to dtype
 *            (bf16: round to nearest even)
 * Every pointer must be 16-byte aligned.  Asynchronous; argument errors are found on
 * the host before anything is enqueued.  Bit-exact for bf16 (fp64 sums of bf16
 * values are exact).
 */
SSA_API ssa_status ssa_pool(int32_t dtype, int32_t hkv, int32_t d, int64_t N, const ssa_partition* blk,
                            const void* k, const void* v, void* ks, void* vs, void* kc, void* vc, void* stream);

/*
 * ssa_geo_select -- 3D-aware block routing (LSRM "3D 感知空间块路由机制", voxel-only
 * case: no camera projection): every token selects the topk blocks of its
 * sequence nearest to it, the distance to a block being the shortest Euclidean
 * distance between the token's voxel centre and the voxel centres of the block's
 * tokens; ties go to the lower block id; k_eff = min(topk, blocks in the
 * sequence).  Squared distances are exact integers: bit-exact integer work.
 *   coords   int32 [N, 3] device, 0 <= x, y, z < R, R <= 32768
 *   blk      block partition from ssa_bin with edge m_cmp (device arrays)
 *   sel      int32 [N, hkv, topk] device, caller-owned: global block ids,
 *            ascending, padded with -1; the same selection for every KV group
 *            (the layout of ssa_saved.sel)
 *   ws       device workspace of ssa_workspace_size(SSA_OP_GEO_SELECT, ...) bytes
 * Asynchronous.  SSA_ERR_INVALID_ARG for null pointers or bad sizes (topk must be
 * in 1..32), SSA_ERR_UNSUPPORTED for R > 32768, SSA_ERR_WORKSPACE if ws_bytes is
 * too small; all are found on the host before anything is enqueued.
 */
SSA_API ssa_status ssa_geo_select(const int32_t* coords, const int32_t* cu_seqlens, int32_t S, int64_t N,
                                  int32_t R, const ssa_partition* blk, int32_t m_cmp, int32_t topk,
                                  int32_t hkv, int32_t* sel, void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_forward -- steps 2-6: mean-pool compression; compressed attention of every
 * query against all blocks of its sequence; top-k block selection by the
 * softmax probability summed over the query heads of a GQA group (ties go to
 * the lower block id; k_eff = min(topk, blocks in the sequence)); full
 * attention over the tokens of the selected blocks; attention inside the
 * query's window; out = sum_c w_c * o_c with w = gates or sigmoid(gates).
 *   q [N, Hq, d], k/v [N, Hkv, d] in params->dtype; gates fp32 [N, Hq, 3]
 *   (branch order: compressed, selected, window); out [N, Hq, d] dtype.
 *   blk/win: partitions from ssa_bin with the same m_cmp / m_win.
 * Asynchronous.  Writes every buffer of `saved`.
 * With params->selection == SSA_SEL_GIVEN the top-k step is skipped and
 * saved->sel is read instead: [N, Hkv, topk] int32, each entry a global id of
 * a block of the token's own sequence or -1 (any order, any padding position;
 * a block listed twice is attended twice).  This is how a routing other than
 * the score top-k (LSRM "3D 感知空间块路由机制": ssa_geo_select) replaces the
 * selection; the backward then holds that selection fixed as usual.  Every
 * entry is checked on the device before use: an id outside the token's
 * sequence is replaced by -1 and ssa_get_device_status then reports
 * SSA_ERR_INVALID_ARG.
 */
SSA_API ssa_status ssa_forward(const ssa_params* p, const int32_t* cu_seqlens, int32_t S, int64_t N,
                               const ssa_partition* blk, const ssa_partition* win, const void* q,
                               const void* k, const void* v, const float* gates, void* out,
                               const ssa_saved* saved, void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_backward -- step 7: gradients of sum(dout * out) with the selection held
 * fixed.  The mean pooling passes gradients through as dK_i += dKc_b / n_b
 * (its rounding is treated as the identity).
 *   dout [N, Hq, d] dtype; outputs fp32: dq [N, Hq, d], dk/dv [N, Hkv, d],
 *   dgates [N, Hq, 3] (w.r.t. the gate inputs, including the sigmoid in
 *   SSA_GATE_LOGITS mode).  `saved` must come from ssa_forward on the same inputs.
 * Asynchronous.  Every output element is written (no accumulation into caller data).
 */
SSA_API ssa_status ssa_backward(const ssa_params* p, const int32_t* cu_seqlens, int32_t S,
                                int64_t N, const ssa_partition* blk, const ssa_partition* win,
                                const void* q, const void* k, const void* v, const float* gates,
                                const ssa_saved* saved, const void* dout, float* dq, float* dk,
                                float* dv, float* dgates, void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_cross_forward -- cross-attention SSA (LSRM: the NSA attention also serves as
 * cross attention between image tokens and voxel tokens): queries of another token
 * set attend the voxel tokens of the same sequence through two branches, the
 * compressed attention over all blocks (with the group-summed top-k selection, or a
 * given selection, as in ssa_forward) and full attention over the tokens of the
 * selected blocks.  The queries have no voxel, so there is no window branch.
 *   q [Nq, Hq, d] dtype, rows of sequence s are q_cu[s] .. q_cu[s+1]-1 (q_cu int32
 *   [S+1], device); k/v [Nkv, Hkv, d] dtype, the voxel tokens; blk: the block
 *   partition from ssa_bin over the voxel tokens (their coordinates and cu_seqlens,
 *   same S; the window partition is not used); gates fp32 [Nq, Hq, 2] (compressed,
 *   selected), weights or logits as params->gate_mode; out [Nq, Hq, d] dtype.
 *   saved: kc/vc [Hkv, B, d], ks/vs [Hkv, Nkv, d], o_branch fp32 [2, Nq, Hq, d],
 *   lse fp32 [2, Nq, Hq], sel int32 [Nq, Hkv, topk].
 *   ws: ssa_workspace_size(SSA_OP_CROSS_FORWARD, p, S, Nq, B, 0) bytes.
 * Every sequence with queries must have voxel tokens: the call checks this on the
 * device and synchronises the stream once to read the check (SSA_ERR_INVALID_ARG
 * if it fails, before any attention kernel runs).  Otherwise asynchronous.
 */
SSA_API ssa_status ssa_cross_forward(const ssa_params* p, const int32_t* q_cu, int32_t S, int64_t Nq,
                                     int64_t Nkv, const ssa_partition* blk, const void* q, const void* k,
                                     const void* v, const float* gates, void* out, const ssa_saved* saved,
                                     void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_cross_backward -- gradients of sum(dout * out) of ssa_cross_forward with the
 * selection held fixed: dq [Nq, Hq, d], dk/dv [Nkv, Hkv, d], dgates [Nq, Hq, 2], all
 * fp32 and all written.  dout [Nq, Hq, d] dtype; `saved` from ssa_cross_forward on
 * the same inputs; ws: ssa_workspace_size(SSA_OP_CROSS_BACKWARD, p, S, Nq, B, 0)
 * bytes.  Same check and single stream synchronisation as the forward.
 */
SSA_API ssa_status ssa_cross_backward(const ssa_params* p, const int32_t* q_cu, int32_t S, int64_t Nq,
                                      int64_t Nkv, const ssa_partition* blk, const void* q, const void* k,
                                      const void* v, const float* gates, const ssa_saved* saved,
                                      const void* dout, float* dq, float* dk, float* dv, float* dgates,
                                      void* ws, size_t ws_bytes, void* stream);

/*
 * One rank's share of a batch whose sequences are split across ranks by whole blocks
 * (LSRM, "块感知序列并行与负载均衡": a rank owns a contiguous range of a sequence's
 * blocks and their tokens; compression and window attention stay local; the keys and
 * values are exchanged; the key gradients go back to their owners).  The rank's query
 * tokens attend every compressed block and the tokens of their selected blocks of the
 * whole sequence (the K / V of all tokens, exchanged by the caller), and their windows,
 * which lie inside the rank's blocks when m_cmp is a multiple of m_win.
 */
typedef struct ssa_sp_local {
  int64_t n;                  /* Nr: this rank's tokens over all sequences */
  const int32_t* cu_seqlens;  /* [S+1] device: this rank's tokens of sequence s are rows cu[s] .. cu[s+1]-1 */
  const int32_t* tokens;      /* [Nr] device: the row of each of them in the all-token arrays (distinct) */
  const ssa_partition* win;   /* ssa_bin of this rank's coordinates with this cu_seqlens, edge m_win */
  const void* k;              /* [Nr, Hkv, d] dtype: this rank's K rows (the values of k[tokens]) */
  const void* v;              /* [Nr, Hkv, d] dtype */
  void* ks;                   /* [Hkv, Nr, d] dtype: their window-ordered copies, written by ssa_sp_forward */
  void* vs;                   /*   and read by ssa_sp_backward */
} ssa_sp_local;

/*
 * ssa_sp_forward -- the rank's forward: for its Nr query tokens q / gates [Nr, Hq, 3]
 * (rows in the order of loc->tokens), out [Nr, Hq, d] = sum_c w_c o_c of the three
 * branches, exactly as ssa_forward computes those rows on the whole batch.
 *   blk: ssa_bin of all N tokens (every rank bins the same coordinates); k, v [N, Hkv, d]
 *   all tokens.  saved: kc / vc [Hkv, B, d] and ks / vs [Hkv, N, d] of all tokens;
 *   o_branch [3, Nr, Hq, d], lse [3, Nr, Hq], sel [Nr, Hkv, topk] of the rank's rows.
 *   ws: ssa_workspace_size(SSA_OP_SP_FORWARD, p, S, Nr, B, loc->win->count) bytes.
 * SSA_ERR_INVALID_ARG if m_cmp is not a multiple of m_win (a window would cross blocks)
 * or params->conv is set.  Asynchronous.
 *
 * ssa_sp_backward -- the rank's backward: dq [Nr, Hq, d] and dgates [Nr, Hq, 3] of its
 * rows, and dk, dv [N, Hkv, d] (all written): the contributions of its query rows to the
 * gradient of every token's key and value.  Summed over the ranks they give the batch's
 * dK, dV (each rank keeps the rows of its own tokens: a reduce-scatter).  `saved` and
 * `loc` as left by ssa_sp_forward on the same inputs.
 *   ws: ssa_workspace_size(SSA_OP_SP_BACKWARD, p, S, Nr, B, loc->win->count) bytes.
 */
SSA_API ssa_status ssa_sp_forward(const ssa_params* p, int32_t S, int64_t N, const ssa_partition* blk,
                                  const ssa_sp_local* loc, const void* q, const void* k, const void* v,
                                  const float* gates, void* out, const ssa_saved* saved, void* ws, size_t ws_bytes,
                                  void* stream);
SSA_API ssa_status ssa_sp_backward(const ssa_params* p, int32_t S, int64_t N, const ssa_partition* blk,
                                   const ssa_sp_local* loc, const void* q, const void* k, const void* v,
                                   const float* gates, const ssa_saved* saved, const void* dout, float* dq,
                                   float* dk, float* dv, float* dgates, void* ws, size_t ws_bytes, void* stream);

/*
 * Workspace bytes needed by `op` (SSA_OP_BIN / _FORWARD / _BACKWARD / _GEO_SELECT /
 * _CROSS_FORWARD / _CROSS_BACKWARD / _SP_FORWARD / _SP_BACKWARD) for the given sizes;
 * B_tot and W_tot are the partition counts (pass N as an upper bound before binning);
 * for the cross ops N is the number of query tokens and W_tot is ignored; for the
 * sequence-parallel ops N is the rank's token count and W_tot its window count.  The workspace must be
 * 256-byte aligned.  Returns 0 for invalid arguments.
 */
SSA_API size_t ssa_workspace_size(int32_t op, const ssa_params* p, int32_t S, int64_t N,
                                  int64_t B_tot, int64_t W_tot);

/* Static, human-readable text of a status code. */
SSA_API const char* ssa_error_string(ssa_status status);

/*
 * Synchronises `stream`, then reads and clears the library's device check word
 * for the current device: SSA_OK, or the status a kernel recorded.
 */
SSA_API ssa_status ssa_get_device_status(void* stream);

/*
 * Tracing (no counterpart on the pages; used by the benchmark to time kernels).
 * ssa_launch_count: number of kernels this library has launched in this
 * process (all devices, all streams).  ssa_profile_enable(1): from now on,
 * record a CUDA event pair on the launching stream around every launch;
 * ssa_profile_enable(0) stops recording.  ssa_profile_read synchronises the
 * recorded events, writes per kernel name (at most max_entries rows, names
 * truncated to name_len-1 chars, NUL-terminated, row i at names + i*name_len)
 * the summed milliseconds and launch counts, clears the records and returns
 * the number of distinct names.  Any output pointer may be NULL.
 */
SSA_API uint64_t ssa_launch_count(void);
SSA_API void ssa_profile_enable(int32_t on);
SSA_API int32_t ssa_profile_read(char* names, int32_t name_len, float* total_ms, int32_t* launches,
                                 int32_t max_entries);

/*
 * Diagnostics (no counterpart on the pages; for tests of the library itself).
 *
 * ssa_diag_wait_timeout: launches one warp that waits on an mbarrier nothing arrives
 * at, with the same bounded waits the tensor-core kernels use (about one second of
 * device time each): first one lane, then the whole warp.  Both give up, the kernel
 * records the timeout in the device check word and returns; gave_up (device int32[2])
 * receives 1 for each wait that gave up.  The following ssa_get_device_status then
 * returns SSA_ERR_TIMEOUT, and the context stays usable.  Asynchronous.
 *
 * ssa_diag_ex2: y_poly[i] = 2^x[i] evaluated on the FMA pipe the way the kernels do
 * for part of their exponentials (x clamped at -127; 2^x = 2^j * 2^f with j = round(x),
 * 2^f a degree-5 polynomial interpolating at the Chebyshev nodes of [-1/2, 1/2]), and
 * y_mufu[i] = the hardware approximation (ex2.approx.ftz.f32).  Device pointers, n
 * values each.  Asynchronous.
 */
SSA_API ssa_status ssa_diag_wait_timeout(int32_t* gave_up, void* stream);
SSA_API ssa_status ssa_diag_ex2(const float* x, float* y_poly, float* y_mufu, int64_t n, void* stream);

/* Library version as major*10000 + minor*100 + patch. */
SSA_API int32_t ssa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H */
