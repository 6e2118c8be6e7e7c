/*
 * fvattn.h -- C ABI of libfvattn.so: the data-parallel hot path of training-free
 * adaptive block-sparse self-attention for video DiTs, built for NVIDIA B200
 * (sm_100a).
 *
 * Sources (page title, section):
 *   [FVAttn] "FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for
 *            Video Generation" (Liu et al.; Chinese translation, English summary
 *            and abstract pages).
 *   [GSRS]   "Sparse Attention for Video Generation Acceleration via Growing
 *            Sparsity and Reduced Search".
 *
 * The path, per attention call of one layer:
 *   fvattn_route      3-D tile permutation of Q and K, block-mean pooling, block
 *                     score softmax, Top-p selection with a Top-k floor, KV block
 *                     lists and per-head work            [FVAttn §2.1, §2.2, §3.1]
 *   fvattn_permute    the same permutation for V (forward) and, inverse, for the
 *                     attention output                   [FVAttn §3.1]
 *   fvattn_sparse_fwd block-sparse attention over the routed lists
 *                                                        [FVAttn §2.1; GSRS §3.2, §A.1]
 *   fvattn_dense_fwd  the same kernel with every block selected (the dense
 *                     baseline every page compares against)
 *   fvattn_order_lists_by_importance  optional: the routed lists in importance
 *                     order (descending block score)     [FVAttn §3.1]
 * Other entry points: fvattn_route_noalloc (routing for callers that cannot hand
 * the library a workspace) and fvattn_wait_selftest (the kernels' bounded waits
 * exercised without a fault).
 * Diagnostic of mask quality, from statistics the attention kernels record:
 *   fvattn_block_importance  exact block importance   [GSRS §5.3, §A.2, §A.3]
 *   fvattn_attention_recall  attention recall of a mask            [GSRS §3.2]
 *   fvattn_select_topp       Top-p + Top-k floor on exact importance: the
 *                            GSRS search over a candidate set [GSRS §5.1, §5.2]
 * A second, static mask generator for the same attention kernel:
 *   fvattn_lvsa_lists  local window + rotating global frames        [LVSA §3]
 * Hilbert-curve block order, used through fvattn_grid.order:
 *   fvattn_hilbert_table  the permutation table of a grid   [FVAttn §3.1; GSRS §A.6]
 * Low-precision V [FVAttn §3.4]:
 *   fvattn_quantize_v       per-channel E4M3 codes and scales of the permuted V
 *   fvattn_permute_quantize_v  the same codes straight from the raster-order V,
 *                           fused with the block-order permutation
 *   fvattn_sparse_fwd_fp8v, fvattn_dense_fwd_fp8v
 *                           attention with that V (8-bit P.V on the tensor cores)
 *
 * Conventions (every entry point):
 *   - Tensors are dense, row-major, on the current CUDA device. A token row of
 *     d elements is contiguous. Shapes are given in the comments as [B,H,N,d].
 *   - N = T*Hh*W tokens in raster (t, y, x) order. nb = ceil(N/block) blocks;
 *     Npad = nb*block. "Permuted" tensors are [B,H,Npad,d] in the grid's block
 *     order (3-D tiles, or an explicit table such as the Hilbert order) with
 *     the last Npad-N rows zero (written by fvattn_route / fvattn_permute).
 *   - The caller owns every buffer, including the workspace; the library never
 *     allocates or frees device memory and keeps no global state beyond a
 *     per-device cache of device properties.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronizes the host, except
 *     fvattn_workspace_status.
 *   - Arguments are validated on the host before any launch: null pointers,
 *     16-byte alignment of tensor pointers, shapes, dtype, block size, p and
 *     k_min. On failure nothing is launched and a status is returned.
 *   - Kernels never trap. A kernel that meets an out-of-range list entry clamps
 *     it and records FVATTN_ERR_INVALID_ARG in the workspace status word; a
 *     bounded wait that runs out records FVATTN_ERR_TIMEOUT there and the kernel
 *     returns. fvattn_workspace_status reads that word back.
 *   - No exception crosses this ABI.
 */
#ifndef FVATTN_H_
#define FVATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FVATTN_API __attribute__((visibility("default")))
#else
#define FVATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FVATTN_OK = 0,
  FVATTN_ERR_INVALID_ARG = 1, /* bad pointer, shape or parameter            */
  FVATTN_ERR_UNSUPPORTED = 2, /* valid but not implemented for this shape    */
  FVATTN_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small  */
  FVATTN_ERR_CUDA = 4,        /* a CUDA runtime call failed                  */
  FVATTN_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out          */
} fvattn_status;

typedef enum {
  FVATTN_BF16 = 0, /* tensor-core path (d = 128) and SIMT path (d = 64)     */
  FVATTN_FP32 = 1  /* SIMT path only (fp32 arithmetic throughout)           */
} fvattn_dtype;

/* Block order of the token sequence [FVAttn §3.1; GSRS §A.6]. */
typedef enum {
  FVATTN_ORDER_TILES = 0, /* 3-D tiles (tt, th, tw), closed-form map          */
  FVATTN_ORDER_TABLE = 1  /* explicit table, e.g. from fvattn_hilbert_table   */
} fvattn_order;

/* Latent video grid and block order. */
typedef struct {
  int T, Hh, W;        /* grid extents; N = T*Hh*W                                  */
  int tt, th, tw;      /* tile extents (>= 1; FVATTN_ORDER_TILES); edge tiles may be
                          partial                                                   */
  int block;           /* tokens per block: 64 or 128                               */
  int order;           /* fvattn_order                                              */
  const int32_t* table;/* FVATTN_ORDER_TABLE: device [N], table[pos] = raster index
                          (t*Hh + y)*W + x of the token at permuted position pos; a
                          permutation of [0, N) (entries outside it are skipped)    */
} fvattn_grid;

typedef enum {
  FVATTN_OP_ROUTE = 0,
  FVATTN_OP_SPARSE_FWD = 1,
  FVATTN_OP_DENSE_FWD = 2,
  FVATTN_OP_DIAG = 3,     /* fvattn_block_importance, fvattn_attention_recall */
  FVATTN_OP_LVSA = 4,     /* fvattn_lvsa_lists */
  FVATTN_OP_HILBERT = 5,  /* fvattn_hilbert_table */
  FVATTN_OP_QUANT_V = 6   /* fvattn_quantize_v */
} fvattn_op;

/* Workspace bytes needed by `op` for these sizes (0 if the sizes are invalid).
 * The workspace must be 256-byte aligned. Its first 256 bytes hold the status
 * word, cleared at the start of every call that takes it. */
FVATTN_API size_t fvattn_workspace_bytes(fvattn_op op, int B, int H, int N, int d, int block);

/* Block-order permutation [FVAttn §3.1; GSRS §A.6].
 * inverse == 0: x [B,H,N,d] (original order) -> y [B,H,Npad,d] (tile order,
 *               pad rows zeroed).
 * inverse != 0: x [B,H,Npad,d] (tile order)  -> y [B,H,N,d] (original order,
 *               pad rows dropped).
 * FVATTN_ORDER_TILES: the token at grid (t,y,x) moves to position pos(t,y,x):
 * tiles in raster order over the tile grid, raster order inside a tile.
 * FVATTN_ORDER_TABLE: position pos holds the token grid->table[pos].
 * x and y must not overlap.
 * d in {64, 128}; dtype BF16 or FP32. Bit-exact copy. */
FVATTN_API fvattn_status fvattn_permute(const void* x, void* y, int B, int H, int N, int d,
                             fvattn_dtype dtype, const fvattn_grid* grid,
                             int inverse, void* stream);

/* Routing front end [FVAttn §2.1, §2.2 Eq. (1), §3.1; GSRS §5.2, §5.3, §A.4].
 * q, k      [B,H,N,d] in ORIGINAL token order.
 * qp_out, kp_out  optional (NULL to skip) [B,H,Npad,d]: q and k permuted to
 *           tile order, written by the same pass that pools them.
 * Per (b,h) and query block i (blocks of the permuted sequence):
 *   qbar_i, kbar_j = fp32 means over the valid tokens of each block;
 *   s_ij = softmax_j(qbar_i . kbar_j / sqrt(d))  (fp32, max-subtracted);
 *   n_p  = the smallest c such that the c largest s_ij sum to >= p
 *          (nb when p >= 1 or when no prefix reaches p);
 *   cnt  = min(nb, max(n_p, k_min)); the selected blocks are the cnt largest
 *          (ties: lower block index ranks first).
 * Outputs:
 *   kv_idx    [B,H,nb,nb] int32: row (b,h,i) holds its cnt selected key blocks
 *             in ascending block index at entries [0, cnt); entries >= cnt are
 *             not written.
 *   kv_cnt    [B,H,nb] int32: cnt per query block.
 *   head_work [B,H] int64: sum_i cnt = nb * L_h of Eq. (1).
 * 0 < p <= 1, k_min >= 1, d in {64,128}, block in {64,128}, N = T*Hh*W,
 * nb <= 4096. Workspace: fvattn_workspace_bytes(FVATTN_OP_ROUTE, ...): the
 * status word, the pooled means (2 x B*H*nb*d fp32) and the block score matrix
 * (B*H*nb*nb fp32). */
FVATTN_API fvattn_status fvattn_route(const void* q, const void* k, int B, int H, int N, int d,
                           fvattn_dtype dtype, const fvattn_grid* grid, float p,
                           int k_min, void* qp_out, void* kp_out, int32_t* kv_idx,
                           int32_t* kv_cnt, int64_t* head_work, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Importance order of the routed lists [FVAttn §3.1: the routing front end
 * yields a block-importance ranking, which slack augmentation consumes in
 * order]: reorders the first kv_cnt[b,h,i] entries of every row of kv_idx, in
 * place, by descending block score of the preceding fvattn_route call made
 * with the same workspace (same B, H, N, d, block; the workspace still holds
 * that call's block scores), ties in ascending block index. The set of each row
 * is unchanged and the attention entry points accept either order (results
 * agree up to fp32 rounding order). kv_idx [B,H,nb,nb] int32 in/out, kv_cnt
 * [B,H,nb] int32 in. A count outside [1, nb] or an entry outside [0, nb) is
 * clamped and recorded as FVATTN_ERR_INVALID_ARG in the route workspace's
 * status word. Workspace: the route's (fvattn_workspace_bytes(FVATTN_OP_ROUTE, ...)). */
FVATTN_API fvattn_status fvattn_order_lists_by_importance(int32_t* kv_idx, const int32_t* kv_cnt, int B, int H,
                                                          int N, int d, int block, void* route_workspace,
                                                          size_t workspace_bytes, void* stream);

/* fvattn_route for callers that cannot allocate device memory at the call
 * site (an engine plugin with no scratch buffer to offer, or a hot loop where
 * cudaMalloc would synchronize the device). The pages have no counterpart to
 * this call; it exists only for how the library is embedded.
 * Same arguments and results as fvattn_route, minus the workspace: the scratch
 * is a library-owned static device array of 96 MiB that every GPU loading the
 * library keeps until exit. Sizes whose route workspace exceeds 96 MiB return
 * FVATTN_ERR_WORKSPACE and launch nothing. All calls on a device share the
 * array, so calls that overlap on the GPU race; the first call on each device
 * looks up the array's address (do it before any stream capture). The address
 * is cached per device and per CUDA context: a call under a context other than
 * the one of that lookup (after cudaDeviceReset, or with a caller-made context
 * current) looks it up again, and that call too belongs before any capture.
 * Nothing is allocated. Kernel-side status words are not reported by this
 * variant. */
FVATTN_API fvattn_status fvattn_route_noalloc(const void* q, const void* k, int B, int H, int N,
                                              int d, fvattn_dtype dtype, const fvattn_grid* grid,
                                              float p, int k_min, void* qp_out, void* kp_out,
                                              int32_t* kv_idx, int32_t* kv_cnt,
                                              int64_t* head_work, void* stream);

/* Block-sparse attention forward [FVAttn §2.1; GSRS §3.2, §A.1].
 * qp, kp, vp [B,H,Npad,d] in tile order (pad rows zero), op [B,H,Npad,d] out.
 * For every query token of query block i: softmax over the valid keys (index
 * < N) of the key blocks kv_idx[b,h,i,0..cnt) of scale * q.k, times V.
 * lse: optional [B,H,Npad] fp32 natural-log sum of exp of the scaled logits
 * over the attended keys (NULL to skip). Rows >= N of op and lse are written
 * but carry no meaning.
 * block_lse: optional [B,H,nb,Npad] fp32 (key block major) [GSRS §5.3, §A.3]:
 * entry (b,h,j,r) = natural-log sum of exp of the scaled logits of row r over
 * the valid keys of key block j, written only for the (row, key block) pairs
 * the row attends (its block's list); other entries are left untouched. With
 * lse it gives the exact block importance (fvattn_block_importance). NULL to
 * skip; the tensor-core kernel then does no extra work. kv_idx/kv_cnt as produced by fvattn_route (any order
 * of entries within a row is accepted). scale > 0 (1/sqrt(d) is the usual).
 * BF16 (d 64 or 128, block 64 or 128) runs the tcgen05/TMEM tensor-core
 * kernel (bf16 MMA, fp32 accumulation and softmax, P rounded to bf16); it
 * processes 256 query rows at a time over the union of their blocks' lists,
 * masking each row to its own block's list. FP32 runs the SIMT kernel (fp32
 * throughout; the tensor cores have no fp32 path with that accuracy).
 * Workspace: fvattn_workspace_bytes(FVATTN_OP_SPARSE_FWD, ...). */
FVATTN_API fvattn_status fvattn_sparse_fwd(const void* qp, const void* kp, const void* vp,
                                void* op, float* lse, float* block_lse,
                                const int32_t* kv_idx,
                                const int32_t* kv_cnt, int B, int H, int N, int d,
                                fvattn_dtype dtype, int block, float scale,
                                void* workspace, size_t workspace_bytes,
                                void* stream);

/* Dense attention forward [FVAttn §4.1: dense FlashAttention is the 1.00x
 * baseline of every latency table]: fvattn_sparse_fwd with every key block
 * selected, on the same kernels (block_lse, when given, is written for every
 * (row, key block) pair). Same arguments, layouts, ownership and errors as
 * fvattn_sparse_fwd without kv_idx/kv_cnt.
 * Workspace: fvattn_workspace_bytes(FVATTN_OP_DENSE_FWD, ...). */
FVATTN_API fvattn_status fvattn_dense_fwd(const void* qp, const void* kp, const void* vp,
                               void* op, float* lse, float* block_lse, int B, int H, int N,
                               int d,
                               fvattn_dtype dtype, int block, float scale,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* Per-channel FP8 quantization of V [FVAttn §3.4: the GPU quantizes V in a
 * step of its own before attention; the pages name no format].
 * vp [B,H,Npad,128] bf16 in tile order (the input of fvattn_sparse_fwd);
 * vq [B,H,Npad,128] uint8 E4M3 codes out (OCP FP8 E4M3: sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, largest finite 448); vscale [B,H,128] fp32 out.
 * For each (b,h,channel c): amax_c = max |v| over the valid rows (< N);
 *   vscale[c] = fp32(amax_c / 448) and
 *   vq[r,c]   = round-to-nearest-even E4M3 of fp32(v[r,c] * fp32(448 / amax_c)),
 * saturating at +-448 (both fp32 operations correctly rounded); a channel with
 * amax_c < 2^-100 gets codes 0 and scale 0; rows >= N get code 0. The
 * dequantized value is E4M3(vq) * vscale. V must be finite (a NaN is left out
 * of amax_c and encodes as the NaN code). d must be 128 (FVATTN_ERR_UNSUPPORTED
 * otherwise); vp, vq and vscale 16-byte aligned and not overlapping.
 * Workspace: fvattn_workspace_bytes(FVATTN_OP_QUANT_V, ...) (per-channel maxima). */
FVATTN_API fvattn_status fvattn_quantize_v(const void* vp, int B, int H, int N, int d, int block,
                                           uint8_t* vq, float* vscale, void* workspace,
                                           size_t workspace_bytes, void* stream);

/* The block-order permutation of V fused with its per-channel FP8 quantization
 * [FVAttn §3.1 block order; §3.4 the GPU quantizes V before attention]:
 * v [B,H,N,128] bf16 in raster order (the input of fvattn_permute) in, vq
 * [B,H,Npad,128] uint8 and vscale [B,H,128] fp32 out, equal bit for bit to
 * fvattn_permute followed by fvattn_quantize_v (same definition of codes,
 * scales, zero channels and zero pad rows; the grid's order, tiles or table,
 * places the rows). V is read twice (channel maxima, then gather and encode)
 * and the permuted bf16 V is never written: 1.5 B of traffic per V element
 * less than the two calls. d must be 128 (FVATTN_ERR_UNSUPPORTED otherwise);
 * v, vq and vscale 16-byte aligned and not overlapping; grid as for
 * fvattn_permute. Workspace: fvattn_workspace_bytes(FVATTN_OP_QUANT_V, ...). */
FVATTN_API fvattn_status fvattn_permute_quantize_v(const void* v, int B, int H, int N, int d,
                                                   const fvattn_grid* grid, uint8_t* vq, float* vscale,
                                                   void* workspace, size_t workspace_bytes, void* stream);

/* Block-sparse attention forward with the FP8 V of fvattn_quantize_v:
 * fvattn_sparse_fwd's definition with V replaced by E4M3(vq) * vscale. qp, kp
 * bf16 [B,H,Npad,128]; vq, vscale as written by fvattn_quantize_v (16-byte
 * aligned). Runs the tensor-core kernel with an 8-bit P.V product
 * (kind::f8f6f4): P is rounded to E4M3 too, relative to a reference 2^4 below
 * the running row max (so P <= 256 < 448), with row sums over the rounded P;
 * the channel scales are applied with 1/l at the end. Q.K^T and the running
 * max stay as in fvattn_sparse_fwd; lse and block_lse are formed from the row
 * sums of the rounded P, so they carry its rounding (relative error of the sums
 * at most about 2^-4). d must be 128 (FVATTN_ERR_UNSUPPORTED otherwise).
 * Workspace: as fvattn_sparse_fwd. */
FVATTN_API fvattn_status fvattn_sparse_fwd_fp8v(const void* qp, const void* kp, const uint8_t* vq,
                                                const float* vscale, void* op, float* lse,
                                                float* block_lse, const int32_t* kv_idx,
                                                const int32_t* kv_cnt, int B, int H, int N, int d,
                                                int block, float scale, void* workspace,
                                                size_t workspace_bytes, void* stream);

/* Dense attention forward with the FP8 V: fvattn_sparse_fwd_fp8v with every key
 * block selected. Workspace: as fvattn_dense_fwd. */
FVATTN_API fvattn_status fvattn_dense_fwd_fp8v(const void* qp, const void* kp, const uint8_t* vq,
                                               const float* vscale, void* op, float* lse,
                                               float* block_lse, int B, int H, int N, int d,
                                               int block, float scale, void* workspace,
                                               size_t workspace_bytes, void* stream);

/* Exact block importance [GSRS §5.3, §A.2, §A.3] from the block_lse and lse
 * of one attention call (sparse or dense, same B, H, N, block):
 *   importance[b,h,i,j] = (1/n_i) * sum over the valid rows r of query block i
 *                         of exp(block_lse[b,h,j,r] - lse[b,h,r])
 * for the key blocks j in row (b,h,i) of kv_idx/kv_cnt (the evaluated set;
 * both NULL = every block, for a dense call), and 0 for every other j;
 * n_i = valid rows of block i. Each row of importance sums to 1 over its
 * evaluated set. importance [B,H,nb,nb] fp32 is fully written.
 * Workspace: fvattn_workspace_bytes(FVATTN_OP_DIAG, ...) (status word only). */
FVATTN_API fvattn_status fvattn_block_importance(const float* block_lse, const float* lse,
                                                 const int32_t* kv_idx, const int32_t* kv_cnt,
                                                 int B, int H, int N, int block,
                                                 float* importance, void* workspace,
                                                 size_t workspace_bytes, void* stream);

/* Top-p selection with a Top-k floor on given importance rows [GSRS §5.1,
 * §5.2, §5.3, §A.4]: the search step of GSRS, where the exact importance of a
 * candidate set (fvattn_block_importance of a call over the candidate lists)
 * chooses the blocks to keep. importance [B,H,nb,nb] fp32, each row
 * non-negative and summing to one over its evaluated blocks (0 elsewhere).
 * Per row, as in fvattn_route but without the softmax: n_p = the smallest c
 * whose c largest importances sum to >= p (nb when p >= 1 or when no prefix
 * reaches p), cnt = min(nb, max(n_p, k_min)), ties by lower block index; the
 * selected blocks go to kv_idx [B,H,nb,nb] (ascending at [0, cnt)), kv_cnt
 * [B,H,nb], head_work [B,H] = sum_i cnt. With p < 1 and k_min no larger than
 * the candidate count, only candidates are selected. Entries outside [0, 1]
 * are clamped and recorded as FVATTN_ERR_INVALID_ARG.
 * Workspace: fvattn_workspace_bytes(FVATTN_OP_DIAG, ...). */
FVATTN_API fvattn_status fvattn_select_topp(const float* importance, int B, int H, int N, int block,
                                            float p, int k_min, int32_t* kv_idx, int32_t* kv_cnt,
                                            int64_t* head_work, void* workspace,
                                            size_t workspace_bytes, void* stream);

/* Attention recall of a block mask [GSRS §3.2]: the fraction of the attention
 * weight that the listed blocks capture,
 *   recall[b,h,i] = sum over t < kv_cnt[b,h,i] of importance[b,h,i,kv_idx[b,h,i,t]],
 * where importance comes from fvattn_block_importance of a dense call (so it
 * is normalised over every key). recall [B,H,nb] fp32.
 * Workspace: fvattn_workspace_bytes(FVATTN_OP_DIAG, ...). */
FVATTN_API fvattn_status fvattn_attention_recall(const float* importance, const int32_t* kv_idx,
                                                 const int32_t* kv_cnt, int B, int H, int N,
                                                 int block, float* recall, void* workspace,
                                                 size_t workspace_bytes, void* stream);

/* Hilbert-curve token order of grid (T, Hh, W) [FVAttn §3.1; GSRS §A.6], for
 * FVATTN_ORDER_TABLE grids. Tokens are ordered by their index on the 3-D
 * Hilbert curve over (t, y, x) of the smallest cube of side 2^b holding the
 * grid (b = bits of max(T, Hh, W)); the index is Skilling's ("Programming the
 * Hilbert curve", 2004) with t as the first axis. table [N] int32 (device) gets
 * table[pos] = raster index of the pos-th token along the curve. Built once per
 * grid (one key pass, a bitonic sort of next_pow2(N) 64-bit keys, one gather).
 * Uses only T, Hh, W and block of `grid`. Needs 3b + bits(N) <= 64
 * (FVATTN_ERR_UNSUPPORTED otherwise). Workspace:
 * fvattn_workspace_bytes(FVATTN_OP_HILBERT, 1, 1, N, 64, block). */
FVATTN_API fvattn_status fvattn_hilbert_table(const fvattn_grid* grid, int32_t* table,
                                              void* workspace, size_t workspace_bytes,
                                              void* stream);

/* KV block lists of the LVSA static pattern [LVSA §3], in the layout that
 * fvattn_route produces and fvattn_sparse_fwd consumes.
 * Frames: query frame t attends A(t) = G ∪ W(t) with
 *   G    = { g in [0,T) : g = step (mod period) }  (equidistant global frames,
 *          rotated by the denoising step);
 *   W(t) = [t-window, t+window] clipped to [0,T), then expanded until
 *          |A(t)| = |G| + min(2*window+1, T-|G|) for every t: each pass adds the
 *          current deficit, ceil(deficit/2) frames after t and the rest before
 *          t, a clipped side handing its share to the other side.
 * Blocks: blocks of the tile-ordered sequence of `grid` (as fvattn_permute);
 * key block j is listed for query block i when a valid token of i lies in a
 * frame tq and a valid token of j in a frame of A(tq).
 * Outputs, the same for every (b,h): kv_idx [B,H,nb,nb] (ascending at entries
 * [0,cnt)), kv_cnt [B,H,nb], head_work [B,H] = sum_i cnt.
 * T <= 1024, window >= 0, period >= 1, any step. Workspace:
 * fvattn_workspace_bytes(FVATTN_OP_LVSA, B, H, N, d, block) for any valid d. */
FVATTN_API fvattn_status fvattn_lvsa_lists(int B, int H, const fvattn_grid* grid, int window,
                                           int period, int step, int32_t* kv_idx, int32_t* kv_cnt,
                                           int64_t* head_work, void* workspace,
                                           size_t workspace_bytes, void* stream);

/* Synchronizes `stream` and returns the status word that the kernels of the
 * last call using `workspace` recorded (FVATTN_OK if none). */
FVATTN_API fvattn_status fvattn_workspace_status(const void* workspace, void* stream);

/* Self-test of the bounded device waits (failure detection; the pages have no
 * counterpart: their runtime balances stragglers but detects no faults).
 * Every wait of the library's kernels on an mbarrier gives up after a fixed
 * limit of the GPU's global timer (2 s), raises an abort flag that releases
 * every other waiter of the block, and records FVATTN_ERR_TIMEOUT in the
 * workspace status word, so a lost arrival ends the kernel instead of hanging
 * the GPU. This call runs those waits on barriers that nothing arrives at: one
 * block of 64 threads, no other memory touched. After the stream reaches it
 * (about two limits, 4 s), fvattn_workspace_status reads FVATTN_ERR_TIMEOUT and
 * the device context is still usable.
 *   results  [8] int64, device, written: [0] 1 if the first wait succeeded
 *            (expected 0), [1] its duration in ns (about the limit), [2] and [3]
 *            the same for a wait in another warp released by the abort flag,
 *            [4] and [5] for the final-drain form of the wait (no abort flag),
 *            [6] the limit in ns, [7] the abort flag (expected 1).
 * Workspace: 256 bytes, 256-byte aligned (fvattn_workspace_bytes of
 * FVATTN_OP_DENSE_FWD gives that size). Returns FVATTN_OK once launched. */
FVATTN_API fvattn_status fvattn_wait_selftest(int64_t* results, void* workspace, size_t workspace_bytes,
                                              void* stream);

/* Static string for a status code (never NULL). */
FVATTN_API const char* fvattn_status_string(fvattn_status status);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_H_ */
