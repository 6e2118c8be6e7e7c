// api.cu -- the extern "C" entry points of libfvattn.so (declared in
// include/fvattn.h): host-side validation, workspace layout, TMA tensor maps
// and kernel dispatch. No entry point allocates device memory.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace fvattn {
cudaError_t launch_permute(const void* x, void* y, int BH, int N, int d, int esize, int bs,
                           const TileGeom& g, int inverse, cudaStream_t st);
cudaError_t launch_gather_pool(const void* q, const void* k, void* qp, void* kp, float* qbar,
                               float* kbar, int BH, int N, int d, bool bf16, int bs,
                               const TileGeom& g, cudaStream_t st);
size_t route_scores_bytes(int BH, int nb);
cudaError_t launch_select_topp(const float* rows_in, int BH, int nb, float p, int k_min, int* kv_idx,
                               int* kv_cnt, unsigned long long* head_work, int* status,
                               cudaStream_t st);
cudaError_t launch_route_select(const float* qbar, const float* kbar, float* S, int BH, int nb, int d,
                                float scale, float p, int k_min, int* kv_idx, int* kv_cnt,
                                unsigned long long* head_work, int* status, cudaStream_t st);
cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, void* o, float* lse,
                             float* blse, const int* kv_idx, const int* kv_cnt, int BH, int N,
                             int d, int bs, bool bf16, float scale, int* status, cudaStream_t st);
cudaError_t launch_attn_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              void* out, float* lse, float* blse, const float* vscale,
                              const int* kv_idx, const int* kv_cnt,
                              uint32_t* ulist, int* ucnt, int* local_order,
                              unsigned long long* head_total, int* head_order, int BH, int N,
                              int nb, int bs, int d, float scale, int* status,
                              unsigned long long* counter, int num_sms, cudaStream_t st);
cudaError_t launch_block_importance(const float* blse, const float* lse, const int* kv_idx,
                                    const int* kv_cnt, int BH, int N, int bs, float* importance,
                                    int* status, cudaStream_t st);
cudaError_t launch_attention_recall(const float* importance, const int* kv_idx, const int* kv_cnt,
                                    int BH, int nb, float* recall, int* status, cudaStream_t st);
cudaError_t launch_lvsa_lists(const TileGeom& g, int N, int bs, int window, int per, int step,
                              int BH, int* kv_idx, int* kv_cnt, unsigned long long* head_work,
                              uint32_t* frames, cudaStream_t st);
cudaError_t launch_hilbert_table(int T, int Hh, int W, int* table, unsigned long long* keys,
                                 cudaStream_t st);
cudaError_t launch_quantize_v(const void* v, int BH, int N, int npad, uint8_t* vq, float* vscale,
                              unsigned int* amax_bits, cudaStream_t st);
size_t vquant_ws_bytes(int BH);
cudaError_t launch_wait_selftest(long long* out, int* status, cudaStream_t st);
cudaError_t launch_order_lists(const float* S, int BH, int nb, int* kv_idx, const int* kv_cnt, int* status,
                               cudaStream_t st);
cudaError_t launch_permute_quantize_v(const void* v, int BH, int N, int bs, const TileGeom& g, uint8_t* vq,
                                      float* vscale, unsigned int* amax_bits, cudaStream_t st);
int hilbert_bits(int extent);
int next_pow2(int n);
}  // namespace fvattn

namespace {

using fvattn::align_up;
using fvattn::kWsHeaderBytes;

constexpr int kMaxBlocks = 4096;   // nb limit (route rows live in shared memory)
constexpr int kMaxHeads = 4096;    // B*H limit (the work planner sorts heads in shared memory)
constexpr int kMaxFrames = 1024;   // LVSA frame bitmasks hold 32 words
constexpr size_t kLvsaBlockBytes = 128;   // one frame bitmask per block in the LVSA workspace

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool valid_dtype(fvattn_dtype dt) { return dt == FVATTN_BF16 || dt == FVATTN_FP32; }
int elem_size(fvattn_dtype dt) { return dt == FVATTN_BF16 ? 2 : 4; }
bool valid_d(int d) { return d == 64 || d == 128; }
bool valid_block(int b) { return b == 64 || b == 128; }

bool valid_sizes(int B, int H, int N, int d, int block) {
  if (B < 1 || H < 1 || N < 1 || !valid_d(d) || !valid_block(block)) return false;
  const long long bh = static_cast<long long>(B) * H;
  if (bh > kMaxHeads) return false;
  const long long nb = (static_cast<long long>(N) + block - 1) / block;
  if (nb > kMaxBlocks) return false;
  return true;
}

int num_blocks(int N, int block) { return (N + block - 1) / block; }

// ------------------------------------------------------------- workspace layout
// Route workspace: status header, the pooled q and k means, and the block score
// matrix [B*H, nb, nb] fp32 that the selection kernel reads back.
struct RouteWs {
  size_t qbar, kbar, scores, total;
};
RouteWs route_ws(int B, int H, int N, int d, int block) {
  const int nb = num_blocks(N, block);
  const size_t bars = static_cast<size_t>(B) * H * nb * d * sizeof(float);
  RouteWs w;
  w.qbar = kWsHeaderBytes;
  w.kbar = w.qbar + align_up(bars, 256);
  w.scores = w.kbar + align_up(bars, 256);
  w.total = w.scores + align_up(fvattn::route_scores_bytes(B * H, nb), 256);
  return w;
}

// The tensor-core kernel works on units of 256 query rows = 256/block query
// blocks; the sparse path first merges each unit's KV lists into one union list.
struct AttnWs {
  size_t ulist, ucnt, local_order, head_total, head_order, total;
};
AttnWs sparse_ws(int B, int H, int N, int block) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t nb = num_blocks(N, block);
  const size_t groups = (nb + 256 / block - 1) / (256 / block);
  AttnWs w;
  w.ulist = kWsHeaderBytes;
  w.ucnt = w.ulist + align_up(bh * groups * nb * sizeof(uint32_t), 256);
  w.local_order = w.ucnt + align_up(bh * groups * sizeof(int), 256);
  w.head_total = w.local_order + align_up(bh * groups * sizeof(int), 256);
  w.head_order = w.head_total + align_up(bh * sizeof(unsigned long long), 256);
  w.total = w.head_order + align_up(bh * sizeof(int), 256);
  return w;
}

// ------------------------------------------------------------- device properties
// Per-device SM count, cached; calls from several host threads may race to fill
// an entry, so the entries are atomics (every writer stores the same value).
int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised exactly once even when several host threads call at the same time).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// [rows, d] bf16 (d = 64 or 128), row stride 2d bytes; box = box_rows rows x 64
// columns, 128-byte swizzle.
bool make_row_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows, int d) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, 128] bytes (E4M3 V), row stride 128 B; box = box_rows rows x 128 bytes,
// 128-byte swizzle.
bool make_byte_row_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

fvattn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FVATTN_OK : FVATTN_ERR_CUDA; }

fvattn::TileGeom geom_of(const fvattn_grid* g) {
  return fvattn::TileGeom{g->T, g->Hh, g->W, g->tt, g->th, g->tw,
                          g->order == FVATTN_ORDER_TABLE ? g->table : nullptr};
}

bool valid_grid(const fvattn_grid* g, int N) {
  if (!g) return false;
  if (g->T < 1 || g->Hh < 1 || g->W < 1) return false;
  if (!valid_block(g->block)) return false;
  if (g->order == FVATTN_ORDER_TILES) {
    if (g->tt < 1 || g->th < 1 || g->tw < 1) return false;
  } else if (g->order == FVATTN_ORDER_TABLE) {
    if (!g->table || !aligned(g->table, 4)) return false;
  } else {
    return false;
  }
  const long long n = static_cast<long long>(g->T) * g->Hh * g->W;
  return n == N;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

fvattn_status check_ws(const void* ws, size_t have, size_t need) {
  if (!ws || !aligned(ws, 256) || have < need) return FVATTN_ERR_WORKSPACE;
  return FVATTN_OK;
}

// Common validation and dispatch of the attention forward (sparse or dense).
// vscale != nullptr: vp holds E4M3 codes [B*H, Npad, 128] with per-channel
// scales vscale [B*H, 128] (tensor-core path only).
fvattn_status attention_fwd(const void* qp, const void* kp, const void* vp, const float* vscale,
                            void* op, float* lse,
                            float* block_lse, const int32_t* kv_idx, const int32_t* kv_cnt, bool sparse, int B,
                            int H, int N, int d, fvattn_dtype dtype, int block, float scale,
                            void* ws, size_t ws_bytes, void* stream) {
  if (!qp || !kp || !vp || !op) return FVATTN_ERR_INVALID_ARG;
  if (vscale && !aligned(vscale, 16)) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(qp, 16) || !aligned(kp, 16) || !aligned(vp, 16) || !aligned(op, 16))
    return FVATTN_ERR_INVALID_ARG;
  if (lse && !aligned(lse, 4)) return FVATTN_ERR_INVALID_ARG;
  if (block_lse && !aligned(block_lse, 4)) return FVATTN_ERR_INVALID_ARG;
  if (sparse && (!kv_idx || !kv_cnt || !aligned(kv_idx, 4) || !aligned(kv_cnt, 4)))
    return FVATTN_ERR_INVALID_ARG;
  if (!valid_dtype(dtype) || !valid_sizes(B, H, N, d, block)) return FVATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FVATTN_ERR_INVALID_ARG;
  const bool tensor_core = dtype == FVATTN_BF16;   // d is 64 or 128 (checked above)
  if (vscale && !(tensor_core && d == 128)) return FVATTN_ERR_UNSUPPORTED;
  const size_t need = fvattn_workspace_bytes(sparse ? FVATTN_OP_SPARSE_FWD : FVATTN_OP_DENSE_FWD,
                                             B, H, N, d, block);
  const fvattn_status wst = check_ws(ws, ws_bytes, need);
  if (wst != FVATTN_OK) return wst;

  auto st = static_cast<cudaStream_t>(stream);
  auto base = static_cast<uint8_t*>(ws);
  auto hdr = reinterpret_cast<fvattn::WsHeader*>(base);
  const int BH = B * H;
  const int nb = num_blocks(N, block);
  if (cudaMemsetAsync(base, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;

  if (!tensor_core) {
    return from_cuda(fvattn::launch_attn_simt(qp, kp, vp, op, lse, block_lse, sparse ? kv_idx : nullptr,
                                              sparse ? kv_cnt : nullptr, BH, N, d, block,
                                              dtype == FVATTN_BF16, scale, &hdr->status, st));
  }
  const uint64_t rows = static_cast<uint64_t>(BH) * nb * block;
  CUtensorMap tq, tk, tv;
  if (!make_row_map(&tq, qp, rows, 128, d) || !make_row_map(&tk, kp, rows, block, d) ||
      !(vscale ? make_byte_row_map(&tv, vp, rows, block) : make_row_map(&tv, vp, rows, block, d)))
    return FVATTN_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return FVATTN_ERR_CUDA;
  uint32_t* ulist = nullptr;
  int* ucnt = nullptr;
  int* local_order = nullptr;
  unsigned long long* head_total = nullptr;
  int* head_order = nullptr;
  if (sparse) {
    const AttnWs w = sparse_ws(B, H, N, block);
    ulist = reinterpret_cast<uint32_t*>(base + w.ulist);
    ucnt = reinterpret_cast<int*>(base + w.ucnt);
    local_order = reinterpret_cast<int*>(base + w.local_order);
    head_total = reinterpret_cast<unsigned long long*>(base + w.head_total);
    head_order = reinterpret_cast<int*>(base + w.head_order);
  }
  return from_cuda(fvattn::launch_attn_sm100(
      tq, tk, tv, op, lse, block_lse, vscale, sparse ? kv_idx : nullptr, sparse ? kv_cnt : nullptr, ulist, ucnt,
      local_order, head_total, head_order, BH, N, nb, block, d, scale, &hdr->status, &hdr->counter,
      sms, st));
}

}  // namespace

extern "C" {

size_t fvattn_workspace_bytes(fvattn_op op, int B, int H, int N, int d, int block) {
  if (!valid_sizes(B, H, N, d, block)) return 0;
  switch (op) {
    case FVATTN_OP_ROUTE: return route_ws(B, H, N, d, block).total;
    case FVATTN_OP_SPARSE_FWD: return sparse_ws(B, H, N, block).total;
    case FVATTN_OP_DENSE_FWD: return kWsHeaderBytes;
    case FVATTN_OP_DIAG: return kWsHeaderBytes;
    case FVATTN_OP_LVSA: return kWsHeaderBytes + align_up(num_blocks(N, block) * kLvsaBlockBytes, 256);
    case FVATTN_OP_HILBERT:
      return kWsHeaderBytes + align_up(static_cast<size_t>(fvattn::next_pow2(N)) * 8, 256);
    case FVATTN_OP_QUANT_V:
      return kWsHeaderBytes + align_up(fvattn::vquant_ws_bytes(B * H), 256);
  }
  return 0;
}

fvattn_status fvattn_permute(const void* x, void* y, int B, int H, int N, int d,
                             fvattn_dtype dtype, const fvattn_grid* grid, int inverse,
                             void* stream) {
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return FVATTN_ERR_INVALID_ARG;
  if (!valid_dtype(dtype) || !valid_grid(grid, N)) return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, d, grid->block)) return FVATTN_ERR_INVALID_ARG;
  const int es = elem_size(dtype);
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t orig_bytes = bh * N * d * es;
  const size_t perm_bytes = bh * num_blocks(N, grid->block) * grid->block * d * es;
  if (ranges_overlap(x, inverse ? perm_bytes : orig_bytes, y, inverse ? orig_bytes : perm_bytes))
    return FVATTN_ERR_INVALID_ARG;
  return from_cuda(fvattn::launch_permute(x, y, B * H, N, d, es, grid->block, geom_of(grid),
                                          inverse ? 1 : 0, static_cast<cudaStream_t>(stream)));
}

fvattn_status fvattn_route(const void* q, const void* k, int B, int H, int N, int d,
                           fvattn_dtype dtype, const fvattn_grid* grid, float p, int k_min,
                           void* qp_out, void* kp_out, int32_t* kv_idx, int32_t* kv_cnt,
                           int64_t* head_work, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!q || !k || !kv_idx || !kv_cnt || !head_work) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(kv_idx, 4) || !aligned(kv_cnt, 4) ||
      !aligned(head_work, 8))
    return FVATTN_ERR_INVALID_ARG;
  if ((qp_out && !aligned(qp_out, 16)) || (kp_out && !aligned(kp_out, 16)))
    return FVATTN_ERR_INVALID_ARG;
  if (!valid_dtype(dtype) || !valid_grid(grid, N)) return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, d, grid->block)) return FVATTN_ERR_INVALID_ARG;
  if (!(p > 0.f && p <= 1.f) || k_min < 1) return FVATTN_ERR_INVALID_ARG;
  const int block = grid->block;
  const int nb = num_blocks(N, block);
  const RouteWs w = route_ws(B, H, N, d, block);
  const fvattn_status wst = check_ws(workspace, workspace_bytes, w.total);
  if (wst != FVATTN_OK) return wst;

  auto st = static_cast<cudaStream_t>(stream);
  auto base = static_cast<uint8_t*>(workspace);
  auto hdr = reinterpret_cast<fvattn::WsHeader*>(base);
  float* qbar = reinterpret_cast<float*>(base + w.qbar);
  float* kbar = reinterpret_cast<float*>(base + w.kbar);
  const int BH = B * H;
  if (cudaMemsetAsync(base, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  if (cudaMemsetAsync(head_work, 0, sizeof(int64_t) * BH, st) != cudaSuccess)
    return FVATTN_ERR_CUDA;
  cudaError_t e = fvattn::launch_gather_pool(q, k, qp_out, kp_out, qbar, kbar, BH, N, d,
                                             dtype == FVATTN_BF16, block, geom_of(grid), st);
  if (e != cudaSuccess) return FVATTN_ERR_CUDA;
  const float scale = 1.0f / std::sqrt(static_cast<float>(d));
  float* scores = reinterpret_cast<float*>(base + w.scores);
  e = fvattn::launch_route_select(qbar, kbar, scores, BH, nb, d, scale, p, k_min, kv_idx, kv_cnt,
                                  reinterpret_cast<unsigned long long*>(head_work), &hdr->status,
                                  st);
  return from_cuda(e);
}

fvattn_status fvattn_order_lists_by_importance(int32_t* kv_idx, const int32_t* kv_cnt, int B, int H, int N,
                                               int d, int block, void* route_workspace,
                                               size_t workspace_bytes, void* stream) {
  if (!kv_idx || !kv_cnt || !aligned(kv_idx, 4) || !aligned(kv_cnt, 4)) return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, d, block)) return FVATTN_ERR_INVALID_ARG;
  const RouteWs w = route_ws(B, H, N, d, block);
  const fvattn_status wst = check_ws(route_workspace, workspace_bytes, w.total);
  if (wst != FVATTN_OK) return wst;
  auto base = static_cast<uint8_t*>(route_workspace);
  auto hdr = reinterpret_cast<fvattn::WsHeader*>(base);
  return from_cuda(fvattn::launch_order_lists(reinterpret_cast<const float*>(base + w.scores), B * H,
                                              num_blocks(N, block), kv_idx, kv_cnt, &hdr->status,
                                              static_cast<cudaStream_t>(stream)));
}

fvattn_status fvattn_sparse_fwd(const void* qp, const void* kp, const void* vp, void* op,
                                float* lse, float* block_lse, const int32_t* kv_idx,
                                const int32_t* kv_cnt, int B, int H, int N, int d,
                                fvattn_dtype dtype, int block, float scale, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return attention_fwd(qp, kp, vp, nullptr, op, lse, block_lse, kv_idx, kv_cnt, true, B, H, N, d, dtype,
                       block, scale, workspace, workspace_bytes, stream);
}

fvattn_status fvattn_dense_fwd(const void* qp, const void* kp, const void* vp, void* op,
                               float* lse, float* block_lse, int B, int H, int N, int d,
                               fvattn_dtype dtype, int block, float scale, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return attention_fwd(qp, kp, vp, nullptr, op, lse, block_lse, nullptr, nullptr, false, B, H, N, d,
                       dtype, block, scale, workspace, workspace_bytes, stream);
}

fvattn_status fvattn_quantize_v(const void* vp, int B, int H, int N, int d, int block, uint8_t* vq,
                                float* vscale, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (!vp || !vq || !vscale) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(vp, 16) || !aligned(vq, 16) || !aligned(vscale, 16)) return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, d, block)) return FVATTN_ERR_INVALID_ARG;
  if (d != 128) return FVATTN_ERR_UNSUPPORTED;
  const size_t npad = static_cast<size_t>(num_blocks(N, block)) * block;
  const size_t bh = static_cast<size_t>(B) * H;
  if (ranges_overlap(vp, bh * npad * d * 2, vq, bh * npad * d) ||
      ranges_overlap(vp, bh * npad * d * 2, vscale, bh * d * 4) ||
      ranges_overlap(vq, bh * npad * d, vscale, bh * d * 4))
    return FVATTN_ERR_INVALID_ARG;
  const size_t need = fvattn_workspace_bytes(FVATTN_OP_QUANT_V, B, H, N, d, block);
  const fvattn_status wst = check_ws(workspace, workspace_bytes, need);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto base = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(base, 0, need, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_quantize_v(vp, B * H, N, static_cast<int>(npad), vq, vscale,
                                             reinterpret_cast<unsigned int*>(base + kWsHeaderBytes),
                                             st));
}

fvattn_status fvattn_permute_quantize_v(const void* v, int B, int H, int N, int d, const fvattn_grid* grid,
                                        uint8_t* vq, float* vscale, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  if (!v || !vq || !vscale) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(vq, 16) || !aligned(vscale, 16)) return FVATTN_ERR_INVALID_ARG;
  if (!valid_grid(grid, N) || !valid_sizes(B, H, N, d, grid->block)) return FVATTN_ERR_INVALID_ARG;
  if (d != 128) return FVATTN_ERR_UNSUPPORTED;
  const int block = grid->block;
  const size_t npad = static_cast<size_t>(num_blocks(N, block)) * block;
  const size_t bh = static_cast<size_t>(B) * H;
  if (ranges_overlap(v, bh * N * d * 2, vq, bh * npad * d) ||
      ranges_overlap(v, bh * N * d * 2, vscale, bh * d * 4) ||
      ranges_overlap(vq, bh * npad * d, vscale, bh * d * 4))
    return FVATTN_ERR_INVALID_ARG;
  const size_t need = fvattn_workspace_bytes(FVATTN_OP_QUANT_V, B, H, N, d, block);
  const fvattn_status wst = check_ws(workspace, workspace_bytes, need);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto base = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(base, 0, need, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_permute_quantize_v(v, B * H, N, block, geom_of(grid), vq, vscale,
                                                     reinterpret_cast<unsigned int*>(base + kWsHeaderBytes), st));
}

fvattn_status fvattn_sparse_fwd_fp8v(const void* qp, const void* kp, const uint8_t* vq,
                                     const float* vscale, void* op, float* lse, float* block_lse,
                                     const int32_t* kv_idx, const int32_t* kv_cnt, int B, int H,
                                     int N, int d, int block, float scale, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!vscale) return FVATTN_ERR_INVALID_ARG;
  return attention_fwd(qp, kp, vq, vscale, op, lse, block_lse, kv_idx, kv_cnt, true, B, H, N, d,
                       FVATTN_BF16, block, scale, workspace, workspace_bytes, stream);
}

fvattn_status fvattn_dense_fwd_fp8v(const void* qp, const void* kp, const uint8_t* vq,
                                    const float* vscale, void* op, float* lse, float* block_lse,
                                    int B, int H, int N, int d, int block, float scale,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!vscale) return FVATTN_ERR_INVALID_ARG;
  return attention_fwd(qp, kp, vq, vscale, op, lse, block_lse, nullptr, nullptr, false, B, H, N, d,
                       FVATTN_BF16, block, scale, workspace, workspace_bytes, stream);
}

fvattn_status fvattn_block_importance(const float* block_lse, const float* lse,
                                      const int32_t* kv_idx, const int32_t* kv_cnt, int B, int H,
                                      int N, int block, float* importance, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!block_lse || !lse || !importance) return FVATTN_ERR_INVALID_ARG;
  if ((kv_idx == nullptr) != (kv_cnt == nullptr)) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(block_lse, 4) || !aligned(lse, 4) || !aligned(importance, 4) ||
      (kv_idx && (!aligned(kv_idx, 4) || !aligned(kv_cnt, 4))))
    return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, 64, block)) return FVATTN_ERR_INVALID_ARG;
  const fvattn_status wst = check_ws(workspace, workspace_bytes, kWsHeaderBytes);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto hdr = static_cast<fvattn::WsHeader*>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_block_importance(block_lse, lse, kv_idx, kv_cnt, B * H, N, block,
                                                   importance, &hdr->status, st));
}

fvattn_status fvattn_attention_recall(const float* importance, const int32_t* kv_idx,
                                      const int32_t* kv_cnt, int B, int H, int N, int block,
                                      float* recall, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  if (!importance || !kv_idx || !kv_cnt || !recall) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(importance, 4) || !aligned(kv_idx, 4) || !aligned(kv_cnt, 4) || !aligned(recall, 4))
    return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, 64, block)) return FVATTN_ERR_INVALID_ARG;
  const fvattn_status wst = check_ws(workspace, workspace_bytes, kWsHeaderBytes);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto hdr = static_cast<fvattn::WsHeader*>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_attention_recall(importance, kv_idx, kv_cnt, B * H,
                                                   num_blocks(N, block), recall, &hdr->status, st));
}

fvattn_status fvattn_select_topp(const float* importance, int B, int H, int N, int block, float p,
                                int k_min, int32_t* kv_idx, int32_t* kv_cnt, int64_t* head_work,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!importance || !kv_idx || !kv_cnt || !head_work) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(importance, 4) || !aligned(kv_idx, 4) || !aligned(kv_cnt, 4) || !aligned(head_work, 8))
    return FVATTN_ERR_INVALID_ARG;
  if (!valid_sizes(B, H, N, 64, block)) return FVATTN_ERR_INVALID_ARG;
  if (!(p > 0.f && p <= 1.f) || k_min < 1) return FVATTN_ERR_INVALID_ARG;
  const fvattn_status wst = check_ws(workspace, workspace_bytes, kWsHeaderBytes);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto hdr = static_cast<fvattn::WsHeader*>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  if (cudaMemsetAsync(head_work, 0, sizeof(int64_t) * B * H, st) != cudaSuccess)
    return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_select_topp(importance, B * H, num_blocks(N, block), p, k_min, kv_idx,
                                              kv_cnt, reinterpret_cast<unsigned long long*>(head_work),
                                              &hdr->status, st));
}

fvattn_status fvattn_lvsa_lists(int B, int H, const fvattn_grid* grid, int window, int period,
                                int step, int32_t* kv_idx, int32_t* kv_cnt, int64_t* head_work,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!grid || !kv_idx || !kv_cnt || !head_work) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(kv_idx, 4) || !aligned(kv_cnt, 4) || !aligned(head_work, 8))
    return FVATTN_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(grid->T) * grid->Hh * grid->W;
  if (n < 1 || n > (1ll << 30)) return FVATTN_ERR_INVALID_ARG;
  const int N = static_cast<int>(n);
  if (!valid_grid(grid, N) || !valid_sizes(B, H, N, 64, grid->block)) return FVATTN_ERR_INVALID_ARG;
  if (grid->T > kMaxFrames || window < 0 || period < 1) return FVATTN_ERR_INVALID_ARG;
  const size_t need = fvattn_workspace_bytes(FVATTN_OP_LVSA, B, H, N, 64, grid->block);
  const fvattn_status wst = check_ws(workspace, workspace_bytes, need);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto base = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(base, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  if (cudaMemsetAsync(head_work, 0, sizeof(int64_t) * B * H, st) != cudaSuccess)
    return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_lvsa_lists(
      geom_of(grid), N, grid->block, window, period, step, B * H, kv_idx, kv_cnt,
      reinterpret_cast<unsigned long long*>(head_work),
      reinterpret_cast<uint32_t*>(base + kWsHeaderBytes), st));
}

fvattn_status fvattn_hilbert_table(const fvattn_grid* grid, int32_t* table, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (!grid || !table || !aligned(table, 4)) return FVATTN_ERR_INVALID_ARG;
  if (grid->T < 1 || grid->Hh < 1 || grid->W < 1 || !valid_block(grid->block))
    return FVATTN_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(grid->T) * grid->Hh * grid->W;
  if (n > static_cast<long long>(kMaxBlocks) * grid->block) return FVATTN_ERR_INVALID_ARG;
  const int N = static_cast<int>(n);
  const int b = fvattn::hilbert_bits(std::max(grid->T, std::max(grid->Hh, grid->W)));
  if (3 * b + fvattn::hilbert_bits(N) > 64) return FVATTN_ERR_UNSUPPORTED;
  const size_t need = fvattn_workspace_bytes(FVATTN_OP_HILBERT, 1, 1, N, 64, grid->block);
  const fvattn_status wst = check_ws(workspace, workspace_bytes, need);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto base = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(base, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_hilbert_table(
      grid->T, grid->Hh, grid->W, table, reinterpret_cast<unsigned long long*>(base + kWsHeaderBytes), st));
}

fvattn_status fvattn_wait_selftest(int64_t* results, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!results || !aligned(results, 8)) return FVATTN_ERR_INVALID_ARG;
  const fvattn_status wst = check_ws(workspace, workspace_bytes, kWsHeaderBytes);
  if (wst != FVATTN_OK) return wst;
  auto st = static_cast<cudaStream_t>(stream);
  auto hdr = static_cast<fvattn::WsHeader*>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, st) != cudaSuccess) return FVATTN_ERR_CUDA;
  if (cudaMemsetAsync(results, 0, 8 * sizeof(int64_t), st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return from_cuda(fvattn::launch_wait_selftest(reinterpret_cast<long long*>(results), &hdr->status, st));
}

fvattn_status fvattn_workspace_status(const void* workspace, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return FVATTN_ERR_WORKSPACE;
  int h = 0;
  auto st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FVATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FVATTN_ERR_CUDA;
  return static_cast<fvattn_status>(h);
}

const char* fvattn_status_string(fvattn_status s) {
  switch (s) {
    case FVATTN_OK: return "ok";
    case FVATTN_ERR_INVALID_ARG: return "invalid argument";
    case FVATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case FVATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FVATTN_ERR_CUDA: return "CUDA runtime error";
    case FVATTN_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
