// importance.cu -- exact block importance and attention recall from the block
// log-sum-exps that the attention kernels record
// [GSRS §5.3, §A.3: per-block log-sum-exp statistics recorded during the
// attention pass are normalised with each row's own log-sum-exp, after the
// kernel, to recover the exact importance; GSRS §A.2: the weights of the
// evaluated blocks sum to one; GSRS §3.2: attention recall].
//
//   importance[b,h,i,j] = (1/n_i) * sum over valid rows r of query block i of
//                         exp(block_lse[b,h,j,r] - lse[b,h,r])
// for the key blocks j that block i evaluated (its list, or all blocks), 0 for
// the others; n_i = valid rows of block i.
//   recall[b,h,i] = sum over the blocks of a list of importance[b,h,i,j].
//
// Both kernels are a few MB of reads per call next to the attention pass:
// one CTA per (b, h, query block), one warp per evaluated key block, rows
// read contiguously (block_lse is laid out [key block][row]).
#include "common.cuh"

namespace fvattn {

constexpr int kImpThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Valid list length of row (bh, i), or nb without lists; records and clamps bad counts.
__device__ __forceinline__ int list_len(const int* kv_cnt, size_t row, int nb, int* status) {
  if (!kv_cnt) return nb;
  int c = kv_cnt[row];
  if (c < 1 || c > nb) {
    if (threadIdx.x == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
    c = min(max(c, 1), nb);
  }
  return c;
}

__global__ void __launch_bounds__(kImpThreads)
    block_importance_kernel(const float* __restrict__ blse, const float* __restrict__ lse,
                            const int* __restrict__ kv_idx, const int* __restrict__ kv_cnt,
                            int nb, int N, int bs, float* __restrict__ importance, int* status) {
  extern __shared__ float lse_s[];   // bs floats: the row LSEs of this query block
  const int bh = blockIdx.x / nb;
  const int i = blockIdx.x - bh * nb;
  const size_t npad = static_cast<size_t>(nb) * bs;
  const size_t row0 = static_cast<size_t>(bh) * npad + static_cast<size_t>(i) * bs;
  const int nr = min(bs, N - i * bs);
  const size_t irow = static_cast<size_t>(bh) * nb + i;
  float* out = importance + irow * nb;
  for (int r = threadIdx.x; r < nr; r += blockDim.x) lse_s[r] = lse[row0 + r];
  for (int j = threadIdx.x; j < nb; j += blockDim.x) out[j] = 0.f;
  __syncthreads();
  const int cnt = list_len(kv_cnt, irow, nb, status);
  const int* list = kv_idx ? kv_idx + irow * nb : nullptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float inv_n = 1.f / static_cast<float>(nr);
  for (int t = warp; t < cnt; t += kImpThreads / 32) {
    const int j = list ? list[t] : t;
    if (j < 0 || j >= nb) {
      if (lane == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
      continue;
    }
    const float* src = blse + (static_cast<size_t>(bh) * nb + j) * npad + static_cast<size_t>(i) * bs;
    float acc = 0.f;
    for (int r = lane; r < nr; r += 32) acc += expf(src[r] - lse_s[r]);
    acc = warp_sum(acc);
    if (lane == 0) out[j] = acc * inv_n;
  }
}

// One warp per (b, h, query block).
__global__ void __launch_bounds__(kImpThreads)
    attention_recall_kernel(const float* __restrict__ importance, const int* __restrict__ kv_idx,
                            const int* __restrict__ kv_cnt, int rows, int nb, float* __restrict__ recall,
                            int* status) {
  const int wid = (blockIdx.x * kImpThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= rows) return;
  const size_t irow = static_cast<size_t>(wid);
  int c = kv_cnt[irow];
  if (c < 1 || c > nb) {
    if (lane == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
    c = min(max(c, 1), nb);
  }
  const int* list = kv_idx + irow * nb;
  const float* imp = importance + irow * nb;
  float acc = 0.f;
  for (int t = lane; t < c; t += 32) {
    const int j = list[t];
    if (j >= 0 && j < nb) acc += imp[j];
    else record_status(status, FVATTN_ERR_INVALID_ARG);
  }
  acc = warp_sum(acc);
  if (lane == 0) recall[irow] = acc;
}

cudaError_t launch_block_importance(const float* blse, const float* lse, const int* kv_idx,
                                    const int* kv_cnt, int BH, int N, int bs, float* importance,
                                    int* status, cudaStream_t st) {
  const int nb = (N + bs - 1) / bs;
  block_importance_kernel<<<static_cast<unsigned>(BH) * nb, kImpThreads, bs * sizeof(float), st>>>(
      blse, lse, kv_idx, kv_cnt, nb, N, bs, importance, status);
  return cudaGetLastError();
}

cudaError_t launch_attention_recall(const float* importance, const int* kv_idx, const int* kv_cnt,
                                    int BH, int nb, float* recall, int* status, cudaStream_t st) {
  const int rows = BH * nb;
  const int warps_per_cta = kImpThreads / 32;
  attention_recall_kernel<<<(rows + warps_per_cta - 1) / warps_per_cta, kImpThreads, 0, st>>>(
      importance, kv_idx, kv_cnt, rows, nb, recall, status);
  return cudaGetLastError();
}

}  // namespace fvattn
