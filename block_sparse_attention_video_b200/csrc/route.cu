// route.cu -- block scores, softmax and Top-p / Top-k-floor selection
// [FVAttn §2.1, §2.2 Eq. (1), §3.1; GSRS §5.2, §5.3, §A.4].
//
// Two kernels, each at high occupancy:
//   1. block_scores_kernel: S[b,h,i,j] = scale * qbar_i . kbar_j for every pair
//      of blocks, fp32, as a 64 x 64 tiled SIMT product (4 x 4 outputs per
//      thread, both tiles staged k-major in shared memory); S goes to the route
//      workspace.
//   2. select_rows_kernel: one warp per (b, h, query block) row, the row staged
//      in shared memory: max-subtracted softmax (expf, fixed-order warp sums),
//      then the Top-p cut found without sorting: the largest value v* with
//      F(v*) = sum_{s_j >= v*} s_j >= p, located by bisection on the bit
//      pattern of non-negative floats (the computed F is monotone in v because
//      fp32 sums of non-negative terms are monotone in each term); ties at v*
//      are taken in block-index order until the sum reaches p. F only changes at
//      the row's values, so v* is one of them: the bisection also counts the
//      values at or above each bound and stops as soon as one distinct value is
//      left between them, which is then v*. If the Top-k floor is larger, the
//      k_min-th largest value is found the same way on counts. The selected
//      blocks are compacted in ascending index order with warp ballots, the
//      count is stored and added to the per-head work.
// Deterministic: every sum has a fixed order.
#include <cfloat>

#include "common.cuh"

namespace fvattn {

constexpr int kRouteThreads = 256;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// F(thr) = sum of s_j >= thr, same association order for every thr.
__device__ __forceinline__ float mass_at_least(const float* s, int nb, float thr, int lane) {
  float a = 0.f;
  for (int j = lane; j < nb; j += 32) {
    const float v = s[j];
    a += v >= thr ? v : 0.f;
  }
  return warp_sum(a);
}

__device__ __forceinline__ int count_at_least(const float* s, int nb, float thr, int lane) {
  unsigned c = 0u;
  for (int j = lane; j < nb; j += 32) c += s[j] >= thr ? 1u : 0u;
  return static_cast<int>(__reduce_add_sync(0xffffffffu, c));
}

// The only value of the row in [lo, hi) (the caller knows there is exactly one).
__device__ __forceinline__ uint32_t only_value_below(const float* s, int nb, uint32_t hi, int lane) {
  unsigned m = 0u;
  for (int j = lane; j < nb; j += 32) {
    const unsigned b = __float_as_uint(s[j]);
    if (b < hi) m = max(m, b);
  }
  return __reduce_max_sync(0xffffffffu, m);
}

// One importance row (already scaled logits in s[0..nb)), one warp.
// With softmax == false the row already holds importances (non-negative,
// summing to one over the evaluated blocks) and goes straight to selection.
__device__ void select_row(float* s, int nb, float p, int k_min, int* __restrict__ out_idx,
                           int* __restrict__ out_cnt, unsigned long long* head_work,
                           int* status, int lane, bool softmax) {
  if (softmax) {
    // softmax over the row, max subtracted
    float m = -FLT_MAX;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, s[j]);
    m = warp_max(m);
    float z = 0.f;
    for (int j = lane; j < nb; j += 32) {
      const float e = expf(s[j] - m);
      s[j] = e;
      z += e;
    }
    z = warp_sum(z);
    for (int j = lane; j < nb; j += 32) s[j] = s[j] / z;
  } else {
    // negative or non-finite importances are invalid input: clamped to 0, recorded
    bool bad = false;
    for (int j = lane; j < nb; j += 32) {
      const float v = s[j];
      if (!(v >= 0.f && v <= 1.f)) {
        s[j] = v > 1.f ? 1.f : 0.f;
        bad = true;
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
  }
  __syncwarp();

  int cnt;
  float thr;      // selected: s > thr, plus the first take_eq entries equal to thr
  int take_eq;
  if (p >= 1.f || k_min >= nb) {
    cnt = nb;
    thr = -1.f;
    take_eq = 0;
  } else {
    int n_p;
    float vstar = 0.f;
    int cgt = 0;
    const float total = mass_at_least(s, nb, 0.f, lane);
    if (total < p) {
      n_p = nb;
    } else {
      uint32_t lo = 0u, hi = 0x3F800001u;          // F(lo) >= p > F(hi)
      int c_lo = nb, c_hi = 0;                     // values at or above lo, hi
      while (hi - lo > 1u && c_lo - c_hi > 1) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const float fm = mass_at_least(s, nb, __uint_as_float(mid), lane);
        const int cm = count_at_least(s, nb, __uint_as_float(mid), lane);
        if (fm >= p) { lo = mid; c_lo = cm; } else { hi = mid; c_hi = cm; }
      }
      // One value left in [lo, hi): it is v*. (Otherwise lo and hi are adjacent
      // floats and v* = lo.)
      if (c_lo - c_hi == 1) lo = only_value_below(s, nb, hi, lane);
      vstar = __uint_as_float(lo);
      float sgt = 0.f;
      int ceq = 0;
      for (int j = lane; j < nb; j += 32) {
        const float v = s[j];
        if (v > vstar) { sgt += v; ++cgt; }
        ceq += v == vstar ? 1 : 0;
      }
      sgt = warp_sum(sgt);
      cgt = warp_sum_int(cgt);
      ceq = warp_sum_int(ceq);
      int need = 1;
      float acc = sgt + vstar;
      while (acc < p && need < ceq) { acc += vstar; ++need; }
      n_p = cgt + need;
    }
    cnt = min(nb, max(n_p, k_min));
    if (cnt == nb) {
      thr = -1.f;
      take_eq = 0;
    } else if (cnt == n_p) {
      thr = vstar;
      take_eq = cnt - cgt;
    } else {
      uint32_t lo = 0u, hi = 0x3F800001u;          // count(lo) >= cnt > count(hi)
      int c_lo = nb, c_hi = 0;
      while (hi - lo > 1u && c_lo - c_hi > 1) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const int cm = count_at_least(s, nb, __uint_as_float(mid), lane);
        if (cm >= cnt) { lo = mid; c_lo = cm; } else { hi = mid; c_hi = cm; }
      }
      if (c_lo - c_hi == 1) lo = only_value_below(s, nb, hi, lane);
      thr = __uint_as_float(lo);
      int gt = 0;
      for (int j = lane; j < nb; j += 32) gt += s[j] > thr ? 1 : 0;
      take_eq = cnt - warp_sum_int(gt);
    }
  }

  // compaction in ascending block index
  const unsigned lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
  for (int base = 0; base < nb; base += 32) {
    const int j = base + lane;
    const float v = j < nb ? s[j] : -2.f;
    const bool eq = v == thr;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eqb & lt_mask);
    const bool sel = v > thr || (eq && eq_rank < take_eq);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) out_idx[written + __popc(sb & lt_mask)] = j;
    written += __popc(sb);
    eq_seen += __popc(eqb);
  }
  if (lane == 0) {
    *out_cnt = cnt;
    atomicAdd(head_work, static_cast<unsigned long long>(cnt));
    if (written != cnt) record_status(status, FVATTN_ERR_INVALID_ARG);
  }
}

constexpr int kTile = 64;        // score tile: 64 query blocks x 64 key blocks
constexpr int kTilePad = kTile + 4;

// S tile = scale * Qtile . Ktile^T over d; 16 x 16 threads, 4 x 4 outputs each.
__global__ void __launch_bounds__(kRouteThreads)
    block_scores_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, int nb, int d,
                        float scale, float* __restrict__ S) {
  extern __shared__ float4 smem_f4[];
  float* qs = reinterpret_cast<float*>(smem_f4);   // [d][kTilePad], k-major
  float* ks = qs + d * kTilePad;                   // [d][kTilePad]
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
  const float* qb = qbar + static_cast<size_t>(bh) * nb * d;
  const float* kb = kbar + static_cast<size_t>(bh) * nb * d;
  const int d4 = d >> 2;
  // rows of the tile are the fastest index so that the transposing stores hit distinct banks
  for (int e = threadIdx.x; e < kTile * d4; e += kRouteThreads) {
    const int r = e % kTile, c = (e / kTile) * 4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (i0 + r < nb) a = *reinterpret_cast<const float4*>(qb + static_cast<size_t>(i0 + r) * d + c);
    if (j0 + r < nb) b = *reinterpret_cast<const float4*>(kb + static_cast<size_t>(j0 + r) * d + c);
    qs[(c + 0) * kTilePad + r] = a.x;
    qs[(c + 1) * kTilePad + r] = a.y;
    qs[(c + 2) * kTilePad + r] = a.z;
    qs[(c + 3) * kTilePad + r] = a.w;
    ks[(c + 0) * kTilePad + r] = b.x;
    ks[(c + 1) * kTilePad + r] = b.y;
    ks[(c + 2) * kTilePad + r] = b.z;
    ks[(c + 3) * kTilePad + r] = b.w;
  }
  __syncthreads();
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
  for (int kk = 0; kk < d; ++kk) {
    const float4 qa = *reinterpret_cast<const float4*>(qs + kk * kTilePad + ty * 4);
    const float4 kv = *reinterpret_cast<const float4*>(ks + kk * kTilePad + tx * 4);
    const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
    const float kf[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(qv[a], kf[c], acc[a][c]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty * 4 + a;
    if (i >= nb) break;
    float* row = S + (static_cast<size_t>(bh) * nb + i) * nb;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      if (j < nb) row[j] = acc[a][c] * scale;
    }
  }
}

// One warp per row of S: stage the row in shared memory, then select.
__global__ void __launch_bounds__(kRouteThreads)
    select_rows_kernel(const float* __restrict__ S, int rows, int nb, float p, int k_min,
                       int* __restrict__ kv_idx, int* __restrict__ kv_cnt,
                       unsigned long long* __restrict__ head_work, int* status, bool softmax) {
  extern __shared__ float4 smem_f4[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* srow = reinterpret_cast<float*>(smem_f4) + static_cast<size_t>(warp) * nb;
  const int r = blockIdx.x * (kRouteThreads / 32) + warp;
  if (r >= rows) return;
  const float* src = S + static_cast<size_t>(r) * nb;
  for (int j = lane; j < nb; j += 32) srow[j] = src[j];
  __syncwarp();
  const int bh = r / nb;
  select_row(srow, nb, p, k_min, kv_idx + static_cast<size_t>(r) * nb, kv_cnt + r, head_work + bh,
             status, lane, softmax);
}

size_t route_scores_bytes(int BH, int nb) {
  return static_cast<size_t>(BH) * nb * nb * sizeof(float);
}

cudaError_t launch_route_select(const float* qbar, const float* kbar, float* S, int BH, int nb, int d,
                                float scale, float p, int k_min, int* kv_idx, int* kv_cnt,
                                unsigned long long* head_work, int* status, cudaStream_t st) {
  const size_t smem1 = static_cast<size_t>(2) * d * kTilePad * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(block_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem1));
  if (e != cudaSuccess) return e;
  const dim3 g1((nb + kTile - 1) / kTile, (nb + kTile - 1) / kTile, BH);
  block_scores_kernel<<<g1, kRouteThreads, smem1, st>>>(qbar, kbar, nb, d, scale, S);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem2 = static_cast<size_t>(kRouteThreads / 32) * nb * sizeof(float);
  e = cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem2));
  if (e != cudaSuccess) return e;
  const int rows = BH * nb;
  const int warps = kRouteThreads / 32;
  select_rows_kernel<<<(rows + warps - 1) / warps, kRouteThreads, smem2, st>>>(
      S, rows, nb, p, k_min, kv_idx, kv_cnt, head_work, status, true);
  return cudaGetLastError();
}

// Top-p with the Top-k floor on given importance rows [BH, nb, nb] (no softmax).
cudaError_t launch_select_topp(const float* rows_in, int BH, int nb, float p, int k_min, int* kv_idx,
                               int* kv_cnt, unsigned long long* head_work, int* status,
                               cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kRouteThreads / 32) * nb * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int rows = BH * nb;
  const int warps = kRouteThreads / 32;
  select_rows_kernel<<<(rows + warps - 1) / warps, kRouteThreads, smem, st>>>(
      rows_in, rows, nb, p, k_min, kv_idx, kv_cnt, head_work, status, false);
  return cudaGetLastError();
}

}  // namespace fvattn
