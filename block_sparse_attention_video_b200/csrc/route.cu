// route.cu -- block scores, softmax and Top-p / Top-k-floor selection
// [FVAttn §2.1, §2.2 Eq. (1), §3.1; GSRS §5.2, §5.3, §A.4].
//
// Two kernels:
//   1. block_scores_tc_kernel (scores_tc.cu): S[b,h,i,j] = scale * qbar_i . kbar_j
//      for every pair of blocks on the tensor cores, with fp32-level accuracy
//      from a split of each operand into two TF32 parts; S goes to the route
//      workspace with its row stride padded to a multiple of 4 floats.
//   2. select_rows_kernel: one warp per (b, h, query block) row, the row held in
//      registers (32 per lane and up to 48 values per lane; longer rows are staged
//      in shared memory): max-subtracted softmax (the scores arrive as base-2
//      logits, so exp2f; fixed-order warp sums),
//      then the Top-p cut found without sorting: the largest value v* with
//      F(v*) = sum_{s_j >= v*} s_j >= p. F is evaluated with each lane's fp32
//      partial sum (fixed order) rounded to a 2^-31 fixed point and added
//      exactly with one integer warp reduction, so the computed F is monotone in
//      v and deterministic. v* is located by a search on the bit pattern of
//      non-negative floats between the row's smallest and largest value, that
//      alternates interpolation on F with plain bisection (the interpolation
//      usually lands near the cut, the bisection bounds the worst case); each
//      step also counts the values at or above the probe and the search stops as
//      soon as one distinct value is left in the bracket, which is then v*. Ties
//      at v* are taken in block-index order until the sum reaches p. If the Top-k
//      floor is larger, the k_min-th largest value is found the same way on
//      counts. The selected blocks are compacted in ascending index order with
//      warp ballots, the count is stored and added to the per-head work.
// Deterministic: every sum has a fixed order or is an exact integer sum.
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

constexpr float kFix = 2147483648.0f;   // 2^31: masses in [0, 1] as 2^-31 fixed point

// Fixed-point mass of one lane's fp32 partial sum (at most 1 + rounding).
__device__ __forceinline__ uint32_t to_fix(float a) { return __float2uint_rn(a * kFix); }

// Probe of the search: interpolation of F between the bracket's ends on odd
// steps, bisection of the bit range on even steps; always strictly inside
// (lo, hi). lo, hi are bit patterns of non-negative floats, hi - lo > 1.
__device__ __forceinline__ uint32_t probe(uint32_t lo, uint32_t hi, uint32_t f_lo, uint32_t f_hi,
                                          uint32_t target, int step) {
  uint32_t mid = lo + ((hi - lo) >> 1);
  if ((step & 1) && f_lo > f_hi) {
    const float vl = __uint_as_float(lo), vh = __uint_as_float(hi);
    const float t = static_cast<float>(f_lo - target) / static_cast<float>(f_lo - f_hi);
    const uint32_t m = __float_as_uint(fmaf(vh - vl, t, vl));
    mid = min(max(m, lo + 1u), hi - 1u);
  }
  return mid;
}

// One row of up to 32 * VPL values held in registers, value t of a lane being
// element t * 32 + lane. Elements past nb hold -1 (never selected: every
// threshold is a non-negative float).
template <int VPL>
__device__ void select_row_reg(const float* __restrict__ src, int nb, float p, int k_min,
                               int* __restrict__ out_idx, int* __restrict__ out_cnt,
                               unsigned long long* head_work, int* status, int lane, bool softmax) {
  float v[VPL];
#pragma unroll
  for (int t = 0; t < VPL; ++t) {
    const int j = t * 32 + lane;
    v[t] = j < nb ? src[j] : -INFINITY;
  }
  if (softmax) {
    // softmax over the row, max subtracted; pads (-inf) give 0 and are then set to -1
    float m = -FLT_MAX;
#pragma unroll
    for (int t = 0; t < VPL; ++t) m = fmaxf(m, v[t]);
    m = warp_max(m);
    float z = 0.f;
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      v[t] = exp2f(v[t] - m);   // the row holds base-2 logits: 2^(x log2 e) = e^x
      z += v[t];
    }
    z = warp_sum(z);
    const float rz = 1.0f / z;
#pragma unroll
    for (int t = 0; t < VPL; ++t) v[t] = t * 32 + lane < nb ? v[t] * rz : -1.f;
  } else {
    // negative or non-finite importances are invalid input: clamped to 0, recorded
    bool bad = false;
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      if (t * 32 + lane >= nb) {
        v[t] = -1.f;
      } else if (!(v[t] >= 0.f && v[t] <= 1.f)) {
        v[t] = v[t] > 1.f ? 1.f : 0.f;
        bad = true;
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
  }

  // F(x) in fixed point and the number of values >= x, one pass over the row
  auto mass_count = [&](float x, uint32_t& F, int& C) {
    float a = 0.f;
    unsigned c = 0u;
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      const bool ge = v[t] >= x;
      a += ge ? v[t] : 0.f;
      c += ge ? 1u : 0u;
    }
    F = __reduce_add_sync(0xffffffffu, to_fix(a));
    C = static_cast<int>(__reduce_add_sync(0xffffffffu, c));
  };
  auto count_ge = [&](float x) -> int {
    unsigned c = 0u;
#pragma unroll
    for (int t = 0; t < VPL; ++t) c += v[t] >= x ? 1u : 0u;
    return static_cast<int>(__reduce_add_sync(0xffffffffu, c));
  };
  // the only value in [lo, hi) when the caller knows there is exactly one (pads,
  // negative, compare above every bit pattern of a non-negative float)
  auto only_below = [&](uint32_t hi) -> uint32_t {
    unsigned m = 0u;
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      const unsigned bits = __float_as_uint(v[t]);
      if (bits < hi) m = max(m, bits);
    }
    return __reduce_max_sync(0xffffffffu, m);
  };
  // bracket of the valid values: smallest and largest (as bit patterns)
  unsigned vmin = 0x7F800000u, vmax = 0u;
#pragma unroll
  for (int t = 0; t < VPL; ++t) {
    if (v[t] >= 0.f) {
      vmin = min(vmin, __float_as_uint(v[t]));
      vmax = max(vmax, __float_as_uint(v[t]));
    }
  }
  vmin = __reduce_min_sync(0xffffffffu, vmin);
  vmax = __reduce_max_sync(0xffffffffu, vmax);

  int cnt;
  float thr;      // selected: v > thr, plus the first take_eq entries equal to thr
  int take_eq;
  bool tie_split = false;   // some, not all, of the entries equal to thr are taken
  if (p >= 1.f || k_min >= nb) {
    cnt = nb;
    thr = -1.f;
    take_eq = 0;
  } else {
    int n_p;
    float vstar = 0.f;
    int cgt = 0;
    int ceq_star = 1;
    const uint32_t target = to_fix(p);
    uint32_t total;
    int call;
    mass_count(0.f, total, call);
    if (total < target) {
      n_p = nb;
    } else {
      uint32_t lo = vmin, hi = vmax + 1u;          // F(lo) >= target > F(hi)
      uint32_t f_lo = total, f_hi = 0u;
      int c_lo = nb, c_hi = 0;                     // values at or above lo, hi
      for (int step = 1; hi - lo > 1u && c_lo - c_hi > 1; ++step) {
        const uint32_t mid = probe(lo, hi, f_lo, f_hi, target, step);
        uint32_t fm;
        int cm;
        mass_count(__uint_as_float(mid), fm, cm);
        if (fm >= target) { lo = mid; f_lo = fm; c_lo = cm; } else { hi = mid; f_hi = fm; c_hi = cm; }
      }
      // F(lo) > F(hi), so [lo, hi) holds at least one value. Either exactly one
      // is left, which is v*, or lo and hi are adjacent floats and every value
      // in the bracket equals lo = v*. Either way the values above v* are those
      // at or above hi: their mass and count are f_hi and c_hi, and the
      // c_lo - c_hi values equal to v* are taken in index order until p is reached.
      if (c_lo - c_hi == 1) lo = only_below(hi);
      vstar = __uint_as_float(lo);
      cgt = c_hi;
      const int ceq = c_lo - c_hi;
      ceq_star = ceq;
      const uint32_t fstar = to_fix(vstar);
      int need = 1;
      uint32_t acc = f_hi + fstar;
      while (acc < target && need < ceq) { acc += fstar; ++need; }
      n_p = cgt + need;
    }
    cnt = min(nb, max(n_p, k_min));
    if (cnt == nb) {
      thr = -1.f;
      take_eq = 0;
    } else if (cnt == n_p) {
      thr = vstar;
      take_eq = cnt - cgt;
      tie_split = take_eq < ceq_star;
    } else {
      uint32_t lo = vmin, hi = vmax + 1u;          // count(lo) >= cnt > count(hi)
      int c_lo = nb, c_hi = 0;
      while (hi - lo > 1u && c_lo - c_hi > 1) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const int cm = count_ge(__uint_as_float(mid));
        if (cm >= cnt) { lo = mid; c_lo = cm; } else { hi = mid; c_hi = cm; }
      }
      // as above: the values above the threshold are the c_hi at or above hi
      if (c_lo - c_hi == 1) lo = only_below(hi);
      thr = __uint_as_float(lo);
      take_eq = cnt - c_hi;
      tie_split = take_eq < c_lo - c_hi;
    }
  }

  // compaction in ascending block index (cnt and tie_split are warp-uniform)
  const unsigned lt_mask = (1u << lane) - 1u;
  int written = 0;
  if (cnt == nb) {
    // every block: the list is 0 .. nb-1
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      const int j = t * 32 + lane;
      if (j < nb) out_idx[j] = j;
    }
    written = nb;
  } else if (!tie_split) {
    // every entry equal to thr is taken: the selection is v >= thr (pads, -1, are below)
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      const bool sel = v[t] >= thr;
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      if (sel) out_idx[written + __popc(sb & lt_mask)] = t * 32 + lane;
      written += __popc(sb);
    }
  } else {
    int eq_seen = 0;
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
      const int j = t * 32 + lane;
      const bool valid = j < nb;
      const bool eq = valid && v[t] == thr;
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      const int eq_rank = eq_seen + __popc(eqb & lt_mask);
      const bool sel = valid && (v[t] > thr || (eq && eq_rank < take_eq));
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      if (sel) out_idx[written + __popc(sb & lt_mask)] = j;
      written += __popc(sb);
      eq_seen += __popc(eqb);
    }
  }
  if (lane == 0) {
    *out_cnt = cnt;
    atomicAdd(head_work, static_cast<unsigned long long>(cnt));
    if (written != cnt) record_status(status, FVATTN_ERR_INVALID_ARG);
  }
}

// Row stride of the block score matrix: nb padded to a multiple of 4 floats.
__host__ __device__ __forceinline__ int scores_ld(int nb) { return (nb + 3) & ~3; }

cudaError_t launch_block_scores_tc(const float* qbar, const float* kbar, int BH, int nb, int d, float scale,
                                   int ld, float* S, int* status, cudaStream_t st);

// One warp per row of the score (or importance) matrix, read with row stride ld.
template <int VPL>
__global__ void __launch_bounds__(kRouteThreads)
    select_rows_kernel(const float* __restrict__ S, int ld, int rows, int nb, float p, int k_min,
                       int* __restrict__ kv_idx, int* __restrict__ kv_cnt,
                       unsigned long long* __restrict__ head_work, int* status, bool softmax) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (kRouteThreads / 32) + warp;
  if (r >= rows) return;
  const int bh = r / nb;
  select_row_reg<VPL>(S + static_cast<size_t>(r) * ld, nb, p, k_min, kv_idx + static_cast<size_t>(r) * nb,
                      kv_cnt + r, head_work + bh, status, lane, softmax);
}

static cudaError_t launch_select(const float* S, int ld, int BH, int nb, float p, int k_min, int* kv_idx,
                                 int* kv_cnt, unsigned long long* head_work, int* status, bool softmax,
                                 cudaStream_t st) {
  const int rows = BH * nb;
  const int warps = kRouteThreads / 32;
  const dim3 grid((rows + warps - 1) / warps);
  const int vpl = (nb + 31) / 32;
#define FVATTN_SELECT(V)                                                                         \
  select_rows_kernel<V><<<grid, kRouteThreads, 0, st>>>(S, ld, rows, nb, p, k_min, kv_idx, kv_cnt, \
                                                        head_work, status, softmax)
  if (vpl <= 4) FVATTN_SELECT(4);
  else if (vpl <= 8) FVATTN_SELECT(8);
  else if (vpl <= 12) FVATTN_SELECT(12);
  else if (vpl <= 16) FVATTN_SELECT(16);
  else if (vpl <= 20) FVATTN_SELECT(20);
  else if (vpl <= 24) FVATTN_SELECT(24);
  else if (vpl <= 32) FVATTN_SELECT(32);
  else if (vpl <= 40) FVATTN_SELECT(40);
  else if (vpl <= 48) FVATTN_SELECT(48);
  else if (vpl <= 64) FVATTN_SELECT(64);
  else FVATTN_SELECT(128);
#undef FVATTN_SELECT
  return cudaGetLastError();
}

size_t route_scores_bytes(int BH, int nb) {
  return static_cast<size_t>(BH) * nb * scores_ld(nb) * sizeof(float);
}

cudaError_t launch_route_select(const float* qbar, const float* kbar, float* S, int BH, int nb, int d,
                                float scale, float p, int k_min, int* kv_idx, int* kv_cnt,
                                unsigned long long* head_work, int* status, cudaStream_t st) {
  // base-2 logits: the selection's softmax then takes exp2f
  cudaError_t e = launch_block_scores_tc(qbar, kbar, BH, nb, d, scale * 1.4426950408889634f, scores_ld(nb), S,
                                         status, st);
  if (e != cudaSuccess) return e;
  return launch_select(S, scores_ld(nb), BH, nb, p, k_min, kv_idx, kv_cnt, head_work, status, true, st);
}

// Top-p with the Top-k floor on given importance rows [BH, nb, nb] (no softmax).
cudaError_t launch_select_topp(const float* rows_in, int BH, int nb, float p, int k_min, int* kv_idx,
                               int* kv_cnt, unsigned long long* head_work, int* status,
                               cudaStream_t st) {
  return launch_select(rows_in, nb, BH, nb, p, k_min, kv_idx, kv_cnt, head_work, status, false, st);
}

}  // namespace fvattn

namespace fvattn {

// Descending order of (score, then lower block index) as one 64-bit key: the
// float bits mapped to an unsigned order (negatives flipped), then the
// complemented index.
__device__ __forceinline__ unsigned long long importance_key(float s, int j) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(o) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - j);
}

// One CTA per row: the row's cnt selected blocks sorted by descending score
// (bitonic network in shared memory over the next power of two), written back
// over the first cnt entries of the list.
__global__ void __launch_bounds__(kRouteThreads)
    order_lists_kernel(const float* __restrict__ S, int ld, int nb, int* __restrict__ kv_idx,
                       const int* __restrict__ kv_cnt, int* status) {
  extern __shared__ unsigned long long okeys[];
  const int r = blockIdx.x;
  const float* srow = S + static_cast<size_t>(r) * ld;
  int* lst = kv_idx + static_cast<size_t>(r) * nb;
  int cnt = kv_cnt[r];
  if (cnt < 1 || cnt > nb) {
    if (threadIdx.x == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
    cnt = min(max(cnt, 1), nb);
  }
  int n2 = 1;
  while (n2 < cnt) n2 <<= 1;
  for (int t = threadIdx.x; t < n2; t += blockDim.x) {
    unsigned long long key = 0ull;     // pads sort last
    if (t < cnt) {
      int j = lst[t];
      if (j < 0 || j >= nb) {
        record_status(status, FVATTN_ERR_INVALID_ARG);
        j = min(max(j, 0), nb - 1);
      }
      key = importance_key(srow[j], j);
    }
    okeys[t] = key;
  }
  for (int size = 2; size <= n2; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < n2 / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = okeys[lo], y = okeys[hi];
        if ((x < y) == desc) { okeys[lo] = y; okeys[hi] = x; }
      }
    }
  __syncthreads();
  for (int t = threadIdx.x; t < cnt; t += blockDim.x)
    lst[t] = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(okeys[t] & 0xFFFFFFFFull));
}

cudaError_t launch_order_lists(const float* S, int BH, int nb, int* kv_idx, const int* kv_cnt, int* status,
                               cudaStream_t st) {
  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  const size_t smem = static_cast<size_t>(n2) * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(order_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  order_lists_kernel<<<BH * nb, kRouteThreads, smem, st>>>(S, scores_ld(nb), nb, kv_idx, kv_cnt, status);
  return cudaGetLastError();
}

}  // namespace fvattn
