// route.cu -- block scores, softmax and Top-p / Top-k-floor selection
// [FVAttn §2.1, §2.2 Eq. (1), §3.1; GSRS §5.2, §5.3, §A.4].
//
// One CTA owns ROWS = 8*RP query blocks of one (b, h):
//   1. scores S[r][j] = scale * qbar_r . kbar_j for every key block j, fp32, by
//      a register-tiled SIMT product (kbar streamed through shared memory in
//      chunks of 128 key blocks); the score rows stay in shared memory;
//   2. one warp per row: max-subtracted softmax (expf, fixed-order warp sums),
//      then the Top-p cut found without sorting: the largest value v* with
//      F(v*) = sum_{s_j >= v*} s_j >= p, located by bisection on the bit
//      pattern of non-negative floats (the computed F is monotone in v because
//      fp32 sums of non-negative terms are monotone in each term); ties at v*
//      are taken in block-index order until the sum reaches p. If the Top-k
//      floor is larger, the k_min-th largest value is found the same way on
//      counts. The selected blocks are compacted in ascending index order with
//      warp ballots, the count is stored and added to the per-head work.
// Deterministic: every sum has a fixed order.
#include <cfloat>

#include "common.cuh"

namespace fvattn {

constexpr int kRouteThreads = 256;
constexpr int kKeyChunk = 128;

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
  int c = 0;
  for (int j = lane; j < nb; j += 32) c += s[j] >= thr ? 1 : 0;
  return warp_sum_int(c);
}

// One importance row (already scaled logits in s[0..nb)), one warp.
__device__ void select_row(float* s, int nb, float p, int k_min, int* __restrict__ out_idx,
                           int* __restrict__ out_cnt, unsigned long long* head_work,
                           int* status, int lane) {
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
      while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (mass_at_least(s, nb, __uint_as_float(mid), lane) >= p) lo = mid; else hi = mid;
      }
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
      while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (count_at_least(s, nb, __uint_as_float(mid), lane) >= cnt) lo = mid; else hi = mid;
      }
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

template <int RP>
__global__ void __launch_bounds__(kRouteThreads)
    route_select_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, int nb,
                        int d, float scale, float p, int k_min, int* __restrict__ kv_idx,
                        int* __restrict__ kv_cnt, unsigned long long* __restrict__ head_work,
                        int* status) {
  constexpr int ROWS = 8 * RP;
  extern __shared__ float4 smem_f4[];
  float* sm = reinterpret_cast<float*>(smem_f4);
  const int ds = d + 4;
  float* qs = sm;                      // ROWS x ds
  float* ks = qs + ROWS * ds;          // kKeyChunk x ds
  float* S = ks + kKeyChunk * ds;      // ROWS x nb

  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * ROWS;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const float* qb = qbar + static_cast<size_t>(bh) * nb * d;
  const float* kb = kbar + static_cast<size_t>(bh) * nb * d;
  const int d4 = d >> 2;

  for (int e = tid; e < ROWS * d4; e += kRouteThreads) {
    const int r = e / d4, c = (e - r * d4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 + r < nb) v = *reinterpret_cast<const float4*>(qb + static_cast<size_t>(i0 + r) * d + c);
    *reinterpret_cast<float4*>(qs + r * ds + c) = v;
  }
  for (int j0 = 0; j0 < nb; j0 += kKeyChunk) {
    __syncthreads();
    for (int e = tid; e < kKeyChunk * d4; e += kRouteThreads) {
      const int r = e / d4, c = (e - r * d4) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + r < nb) v = *reinterpret_cast<const float4*>(kb + static_cast<size_t>(j0 + r) * d + c);
      *reinterpret_cast<float4*>(ks + r * ds + c) = v;
    }
    __syncthreads();
    float acc[RP][4];
#pragma unroll
    for (int a = 0; a < RP; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    for (int kk = 0; kk < d; kk += 4) {
      float4 kv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) kv[c] = *reinterpret_cast<const float4*>(ks + (lane + 32 * c) * ds + kk);
#pragma unroll
      for (int a = 0; a < RP; ++a) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (warp * RP + a) * ds + kk);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float t = acc[a][c];
          t = fmaf(qv.x, kv[c].x, t);
          t = fmaf(qv.y, kv[c].y, t);
          t = fmaf(qv.z, kv[c].z, t);
          t = fmaf(qv.w, kv[c].w, t);
          acc[a][c] = t;
        }
      }
    }
#pragma unroll
    for (int a = 0; a < RP; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = j0 + lane + 32 * c;
        if (j < nb) S[(warp * RP + a) * nb + j] = acc[a][c] * scale;
      }
  }
  __syncthreads();
  for (int a = 0; a < RP; ++a) {
    const int r = warp * RP + a;
    const int i = i0 + r;
    if (i >= nb) break;
    const size_t row = static_cast<size_t>(bh) * nb + i;
    select_row(S + r * nb, nb, p, k_min, kv_idx + row * nb, kv_cnt + row, head_work + bh,
               status, lane);
  }
}

size_t route_select_smem_bytes(int rp, int nb, int d) {
  return (static_cast<size_t>(8 * rp) * (d + 4) + static_cast<size_t>(kKeyChunk) * (d + 4) +
          static_cast<size_t>(8 * rp) * nb) * sizeof(float);
}

int route_select_rows_per_warp(int nb, int d) {
  constexpr size_t kBudget = 200 * 1024;
  for (int rp : {4, 2, 1})
    if (route_select_smem_bytes(rp, nb, d) <= kBudget) return rp;
  return 0;
}

cudaError_t launch_route_select(const float* qbar, const float* kbar, int BH, int nb, int d,
                                float scale, float p, int k_min, int* kv_idx, int* kv_cnt,
                                unsigned long long* head_work, int* status, cudaStream_t st) {
  const int rp = route_select_rows_per_warp(nb, d);
  if (rp == 0) return cudaErrorInvalidValue;
  const size_t smem = route_select_smem_bytes(rp, nb, d);
  const dim3 grid((nb + 8 * rp - 1) / (8 * rp), BH);
  cudaError_t e;
  switch (rp) {
    case 4:
      e = cudaFuncSetAttribute(route_select_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      route_select_kernel<4><<<grid, kRouteThreads, smem, st>>>(qbar, kbar, nb, d, scale, p, k_min, kv_idx, kv_cnt, head_work, status);
      break;
    case 2:
      e = cudaFuncSetAttribute(route_select_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      route_select_kernel<2><<<grid, kRouteThreads, smem, st>>>(qbar, kbar, nb, d, scale, p, k_min, kv_idx, kv_cnt, head_work, status);
      break;
    default:
      e = cudaFuncSetAttribute(route_select_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      route_select_kernel<1><<<grid, kRouteThreads, smem, st>>>(qbar, kbar, nb, d, scale, p, k_min, kv_idx, kv_cnt, head_work, status);
      break;
  }
  return cudaGetLastError();
}

}  // namespace fvattn
