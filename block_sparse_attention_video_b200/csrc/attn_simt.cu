// attn_simt.cu -- block-sparse softmax attention on the CUDA cores, fp32
// arithmetic throughout [FVAttn §2.1: only selected (query block, key block)
// pairs are evaluated; GSRS §A.1: online softmax over key blocks].
//
// Serves FP32 tensors and the shapes the tensor-core kernel does not cover
// (d = 64 or 64-token blocks). One CTA per (b, h, query block, 32-column slice
// of the output); one thread per query row keeps its q row in shared memory,
// a running max m, a running sum l and 32 output accumulators, and updates them
// exactly for every valid key of every selected block:
//   m' = max(m, s),  l' = l*exp(m-m') + exp(s-m'),  o' = o*exp(m-m') + exp(s-m')*v.
// When block_lse is requested, the CTAs of the first output slice also keep a
// per-block max and sum and store each selected block's log-sum-exp
// [GSRS §5.3: per-block statistics recorded during the attention pass].
#include "common.cuh"

namespace fvattn {

constexpr int kSlice = 32;

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ T store_cast(float v);
template <>
__device__ __forceinline__ float store_cast<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 store_cast<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(BS)
    attn_simt_kernel(const T* __restrict__ qp, const T* __restrict__ kp, const T* __restrict__ vp,
                     T* __restrict__ op, float* __restrict__ lse, float* __restrict__ blse,
                     const int* __restrict__ kv_idx,
                     const int* __restrict__ kv_cnt, int nb, int N, float scale, int* status) {
  extern __shared__ float4 smem_f4[];
  float* Qs = reinterpret_cast<float*>(smem_f4);   // BS x (D+1)
  float* Ks = Qs + BS * (D + 1);                    // BS x (D+1)
  float* Vs = Ks + BS * (D + 1);                    // BS x (kSlice+1)

  const int bh = blockIdx.x / nb;
  const int i = blockIdx.x - bh * nb;
  const int d0 = blockIdx.y * kSlice;
  const int row = threadIdx.x;
  const size_t npad = static_cast<size_t>(nb) * BS;
  const size_t head = static_cast<size_t>(bh) * npad;

  for (int e = threadIdx.x; e < BS * D; e += BS) {
    const int r = e / D, c = e - r * D;
    Qs[r * (D + 1) + c] = load_elem<T>(qp + (head + static_cast<size_t>(i) * BS + r) * D + c);
  }
  int cnt = nb;
  const int* list = nullptr;
  if (kv_idx) {
    cnt = kv_cnt[static_cast<size_t>(bh) * nb + i];
    if (cnt < 1 || cnt > nb) {
      if (threadIdx.x == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
      cnt = min(max(cnt, 1), nb);
    }
    list = kv_idx + (static_cast<size_t>(bh) * nb + i) * nb;
  }

  const bool want_blse = blse != nullptr && blockIdx.y == 0;
  float m = -INFINITY, l = 0.f;
  float acc[kSlice];
#pragma unroll
  for (int e = 0; e < kSlice; ++e) acc[e] = 0.f;

  for (int t = 0; t < cnt; ++t) {
    int j = list ? list[t] : t;
    if (j < 0 || j >= nb) {
      if (threadIdx.x == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
      j = 0;
    }
    const int valid = min(BS, N - j * BS);
    __syncthreads();
    for (int e = threadIdx.x; e < BS * D; e += BS) {
      const int r = e / D, c = e - r * D;
      Ks[r * (D + 1) + c] = load_elem<T>(kp + (head + static_cast<size_t>(j) * BS + r) * D + c);
    }
    for (int e = threadIdx.x; e < BS * kSlice; e += BS) {
      const int r = e / kSlice, c = e - r * kSlice;
      Vs[r * (kSlice + 1) + c] = load_elem<T>(vp + (head + static_cast<size_t>(j) * BS + r) * D + d0 + c);
    }
    __syncthreads();
    float bm = -INFINITY, bl = 0.f;
    for (int c = 0; c < valid; ++c) {
      float s = 0.f;
#pragma unroll 8
      for (int kk = 0; kk < D; ++kk) s = fmaf(Qs[row * (D + 1) + kk], Ks[c * (D + 1) + kk], s);
      s *= scale;
      if (want_blse) {
        if (s > bm) {
          bl = bl * expf(bm - s) + 1.f;
          bm = s;
        } else {
          bl += expf(s - bm);
        }
      }
      if (s > m) {
        const float corr = expf(m - s);
        l = l * corr + 1.f;
#pragma unroll
        for (int e = 0; e < kSlice; ++e) acc[e] = fmaf(acc[e], corr, Vs[c * (kSlice + 1) + e]);
        m = s;
      } else {
        const float w = expf(s - m);
        l += w;
#pragma unroll
        for (int e = 0; e < kSlice; ++e) acc[e] = fmaf(w, Vs[c * (kSlice + 1) + e], acc[e]);
      }
    }
    if (want_blse) blse[(static_cast<size_t>(bh) * nb + j) * npad + static_cast<size_t>(i) * BS + row] = bm + logf(bl);
  }
  const float inv = 1.f / l;
  T* orow = op + (head + static_cast<size_t>(i) * BS + row) * D + d0;
#pragma unroll
  for (int e = 0; e < kSlice; ++e) orow[e] = store_cast<T>(acc[e] * inv);
  if (lse && blockIdx.y == 0) lse[head + static_cast<size_t>(i) * BS + row] = m + logf(l);
}

template <typename T, int D, int BS>
static cudaError_t launch_simt_t(const void* q, const void* k, const void* v, void* o, float* lse,
                                 float* blse, const int* kv_idx, const int* kv_cnt, int BH, int nb, int N,
                                 float scale, int* status, cudaStream_t st) {
  const size_t smem = (static_cast<size_t>(BS) * (D + 1) * 2 + static_cast<size_t>(BS) * (kSlice + 1)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D, BS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(BH) * nb, D / kSlice);
  attn_simt_kernel<T, D, BS><<<grid, BS, smem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(o),
      lse, blse, kv_idx, kv_cnt, nb, N, scale, status);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, void* o, float* lse,
                             float* blse, const int* kv_idx, const int* kv_cnt, int BH, int N, int d, int bs,
                             bool bf16, float scale, int* status, cudaStream_t st) {
  const int nb = (N + bs - 1) / bs;
#define FVATTN_SIMT_CASE(T, D_, BS_)                                                         \
  if (d == D_ && bs == BS_)                                                                  \
    return launch_simt_t<T, D_, BS_>(q, k, v, o, lse, blse, kv_idx, kv_cnt, BH, nb, N, scale, status, st);
  if (bf16) {
    FVATTN_SIMT_CASE(__nv_bfloat16, 64, 64)
    FVATTN_SIMT_CASE(__nv_bfloat16, 64, 128)
    FVATTN_SIMT_CASE(__nv_bfloat16, 128, 64)
    FVATTN_SIMT_CASE(__nv_bfloat16, 128, 128)
  } else {
    FVATTN_SIMT_CASE(float, 64, 64)
    FVATTN_SIMT_CASE(float, 64, 128)
    FVATTN_SIMT_CASE(float, 128, 64)
    FVATTN_SIMT_CASE(float, 128, 128)
  }
#undef FVATTN_SIMT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fvattn
