// permute.cu -- block-order permutation of token rows (3-D tiles, or an explicit
// table such as the Hilbert order) [FVAttn §3.1] and the fused
// gather + block-mean pooling pass of the routing front end [FVAttn §3.1:
// block similarity from pooled Q/K].
//
// One CTA moves one block of `bs` consecutive rows of the permuted sequence of
// one (b, h). Rows are copied as 16-byte vectors; each thread keeps up to 8
// independent 16-byte loads in flight before storing. HBM-bound: one read and
// one write of every row.
#include "common.cuh"

namespace fvattn {

constexpr int kCopyThreads = 256;
constexpr int kMaxInflight = 8;

// VPR = 16-byte vectors per token row (row bytes / 16): 8, 16 or 32.
template <int VPR>
__global__ void __launch_bounds__(kCopyThreads)
    permute_rows_kernel(const uint4* __restrict__ x, uint4* __restrict__ y, int nb, int bs, int N,
                        TileGeom g, int inverse) {
  __shared__ int src[256];
  const int bh = blockIdx.x / nb;
  const int i = blockIdx.x - bh * nb;
  for (int r = threadIdx.x; r < bs; r += blockDim.x) {
    const int pos = i * bs + r;
    src[r] = pos < N ? source_index(pos, N, g) : -1;
  }
  __syncthreads();
  const size_t orig_base = static_cast<size_t>(bh) * N;
  const size_t perm_base = static_cast<size_t>(bh) * nb * bs + static_cast<size_t>(i) * bs;
  constexpr int kRowsPerPass = kCopyThreads / VPR;
  const int c = threadIdx.x % VPR;
  const int r0 = threadIdx.x / VPR;
  for (int rb = 0; rb < bs; rb += kRowsPerPass * kMaxInflight) {
    uint4 v[kMaxInflight];
#pragma unroll
    for (int k = 0; k < kMaxInflight; ++k) {
      const int r = rb + r0 + k * kRowsPerPass;
      v[k] = make_uint4(0u, 0u, 0u, 0u);
      if (r < bs) {
        const int s = src[r];
        if (s >= 0) v[k] = inverse ? x[(perm_base + r) * VPR + c] : x[(orig_base + s) * VPR + c];
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxInflight; ++k) {
      const int r = rb + r0 + k * kRowsPerPass;
      if (r < bs) {
        const int s = src[r];
        if (!inverse)
          y[(perm_base + r) * VPR + c] = v[k];
        else if (s >= 0)
          y[(orig_base + s) * VPR + c] = v[k];
      }
    }
  }
}

template <typename T>
__device__ __forceinline__ void accumulate_vec(const uint4& v, float* acc);

template <>
__device__ __forceinline__ void accumulate_vec<__nv_bfloat16>(const uint4& v, float* acc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] += __uint_as_float(w[e] << 16);
    acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void accumulate_vec<float>(const uint4& v, float* acc) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}

// blockIdx.y selects the tensor (0 = q, 1 = k). Writes the permuted rows (when
// the output pointer is not null) and the fp32 mean of the block's valid rows.
template <typename T, int VPR>
__global__ void __launch_bounds__(kCopyThreads)
    gather_pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                       uint4* __restrict__ qp, uint4* __restrict__ kp, float* __restrict__ qbar,
                       float* __restrict__ kbar, int nb, int bs, int N, TileGeom g) {
  constexpr int EPV = 16 / sizeof(T);            // elements per 16-byte vector
  constexpr int D = VPR * EPV;                    // head dim
  constexpr int kRowsPerPass = kCopyThreads / VPR;
  __shared__ int src[256];
  __shared__ float red[kRowsPerPass][D];

  const uint4* x = blockIdx.y == 0 ? q : k;
  uint4* y = blockIdx.y == 0 ? qp : kp;
  float* bar = blockIdx.y == 0 ? qbar : kbar;

  const int bh = blockIdx.x / nb;
  const int i = blockIdx.x - bh * nb;
  for (int r = threadIdx.x; r < bs; r += blockDim.x) {
    const int pos = i * bs + r;
    src[r] = pos < N ? source_index(pos, N, g) : -1;
  }
  __syncthreads();
  const size_t orig_base = static_cast<size_t>(bh) * N;
  const size_t perm_base = static_cast<size_t>(bh) * nb * bs + static_cast<size_t>(i) * bs;
  const int c = threadIdx.x % VPR;
  const int r0 = threadIdx.x / VPR;
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;

  for (int rb = 0; rb < bs; rb += kRowsPerPass * kMaxInflight) {
    uint4 v[kMaxInflight];
#pragma unroll
    for (int kk = 0; kk < kMaxInflight; ++kk) {
      const int r = rb + r0 + kk * kRowsPerPass;
      v[kk] = make_uint4(0u, 0u, 0u, 0u);
      if (r < bs && src[r] >= 0) v[kk] = x[(orig_base + src[r]) * VPR + c];
    }
#pragma unroll
    for (int kk = 0; kk < kMaxInflight; ++kk) {
      const int r = rb + r0 + kk * kRowsPerPass;
      if (r < bs) {
        if (y) y[(perm_base + r) * VPR + c] = v[kk];
        if (src[r] >= 0) accumulate_vec<T>(v[kk], acc);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPV; ++e) red[r0][c * EPV + e] = acc[e];
  __syncthreads();
  const int nvalid = min(bs, N - i * bs);
  for (int col = threadIdx.x; col < D; col += blockDim.x) {
    float s = 0.f;
#pragma unroll 4
    for (int r = 0; r < kRowsPerPass; ++r) s += red[r][col];
    bar[(static_cast<size_t>(bh) * nb + i) * D + col] = s / static_cast<float>(nvalid);
  }
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_permute(const void* x, void* y, int BH, int N, int d, int esize, int bs,
                           const TileGeom& g, int inverse, cudaStream_t st) {
  const int nb = (N + bs - 1) / bs;
  const int vpr = d * esize / 16;
  const dim3 grid(static_cast<unsigned>(BH) * nb);
  auto xs = static_cast<const uint4*>(x);
  auto ys = static_cast<uint4*>(y);
  switch (vpr) {
    case 8: permute_rows_kernel<8><<<grid, kCopyThreads, 0, st>>>(xs, ys, nb, bs, N, g, inverse); break;
    case 16: permute_rows_kernel<16><<<grid, kCopyThreads, 0, st>>>(xs, ys, nb, bs, N, g, inverse); break;
    case 32: permute_rows_kernel<32><<<grid, kCopyThreads, 0, st>>>(xs, ys, nb, bs, N, g, inverse); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_pool(const void* q, const void* k, void* qp, void* kp, float* qbar,
                               float* kbar, int BH, int N, int d, bool bf16, int bs,
                               const TileGeom& g, cudaStream_t st) {
  const int nb = (N + bs - 1) / bs;
  const dim3 grid(static_cast<unsigned>(BH) * nb, 2);
  auto qs = static_cast<const uint4*>(q);
  auto ks = static_cast<const uint4*>(k);
  auto qo = static_cast<uint4*>(qp);
  auto ko = static_cast<uint4*>(kp);
  if (bf16 && d == 128)
    gather_pool_kernel<__nv_bfloat16, 16><<<grid, kCopyThreads, 0, st>>>(qs, ks, qo, ko, qbar, kbar, nb, bs, N, g);
  else if (bf16 && d == 64)
    gather_pool_kernel<__nv_bfloat16, 8><<<grid, kCopyThreads, 0, st>>>(qs, ks, qo, ko, qbar, kbar, nb, bs, N, g);
  else if (!bf16 && d == 128)
    gather_pool_kernel<float, 32><<<grid, kCopyThreads, 0, st>>>(qs, ks, qo, ko, qbar, kbar, nb, bs, N, g);
  else if (!bf16 && d == 64)
    gather_pool_kernel<float, 16><<<grid, kCopyThreads, 0, st>>>(qs, ks, qo, ko, qbar, kbar, nb, bs, N, g);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace fvattn
