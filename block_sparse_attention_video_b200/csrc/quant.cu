// quant.cu -- per-channel FP8 E4M3 quantization of the permuted V, the input
// of the tensor-core attention kernel's 8-bit P.V product.
//
// [FVAttn §3.4]  the GPU quantizes V in a step of its own before attention.
// Reading (the pages name no format): E4M3 codes with one fp32 scale per
// (batch, head, channel), scale_c = amax_c / 448 over the head's valid tokens,
// code = RN-even_e4m3(fp32(v * fp32(448 / amax_c))) saturating at +-448, so the
// largest magnitude of each channel encodes as +-448. A channel with
// amax < 2^-100 gets codes 0 and scale 0. Pad rows (>= N) are written as 0.
// Both fp32 operations use the IEEE round-to-nearest intrinsics, so every code
// is decided exactly.
//
// Layout: V [B*H, Npad, 128] bf16 -> codes [B*H, Npad, 128] u8 (one 128-byte row
// per token, the layout the attention kernel's TMA reads) and scales
// [B*H, 128] fp32.
//
// Two passes, both HBM-bound: (1) the channel maxima, a CTA per (head, slab of
// rows) with 16 threads per row (8 channels = 16 bytes each) reduced in shared
// memory and merged with an integer atomicMax on the float bits (exact for
// values >= 0); (2) the encoding, same thread mapping, 8 bytes stored per
// thread. Both read V rows as 16-byte vectors, so a warp covers two full rows.
//
// Fused with the block-order permutation (launch_permute_quantize_v): the
// maxima do not depend on the token order, so pass (1) reads V in raster order,
// and pass (2) gathers each block's rows from raster order (as the permutation
// does) and encodes them, so V is read twice and the codes written once; the
// permuted bf16 V is never formed. Its codes and scales equal those of the
// permutation followed by the quantization, bit for bit.
#include "common.cuh"

namespace fvattn {

constexpr int kQuantThreads = 256;
constexpr int kQuantRows = 512;       // rows per CTA
constexpr int kQuantD = 128;
constexpr float kE4M3Max = 448.0f;
constexpr float kAmaxZero = 0x1p-100f;

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kQuantThreads)
    vquant_amax_kernel(const uint4* __restrict__ v, int N, int npad,
                       unsigned int* __restrict__ amax_bits) {
  __shared__ float part[kQuantThreads / 16][kQuantD];
  const int bh = blockIdx.y;
  const int cg = threadIdx.x & 15;          // channels 8*cg .. 8*cg+7
  const int r0 = threadIdx.x >> 4;
  const int lo = blockIdx.x * kQuantRows;
  const int hi = min(N, lo + kQuantRows);
  const uint4* base = v + static_cast<size_t>(bh) * npad * (kQuantD / 8);
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.f;
  for (int r = lo + r0; r < hi; r += kQuantThreads / 16) {
    float f[8];
    bf16x8_to_float(__ldg(base + static_cast<size_t>(r) * (kQuantD / 8) + cg), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(f[i]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[r0][cg * 8 + i] = m[i];
  __syncthreads();
  if (threadIdx.x < kQuantD) {
    float a = 0.f;
#pragma unroll
    for (int r = 0; r < kQuantThreads / 16; ++r) a = fmaxf(a, part[r][threadIdx.x]);
    atomicMax(amax_bits + static_cast<size_t>(bh) * kQuantD + threadIdx.x, __float_as_uint(a));
  }
}

__global__ void __launch_bounds__(kQuantThreads)
    vquant_encode_kernel(const uint4* __restrict__ v, int N, int npad,
                         const unsigned int* __restrict__ amax_bits, uint2* __restrict__ vq,
                         float* __restrict__ vscale) {
  const int bh = blockIdx.y;
  const int cg = threadIdx.x & 15;
  const int r0 = threadIdx.x >> 4;
  const unsigned int* am = amax_bits + static_cast<size_t>(bh) * kQuantD;
  float inv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = __uint_as_float(__ldg(am + cg * 8 + i));
    inv[i] = a >= kAmaxZero ? __fdiv_rn(kE4M3Max, a) : 0.f;
  }
  if (blockIdx.x == 0 && threadIdx.x < kQuantD) {
    const float a = __uint_as_float(__ldg(am + threadIdx.x));
    vscale[static_cast<size_t>(bh) * kQuantD + threadIdx.x] = a >= kAmaxZero ? __fdiv_rn(a, kE4M3Max) : 0.f;
  }
  const int lo = blockIdx.x * kQuantRows;
  const int hi = min(npad, lo + kQuantRows);
  const uint4* base = v + static_cast<size_t>(bh) * npad * (kQuantD / 8);
  uint2* out = vq + static_cast<size_t>(bh) * npad * (kQuantD / 8);
  for (int r = lo + r0; r < hi; r += kQuantThreads / 16) {
    uint2 w = make_uint2(0u, 0u);
    if (r < N) {
      float f[8];
      bf16x8_to_float(__ldg(base + static_cast<size_t>(r) * (kQuantD / 8) + cg), f);
      uint32_t h[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        h[i] = cvt_e4m3x2(__fmul_rn(f[2 * i], inv[2 * i]), __fmul_rn(f[2 * i + 1], inv[2 * i + 1]));
      w = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    }
    out[static_cast<size_t>(r) * (kQuantD / 8) + cg] = w;
  }
}

// One CTA per (block of bs permuted rows, head): the rows' raster sources, then
// the encoding of each source row into its permuted position (pad rows 0).
__global__ void __launch_bounds__(kQuantThreads)
    vquant_gather_encode_kernel(const uint4* __restrict__ v, int N, int nb, int bs, TileGeom g,
                                const unsigned int* __restrict__ amax_bits, uint2* __restrict__ vq,
                                float* __restrict__ vscale) {
  __shared__ int src[128];
  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const int cg = threadIdx.x & 15;
  const int r0 = threadIdx.x >> 4;
  for (int r = threadIdx.x; r < bs; r += blockDim.x) {
    const int pos = i * bs + r;
    src[r] = pos < N ? source_index(pos, N, g) : -1;
  }
  const unsigned int* am = amax_bits + static_cast<size_t>(bh) * kQuantD;
  float inv[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float a = __uint_as_float(__ldg(am + cg * 8 + k));
    inv[k] = a >= kAmaxZero ? __fdiv_rn(kE4M3Max, a) : 0.f;
  }
  if (i == 0 && threadIdx.x < kQuantD) {
    const float a = __uint_as_float(__ldg(am + threadIdx.x));
    vscale[static_cast<size_t>(bh) * kQuantD + threadIdx.x] = a >= kAmaxZero ? __fdiv_rn(a, kE4M3Max) : 0.f;
  }
  __syncthreads();
  const uint4* base = v + static_cast<size_t>(bh) * N * (kQuantD / 8);
  uint2* out = vq + (static_cast<size_t>(bh) * nb * bs + static_cast<size_t>(i) * bs) * (kQuantD / 8);
  constexpr int kRowsPerPass = kQuantThreads / 16;
  constexpr int kInflight = 8;
  for (int rb = 0; rb < bs; rb += kRowsPerPass * kInflight) {
    uint4 x[kInflight];
#pragma unroll
    for (int k = 0; k < kInflight; ++k) {
      const int r = rb + r0 + k * kRowsPerPass;
      const int s = r < bs ? src[r] : -1;
      x[k] = s >= 0 ? __ldg(base + static_cast<size_t>(s) * (kQuantD / 8) + cg) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kInflight; ++k) {
      const int r = rb + r0 + k * kRowsPerPass;
      if (r >= bs) continue;
      uint2 w = make_uint2(0u, 0u);
      if (src[r] >= 0) {
        float f[8];
        bf16x8_to_float(x[k], f);
        uint32_t h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          h[e] = cvt_e4m3x2(__fmul_rn(f[2 * e], inv[2 * e]), __fmul_rn(f[2 * e + 1], inv[2 * e + 1]));
        w = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
      }
      out[static_cast<size_t>(r) * (kQuantD / 8) + cg] = w;
    }
  }
}

size_t vquant_ws_bytes(int BH) { return static_cast<size_t>(BH) * kQuantD * sizeof(unsigned int); }

// amax_bits must hold vquant_ws_bytes(BH) zeroed bytes (the caller clears them
// on the same stream).
cudaError_t launch_quantize_v(const void* v, int BH, int N, int npad, uint8_t* vq, float* vscale,
                              unsigned int* amax_bits, cudaStream_t st) {
  const dim3 ga((N + kQuantRows - 1) / kQuantRows, BH);
  vquant_amax_kernel<<<ga, kQuantThreads, 0, st>>>(static_cast<const uint4*>(v), N, npad, amax_bits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 ge((npad + kQuantRows - 1) / kQuantRows, BH);
  vquant_encode_kernel<<<ge, kQuantThreads, 0, st>>>(static_cast<const uint4*>(v), N, npad, amax_bits,
                                                     reinterpret_cast<uint2*>(vq), vscale);
  return cudaGetLastError();
}

// V in raster order [BH, N, 128] bf16 -> codes in the block order of g
// [BH, nb*bs, 128] and scales; amax_bits as above.
cudaError_t launch_permute_quantize_v(const void* v, int BH, int N, int bs, const TileGeom& g, uint8_t* vq,
                                      float* vscale, unsigned int* amax_bits, cudaStream_t st) {
  const int nb = (N + bs - 1) / bs;
  const dim3 ga((N + kQuantRows - 1) / kQuantRows, BH);
  vquant_amax_kernel<<<ga, kQuantThreads, 0, st>>>(static_cast<const uint4*>(v), N, N, amax_bits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 ge(nb, BH);
  vquant_gather_encode_kernel<<<ge, kQuantThreads, 0, st>>>(static_cast<const uint4*>(v), N, nb, bs, g, amax_bits,
                                                            reinterpret_cast<uint2*>(vq), vscale);
  return cudaGetLastError();
}

}  // namespace fvattn
