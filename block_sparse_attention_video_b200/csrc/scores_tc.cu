// scores_tc.cu -- block scores S = scale * qbar . kbar^T on the tensor cores
// [FVAttn §3.1: block-level similarity from pooled Q and K; §2.1].
//
// The score matrix feeds a softmax and a Top-p cut whose parity with an fp64
// reference is judged at 1e-5 relative, so plain TF32 (10 mantissa bits) is too
// coarse. Each fp32 operand x is split into two TF32 parts, hi = tf32(x) (round
// to nearest) and lo = x - hi (exact in fp32; the MMA reads its top 19 bits),
// and the product is accumulated as hi.hi + hi.lo + lo.hi in fp32 on the tensor
// cores (tcgen05.mma kind::tf32, accumulator in TMEM). The dropped lo.lo term and
// the truncation of lo are below 2^-21 of |q||k| per product, the order of fp32
// rounding.
//
// One CTA of 128 threads computes a 128 x 128 tile (query blocks x key blocks) of
// one (b, h). d is staged 32 at a time: every thread loads 16-byte pieces of the
// fp32 means (coalesced; the next stage's loads are in flight while the current
// stage's MMAs run), splits them and stores hi and lo into four 16 KB tiles
// in the 128-byte-swizzled K-major layout the MMA descriptors read (row r at
// r * 128 bytes, 16-byte piece j at position j ^ (r & 7)); one thread then issues
// 4 K-slices x 3 products = 12 MMAs of M = N = 128, K = 8 and commits them to an
// mbarrier that every thread waits on before the tiles are refilled. The
// epilogue reads the accumulator with tcgen05.ld (warp w holds rows 32w..32w+31),
// scales it and passes it through shared memory, 32 columns at a time, so that
// the stores to S are whole 128-byte row pieces. Means past nb read as zero.
//
// Waits are bounded like every wait of the library (2 s of %globaltimer, then
// FVATTN_ERR_TIMEOUT in the status word), and the tensor memory is freed on
// every path.
#include "common.cuh"
#include "sm100.cuh"

namespace fvattn {

namespace {

constexpr int kScThreads = 128;
constexpr int kScTile = 128;               // query blocks and key blocks per tile
constexpr int kScChunk = 32;               // d per stage: one 128-byte row of fp32
constexpr int kScOperandBytes = kScTile * kScChunk * 4;   // 16 KB
constexpr int kScSmemBytes = 4 * kScOperandBytes + 1024;  // hi/lo of both operands + alignment

// kind::tf32: fp32 accumulator (bit 4), A and B TF32 (format 2 in bits [7,10) and
// [10,13)), both K-major, N >> 3 in bits [17,23), M >> 4 in bits [24,29).
constexpr uint32_t kIdescTf32 = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(kScTile >> 3) << 17) |
                                (static_cast<uint32_t>(kScTile >> 4) << 24);

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Generic-proxy stores to shared memory made visible to the tensor cores.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// hi and lo TF32 parts of four fp32 values.
__device__ __forceinline__ void split4(const float4& v, uint4& hi, uint4& lo) {
  hi = make_uint4(to_tf32(v.x), to_tf32(v.y), to_tf32(v.z), to_tf32(v.w));
  lo = make_uint4(__float_as_uint(v.x - __uint_as_float(hi.x)), __float_as_uint(v.y - __uint_as_float(hi.y)),
                  __float_as_uint(v.z - __uint_as_float(hi.z)), __float_as_uint(v.w - __uint_as_float(hi.w)));
}

__global__ void __launch_bounds__(kScThreads)
    block_scores_tc_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, int nb, int d,
                           float scale, int ld, float* __restrict__ S, int* status) {
  extern __shared__ uint8_t sc_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sc_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* a_hi = base;
  uint8_t* a_lo = base + kScOperandBytes;
  uint8_t* b_hi = base + 2 * kScOperandBytes;
  uint8_t* b_lo = base + 3 * kScOperandBytes;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * kScTile, j0 = blockIdx.x * kScTile;
  const float* qb = qbar + static_cast<size_t>(bh) * nb * d;
  const float* kb = kbar + static_cast<size_t>(bh) * nb * d;

  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {   // warp-uniform: the whole warp allocates
    tmem_alloc(&tmem_base, kScTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  volatile int* af = &abort_flag;

  const uint32_t a_hi_s = smem_u32(a_hi), a_lo_s = smem_u32(a_lo);
  const uint32_t b_hi_s = smem_u32(b_hi), b_lo_s = smem_u32(b_lo);
  bool ok = true;
  int issued = 0;
  // A stage is 128 rows x 8 pieces of 16 bytes per operand: 8 pieces of each per
  // thread (row-contiguous across threads). All 16 loads of a stage are issued
  // together, and the next stage's loads are issued before the current stage's
  // MMAs are waited for, so the L2 latency overlaps the tensor-core work.
  constexpr int kPer = kScTile * 8 / kScThreads;
  float4 qa[kPer], ka[kPer];
  auto load_stage = [&](int c) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * kScThreads;
      const int r = e >> 3, j = e & 7;
      qa[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      ka[u] = qa[u];
      if (i0 + r < nb)
        qa[u] = __ldg(reinterpret_cast<const float4*>(qb + static_cast<size_t>(i0 + r) * d + c * kScChunk) + j);
      if (j0 + r < nb)
        ka[u] = __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(j0 + r) * d + c * kScChunk) + j);
    }
  };
  const int nchunks = d / kScChunk;
  load_stage(0);
  for (int c = 0; c < nchunks; ++c) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * kScThreads;
      const int r = e >> 3, j = e & 7;
      const uint32_t off = static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(j ^ (r & 7)) << 4);
      uint4 h, l;
      split4(qa[u], h, l);
      *reinterpret_cast<uint4*>(a_hi + off) = h;
      *reinterpret_cast<uint4*>(a_lo + off) = l;
      split4(ka[u], h, l);
      *reinterpret_cast<uint4*>(b_hi + off) = h;
      *reinterpret_cast<uint4*>(b_lo + off) = l;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kScChunk / 8; ++kk) {   // K = 8 fp32 = 32 bytes per MMA
        const uint32_t o = static_cast<uint32_t>(kk) * 32u;
        const uint64_t ah = umma_desc_sw128(a_hi_s + o, 16, 1024), al = umma_desc_sw128(a_lo_s + o, 16, 1024);
        const uint64_t bhd = umma_desc_sw128(b_hi_s + o, 16, 1024), bl = umma_desc_sw128(b_lo_s + o, 16, 1024);
        umma_tf32(tmem, ah, bhd, kIdescTf32, (c > 0 || kk > 0) ? 1u : 0u);
        umma_tf32(tmem, ah, bl, kIdescTf32, 1u);
        umma_tf32(tmem, al, bhd, kIdescTf32, 1u);
      }
      umma_commit(&mma_bar);
    }
    ++issued;
    if (c + 1 < nchunks) load_stage(c + 1);
    // every thread waits for the MMAs before the tiles are refilled (or read back)
    const bool done = mbar_wait(&mma_bar, static_cast<uint32_t>(c & 1), af, status);
    if (!__syncthreads_and(done)) {
      ok = false;
      break;
    }
  }
  tc_fence_after();
  if (ok) {
    // through shared memory (the operand tiles are free now): 32 columns at a time,
    // warp w writes its rows' values, then every warp stores whole 128-byte row pieces
    float* stage = reinterpret_cast<float*>(base);          // [128 rows][32 + 4]
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
    for (int cc = 0; cc < kScTile / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(t_row + cc * 32, v);
      tmem_wait_ld();
      float* srow = stage + (warp * 32 + lane) * 36;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(srow + 4 * q) =
            make_float4(__uint_as_float(v[4 * q]) * scale, __uint_as_float(v[4 * q + 1]) * scale,
                        __uint_as_float(v[4 * q + 2]) * scale, __uint_as_float(v[4 * q + 3]) * scale);
      __syncthreads();
      // 128 rows x 8 float4 per 32 columns: thread t stores piece t % 8 of rows t / 8 + 16 k
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = tid / 8 + 16 * k, q = tid % 8;
        const int i = i0 + r, j = j0 + cc * 32 + q * 4;
        if (i < nb && j < ld)
          *reinterpret_cast<float4*>(S + (static_cast<size_t>(bh) * nb + i) * ld + j) =
              *reinterpret_cast<const float4*>(stage + r * 36 + 4 * q);
      }
      __syncthreads();
    }
  }
  if (!ok && tid == 0 && issued > 0) {
    // a wait ran out: let any MMA still in flight finish (bounded) before freeing TMEM
    mbar_wait_plain(&mma_bar, static_cast<uint32_t>((issued - 1) & 1));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {   // warp-uniform: every lane of warp 0 passed the barrier
    tc_fence_after();
    tmem_dealloc(tmem, kScTile);
  }
}

}  // namespace

cudaError_t launch_block_scores_tc(const float* qbar, const float* kbar, int BH, int nb, int d, float scale,
                                   int ld, float* S, int* status, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(block_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kScSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((nb + kScTile - 1) / kScTile, (nb + kScTile - 1) / kScTile, BH);
  block_scores_tc_kernel<<<grid, kScThreads, kScSmemBytes, st>>>(qbar, kbar, nb, d, scale, ld, S, status);
  return cudaGetLastError();
}

}  // namespace fvattn
