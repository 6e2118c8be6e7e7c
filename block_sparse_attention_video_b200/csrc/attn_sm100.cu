// attn_sm100.cu -- block-sparse attention forward on the Blackwell tensor cores
// (tcgen05 MMA with TMEM accumulators, TMA-fed), bf16 inputs, d = 128, 128-token
// blocks [FVAttn §2.1: only selected (query block, key block) pairs are
// evaluated; GSRS §3.2: unselected blocks are skipped in the tiling loop;
// GSRS §A.1: online softmax, rescaling earlier partial results when the max
// grows].
//
// Work unit = one query block (128 rows) of one (b, h) with its KV block list.
// Persistent kernel, one CTA per SM, 384 threads (three warpgroups):
//   warps 0-3  softmax / epilogue of tile slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax / epilogue of tile slot 1
//   warp  8    TMA producer (one elected thread); also claims work units from a
//              global counter and publishes them to the other roles
//   warp  9    TMEM allocator and MMA issuer (one elected thread)
//   warps 10-11 idle
// The block launches with 168 registers per thread (384 x 168 = 64,512); the
// third warpgroup drops to 104 and the two softmax warpgroups rise to 200
// (2 x 128 x 200 + 128 x 104 = 64,512; per SMSP 2 x 200 + 104 <= 512). Each
// role ends in its own copy of the teardown so that the compiler allocates
// registers for each role under its own limit.
// Each slot walks its own unit's KV list, so the two slots ping-pong on the
// tensor core: while the softmax warps of one slot exponentiate S, the MMA
// warp runs the other slot's P.V and next Q.K^T.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
// P (bf16, two per 32-bit column) overwrites the first 64 columns of S and is
// the A operand of the P.V MMA straight from TMEM.
// Shared memory: Q0, Q1 (32 KB each) and a ring of 4 K/V stages (32 KB each),
// every tile stored as two 128-byte-swizzled halves of 64 columns, as TMA
// writes them. K-major descriptors for Q and K, an MN-major descriptor for V.
//
// Scheduling [FVAttn §2.2, §3.2: per-head work differs widely across heads]:
// units are claimed in an order the host prepares (heads by descending work,
// then each head's query blocks by descending list length), so heavy units
// start first and units that run together share a head's K/V in L2.
//
// Softmax: exponent base 2 with scale*log2(e) folded in, P rounded to bf16,
// fp32 row sums. The running max is only raised (and O rescaled in TMEM) when
// a block's max exceeds it by more than 8 (a factor 256), which keeps P <= 256.
#include <cfloat>

#include "common.cuh"
#include "sm100.cuh"

namespace fvattn {
namespace sm100 {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int HD = 128;
constexpr int kStages = 4;
constexpr int kTileBytes = BM * HD * 2;  // 32 KB
constexpr int kHalfBytes = 128 * 64 * 2; // 16 KB: 128 rows x 128 bytes
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 200;
constexpr int kRegsControl = 104;
constexpr uint32_t kIdescQK = umma_idesc_bf16(BM, BN, false);
constexpr uint32_t kIdescPV = umma_idesc_bf16(BM, HD, true);
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

struct Params {
  int nb;
  int N;
  int npad;
  int total_units;
  float scale_log2;
  const int* kv_idx;        // nullptr: dense (every block, in order)
  const int* kv_cnt;
  const int* head_order;    // [B*H] rank -> bh
  const int* local_order;   // [B*H*nb] (bh, rank) -> query block
  __nv_bfloat16* out;
  float* lse;
  int* status;
  unsigned long long* counter;
};

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t kv[kStages][kTileBytes];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t unit_full[2][2];
  uint64_t unit_empty[2][2];
  uint64_t mma_done;
  int unit_box[2][2];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + room to align the base

struct Unit {
  int bh, i, cnt;
  const int* list;
};

__device__ __forceinline__ Unit decode_unit(int u, const Params& P) {
  Unit x;
  x.bh = 0;
  x.i = 0;
  x.cnt = 0;
  x.list = nullptr;
  if (u < 0 || u >= P.total_units) return x;
  if (P.kv_idx) {
    const int r = u / P.nb;
    const int k = u - r * P.nb;
    x.bh = __ldg(P.head_order + r);
    x.i = __ldg(P.local_order + static_cast<size_t>(x.bh) * P.nb + k);
    const size_t row = static_cast<size_t>(x.bh) * P.nb + x.i;
    int c = __ldg(P.kv_cnt + row);
    if (c < 1 || c > P.nb) {
      record_status(P.status, FVATTN_ERR_INVALID_ARG);
      c = min(max(c, 1), P.nb);
    }
    x.cnt = c;
    x.list = P.kv_idx + row * P.nb;
  } else {
    x.bh = u / P.nb;
    x.i = u - x.bh * P.nb;
    x.cnt = P.nb;
  }
  return x;
}

__device__ __forceinline__ int block_at(const Unit& x, int k, const Params& P) {
  if (!x.list) return k;
  int j = __ldg(x.list + k);
  if (j < 0 || j >= P.nb) {
    record_status(P.status, FVATTN_ERR_INVALID_ARG);
    j = 0;
  }
  return j;
}

// The op sequence shared by the producer and the MMA issuer. For each slot:
// S(0); then repeatedly PV(k-1) followed by S(k) (or, at the end of a unit, the
// next unit's S(0)). Slots alternate step by step.
template <class GetUnit, class OnS, class OnPV>
__device__ __forceinline__ bool run_schedule(GetUnit&& get_unit, OnS&& on_s, OnPV&& on_pv) {
  Unit st[2];
  int k[2] = {0, 0};
  bool act[2] = {false, false};
#pragma unroll
  for (int X = 0; X < 2; ++X) {
    if (!get_unit(X, st[X])) return false;
    act[X] = st[X].cnt > 0;
    if (act[X]) {
      if (!on_s(X, st[X], 0)) return false;
      k[X] = 1;
    }
  }
#pragma unroll 1
  while (act[0] || act[1]) {
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      if (!act[X]) continue;
      if (!on_pv(X, st[X], k[X] - 1)) return false;
      if (k[X] == st[X].cnt) {
        if (!get_unit(X, st[X])) return false;
        act[X] = st[X].cnt > 0;
        if (!act[X]) continue;
        if (!on_s(X, st[X], 0)) return false;
        k[X] = 1;
      } else {
        if (!on_s(X, st[X], k[X])) return false;
        ++k[X];
      }
    }
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    for (int X = 0; X < 2; ++X) {
      mbar_init(&sm.q_full[X], 1);
      mbar_init(&sm.q_empty[X], 1);
      mbar_init(&sm.s_full[X], 1);
      mbar_init(&sm.p_full[X], 4);
      mbar_init(&sm.o_full[X], 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.unit_full[X][b], 1);
        mbar_init(&sm.unit_empty[X][b], 5);
      }
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // All 384 threads meet here once at the end; then the allocating warp frees TMEM.
  auto teardown = [&]() {
    __syncwarp();
    tc_fence_before();
    asm volatile("barrier.sync 1, %0;" ::"n"(kThreads) : "memory");
    if (warp == 9) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  };

  if (warp >= 8) {
    regs_dec<kRegsControl>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      int qn[2] = {0, 0};
      int un[2] = {0, 0};
      auto get_unit = [&](int X, Unit& x) -> bool {
        const int b = un[X] & 1;
        if (!mbar_wait(&sm.unit_empty[X][b], ((un[X] >> 1) & 1) ^ 1, abort_flag, P.status)) return false;
        int u = static_cast<int>(atomicAdd(P.counter, 1ull));
        if (u >= P.total_units) u = -1;
        sm.unit_box[X][b] = u;
        mbar_arrive(&sm.unit_full[X][b]);
        ++un[X];
        x = decode_unit(u, P);
        return true;
      };
      auto load_kv = [&](const CUtensorMap* tm, int row) -> bool {
        const int s = it % kStages;
        if (!mbar_wait(&sm.kv_empty[s], ((it / kStages) & 1) ^ 1, abort_flag, P.status)) return false;
        mbar_arrive_expect_tx(&sm.kv_full[s], kTileBytes);
        tma_load_2d(sm.kv[s], tm, &sm.kv_full[s], 0, row);
        tma_load_2d(sm.kv[s] + kHalfBytes, tm, &sm.kv_full[s], 64, row);
        ++it;
        return true;
      };
      auto on_s = [&](int X, const Unit& x, int k) -> bool {
        if (k == 0) {
          if (!mbar_wait(&sm.q_empty[X], (qn[X] & 1) ^ 1, abort_flag, P.status)) return false;
          const int row = x.bh * P.npad + x.i * BM;
          mbar_arrive_expect_tx(&sm.q_full[X], kTileBytes);
          tma_load_2d(sm.q[X], &tm_q, &sm.q_full[X], 0, row);
          tma_load_2d(sm.q[X] + kHalfBytes, &tm_q, &sm.q_full[X], 64, row);
          ++qn[X];
        }
        return load_kv(&tm_k, x.bh * P.npad + block_at(x, k, P) * BN);
      };
      auto on_pv = [&](int X, const Unit& x, int k) -> bool {
        return load_kv(&tm_v, x.bh * P.npad + block_at(x, k, P) * BN);
      };
      run_schedule(get_unit, on_s, on_pv);
      // Drain: every load this thread armed has landed before the CTA exits.
      for (int o = max(0, it - kStages); o < it; ++o)
        mbar_wait_plain(&sm.kv_full[o % kStages], (o / kStages) & 1);
      for (int X = 0; X < 2; ++X)
        if (qn[X] > 0) mbar_wait_plain(&sm.q_full[X], (qn[X] - 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0;
      int qn[2] = {0, 0};
      int pn[2] = {0, 0};
      int un[2] = {0, 0};
      const uint32_t q_addr[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      auto get_unit = [&](int X, Unit& x) -> bool {
        const int b = un[X] & 1;
        if (!mbar_wait(&sm.unit_full[X][b], (un[X] >> 1) & 1, abort_flag, P.status)) return false;
        const int u = *reinterpret_cast<volatile int*>(&sm.unit_box[X][b]);
        mbar_arrive(&sm.unit_empty[X][b]);
        ++un[X];
        x = decode_unit(u, P);
        return true;
      };
      auto on_s = [&](int X, const Unit& x, int k) -> bool {
        if (k == 0) {
          if (!mbar_wait(&sm.q_full[X], qn[X] & 1, abort_flag, P.status)) return false;
          ++qn[X];
        }
        const int s = it % kStages;
        if (!mbar_wait(&sm.kv_full[s], (it / kStages) & 1, abort_flag, P.status)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.kv[s]);
        const uint32_t d_tmem = tmem + X * 128;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          umma_ss(d_tmem, umma_desc_sw128(q_addr[X] + off, 16, 1024),
                  umma_desc_sw128(k_addr + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.kv_empty[s]);
        umma_commit(&sm.s_full[X]);
        if (k == x.cnt - 1) umma_commit(&sm.q_empty[X]);
        ++it;
        return true;
      };
      auto on_pv = [&](int X, const Unit& x, int k) -> bool {
        if (!mbar_wait(&sm.p_full[X], pn[X] & 1, abort_flag, P.status)) return false;
        ++pn[X];
        const int s = it % kStages;
        if (!mbar_wait(&sm.kv_full[s], (it / kStages) & 1, abort_flag, P.status)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm.kv[s]);
        const uint32_t p_tmem = tmem + X * 128;
        const uint32_t o_tmem = tmem + 256 + X * 128;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          umma_ts(o_tmem, p_tmem + kk * 8, umma_desc_sw128(v_addr + kk * 2048, kHalfBytes, 1024),
                  kIdescPV, (k > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&sm.kv_empty[s]);
        if (k == x.cnt - 1) umma_commit(&sm.o_full[X]);
        ++it;
        return true;
      };
      run_schedule(get_unit, on_s, on_pv);
      // Drain: every MMA this thread issued has completed before TMEM is freed.
      umma_commit(&sm.mma_done);
      mbar_wait_plain(&sm.mma_done, 0);
    }
  }
    teardown();
    return;
  }

  regs_inc<kRegsSoftmax>();
  {
    // ------------------------------------------------------------ softmax / epilogue
    const int X = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + X * 128;
    const uint32_t tO = tmem + lane_off + 256 + X * 128;
    const int tail = P.N - (P.nb - 1) * BN;  // valid keys in the last block
    const float sl2 = P.scale_log2;
    int n = 0, sn = 0, on = 0;
#pragma unroll 1
    while (true) {
      const int b = n & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.unit_full[X][b], (n >> 1) & 1, abort_flag, P.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&sm.unit_box[X][b]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.unit_empty[X][b]);
      ++n;
      const Unit x = decode_unit(u, P);
      if (x.cnt == 0) break;
      float m_run = -FLT_MAX;
      float l_run = 0.f;
      bool ok = true;
#pragma unroll 1
      for (int k = 0; k < x.cnt; ++k) {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[X], sn & 1, abort_flag, P.status))) { ok = false; break; }
        ++sn;
        tc_fence_after();
        uint32_t s[4][32];
        tmem_ld32(tS + 0, s[0]);
        tmem_ld32(tS + 32, s[1]);
        tmem_ld32(tS + 64, s[2]);
        tmem_ld32(tS + 96, s[3]);
        tmem_wait_ld();
        const int j = block_at(x, k, P);
        if (j == P.nb - 1 && tail < BN) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c * 32 + e >= tail) s[c][e] = __float_as_uint(-INFINITY);
        }
        float mx = -FLT_MAX;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(s[c][e]));
        const float m_new = mx * sl2;
        if (k == 0) {
          m_run = m_new;
        } else if (m_new > m_run + kRescaleThreshold) {
          const float f = ex2_approx(m_run - m_new);
          l_run *= f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(tO + c * 32, o);
          }
          tmem_wait_st();
          m_run = m_new;
        }
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(s[c][2 * e]), sl2, -m_run));
            const float p1 = ex2_approx(fmaf(__uint_as_float(s[c][2 * e + 1]), sl2, -m_run));
            lsum += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        l_run += lsum;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[X]);
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[X], on & 1, abort_flag, P.status))) break;
      ++on;
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const size_t grow = static_cast<size_t>(x.bh) * P.npad + static_cast<size_t>(x.i) * BM + row;
      uint4* orow = reinterpret_cast<uint4*>(P.out + grow * HD);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          orow[c * 4 + e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      }
      if (P.lse) P.lse[grow] = (m_run + __log2f(l_run)) * kLn2;
      tc_fence_before();
    }
  }

  teardown();
}

}  // namespace sm100

// ---------------------------------------------------------------- work order
// Within each head: query blocks by descending list length (ties: lower index).
// Per head: total work. Then heads by descending total (ties: lower index).
__device__ __forceinline__ void bitonic_desc_u32(uint32_t* a, int n) {
  for (int size = 2; size <= n; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < n / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint32_t x = a[lo], y = a[hi];
        if ((x < y) == desc) { a[lo] = y; a[hi] = x; }
      }
    }
  __syncthreads();
}

__device__ __forceinline__ void bitonic_desc_u64(unsigned long long* a, int n) {
  for (int size = 2; size <= n; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < n / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = a[lo], y = a[hi];
        if ((x < y) == desc) { a[lo] = y; a[hi] = x; }
      }
    }
  __syncthreads();
}

__global__ void __launch_bounds__(1024)
    plan_heads_kernel(const int* __restrict__ kv_cnt, int nb, int* __restrict__ local_order,
                      unsigned long long* __restrict__ head_total) {
  __shared__ uint32_t keys[4096];
  __shared__ unsigned long long red[32];
  const int bh = blockIdx.x;
  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  unsigned long long part = 0;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    if (i < nb) {
      const int c = min(max(kv_cnt[static_cast<size_t>(bh) * nb + i], 1), nb);
      keys[i] = (static_cast<uint32_t>(c) << 16) | static_cast<uint32_t>(0xFFFF - i);
      part += static_cast<unsigned long long>(c);
    } else {
      keys[i] = 0u;
    }
  }
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  bitonic_desc_u32(keys, n2);
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    for (int w = 0; w < (blockDim.x + 31) / 32; ++w) t += red[w];
    head_total[bh] = t;
  }
  for (int r = threadIdx.x; r < nb; r += blockDim.x)
    local_order[static_cast<size_t>(bh) * nb + r] = 0xFFFF - static_cast<int>(keys[r] & 0xFFFFu);
}

__global__ void __launch_bounds__(1024)
    plan_rank_kernel(const unsigned long long* __restrict__ head_total, int BH,
                     int* __restrict__ head_order) {
  __shared__ unsigned long long keys[4096];
  int n2 = 1;
  while (n2 < BH) n2 <<= 1;
  for (int i = threadIdx.x; i < n2; i += blockDim.x)
    keys[i] = i < BH ? ((head_total[i] << 16) | static_cast<unsigned long long>(0xFFFF - i)) : 0ull;
  bitonic_desc_u64(keys, n2);
  for (int r = threadIdx.x; r < BH; r += blockDim.x)
    head_order[r] = 0xFFFF - static_cast<int>(keys[r] & 0xFFFFull);
}

// ---------------------------------------------------------------- launcher
size_t attn_sm100_smem_bytes() { return sm100::kSmemBytes; }

cudaError_t launch_attn_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              void* out, float* lse, const int* kv_idx, const int* kv_cnt,
                              int* local_order, unsigned long long* head_total, int* head_order,
                              int BH, int N, int nb, float scale, int* status,
                              unsigned long long* counter, int num_sms, cudaStream_t st) {
  if (kv_idx) {
    plan_heads_kernel<<<BH, 1024, 0, st>>>(kv_cnt, nb, local_order, head_total);
    plan_rank_kernel<<<1, 1024, 0, st>>>(head_total, BH, head_order);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sm100::Params P;
  P.nb = nb;
  P.N = N;
  P.npad = nb * sm100::BM;
  P.total_units = BH * nb;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.kv_idx = kv_idx;
  P.kv_cnt = kv_cnt;
  P.head_order = head_order;
  P.local_order = local_order;
  P.out = static_cast<__nv_bfloat16*>(out);
  P.lse = lse;
  P.status = status;
  P.counter = counter;
  cudaError_t e = cudaFuncSetAttribute(sm100::attn_fwd_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sm100::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int grid = max(1, min(num_sms, P.total_units));
  sm100::attn_fwd_sm100_kernel<<<grid, sm100::kThreads, sm100::kSmemBytes, st>>>(tq, tk, tv, P);
  return cudaGetLastError();
}

}  // namespace fvattn
