// attn_sm100.cu -- block-sparse attention forward on the Blackwell tensor cores
// (tcgen05 MMA with TMEM accumulators, TMA-fed), bf16 inputs, head dimension
// d = 64 or 128, blocks of BN = 64 or 128 tokens [FVAttn §2.1: only selected (query block, key block)
// pairs are evaluated; GSRS §3.2: unselected blocks are skipped in the tiling
// loop; GSRS §A.1: online softmax, rescaling earlier partial results when the
// max grows].
//
// Work unit = 256 consecutive query rows of one (b, h), i.e. G = 256/BN query
// blocks, held as two 128-row Q tiles (slots 0 and 1). The unit walks the
// UNION of its query blocks' KV lists in ascending block order; each union entry
// carries a membership bit per query block. Every K/V block of the union is
// loaded once and feeds both tiles, so adjacent query blocks, whose lists
// overlap heavily, share their K/V traffic. A tile row whose query block did
// not select a key block gets P = 0 for it (no exponentials), which leaves its
// output exactly the softmax over its own selected blocks.
//
// Persistent kernel, one CTA per SM, 384 threads (three warpgroups):
//   warps 0-3  softmax / epilogue of slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax / epilogue of slot 1
//   warp  8    TMA producer (one elected thread); claims work units from a
//              global counter and publishes them to the other roles
//   warp  9    TMEM allocator and MMA issuer (the whole warp walks the unit;
//              one elected lane issues each MMA and commit)
//   warps 10-11 idle
// The block launches with 168 registers per thread (384 x 168 = 64,512); the
// third warpgroup drops to 128 and the two softmax warpgroups rise to 184
// (2 x 128 x 184 + 128 x 128 = 63,488 <= 64,512; per SMSP 2 x 184 + 128 <= 512). Each
// role ends in its own copy of the teardown so that the compiler allocates
// registers for each role under its own limit.
//
// MMA order per unit: S0(0) S1(0), then for k >= 1: PV0(k-1) S0(k) PV1(k-1)
// S1(k), and finally PV0(last) PV1(last): the exponentials of one slot overlap
// the other slot's MMAs. With BN = 64 a slot leaves out its S and P.V of a step
// that neither of its two query blocks selected (the softmax warps skip that
// step too); Q and O of both slots are released after the unit's last MMA.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
// P (bf16, two per 32-bit column) overwrites the first 64 columns of S and is
// the A operand of the P.V MMA straight from TMEM.
// Shared memory: Q0, Q1 (32 KB each) and a 128 KB K/V ring of 4 x 32 KB stages
// of 128 key rows, stored as two 128-byte-swizzled halves of 64 columns, as TMA
// writes them. A step is 128 keys: one 128-token block, or (BN = 64) two
// consecutive union entries whose 64-row tiles fill the two row halves of the
// stage, so every S MMA is N = 128 and every P.V is K = 128 whatever BN is; the
// softmax masks, sums and records each 64-key half of such a step by its own
// entry. K-major descriptors for Q and K, MN-major for V.
//
// Scheduling [FVAttn §2.2, §3.2: per-head work differs widely across heads]:
// units are claimed in an order prepared on the device (heads by descending
// work, then each head's units by descending union length), so heavy units
// start first and units that run together share a head's K/V in L2.
//
// Softmax: exponent base 2 with scale*log2(e) folded in, P rounded to bf16,
// fp32 row sums. The running max is only raised (and O rescaled in TMEM) when a
// block's max exceeds it by more than 8 (a factor 256), which keeps P <= 256.
//
// 8-bit V variant (F8 = true) [FVAttn §3.4: V is quantized on the GPU before
// attention]: V arrives as E4M3 codes [B*H, Npad, 128] with one fp32 scale per
// channel, and P.V runs as a kind::f8f6f4 MMA with P in E4M3 as well (P takes
// 32 TMEM columns per 128 keys, four per 32-bit column; K = 32 per MMA). P is
// formed relative to m_run - 4 with a rescale threshold of 4, so P <= 2^8 stays
// inside E4M3's range (448) while values down to 2^-14 of 2^m_run keep a code.
// The row sums add the E4M3 values actually multiplied (exact f16 pairs, summed
// in f16 over 16 keys, then in fp32), so P/l stays a distribution. The channel
// scales are applied with 1/l in the epilogue. A V stage is 16 KB: one
// 128-byte swizzled row per key, read by an MN-major descriptor.
#include <cfloat>

#include "common.cuh"
#include "sm100.cuh"

namespace fvattn {
namespace sm100 {


constexpr int kUnitRows = 256;
constexpr int kQHalfBytes = 128 * 128;      // 16 KB: 128 rows x 64 columns (128 bytes)
constexpr int kRingBytes = 128 * 1024;
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 184;
constexpr int kRegsControl = 128;
constexpr float kLn2 = 0.6931471805599453f;

// A step covers 128 keys: one 128-token block, or two consecutive union entries
// of 64-token blocks whose K (V) tiles are loaded into the two 64-row halves of
// one 128-row stage. Every step is then an N = 128 S MMA and a K = 128 P.V.
// HD = head dimension, 64 or 128: one or two 64-column (128-byte) halves per row.
template <int BN, bool F8 = false, int HD = 128>
struct Tile {
  static constexpr int kHalves = HD / 64;
  static constexpr int kQTileBytes = 128 * HD * 2;         // 32 KB (d 128), 16 KB (d 64)
  static constexpr int kStepKeys = 128;
  static constexpr int kBPS = kStepKeys / BN;              // union entries per step
  static constexpr int kKVBytes = kStepKeys * HD * 2;      // 32 KB (16 KB) stage
  static constexpr int kKVHalf = kStepKeys * 128;          // one 64-column half of a stage
  static constexpr int kSubBytes = BN * 128;               // one entry's rows within a half
  static constexpr int kStages = kRingBytes / kKVBytes;
  static constexpr int kGroup = kUnitRows / BN;            // query blocks per unit
  static constexpr uint32_t kIdescQK = umma_idesc_bf16(128, kStepKeys, false);
  static constexpr uint32_t kIdescPV =
      F8 ? umma_idesc_e4m3(128, HD, true) : umma_idesc_bf16(128, HD, true);
  static constexpr int kVBytes = F8 ? kStepKeys * HD : kKVBytes;    // V stage bytes
  static constexpr int kPVK = F8 ? 32 : 16;                         // keys per P.V MMA
  static constexpr int kPCols = kStepKeys / (F8 ? 4 : 2);           // TMEM columns of P
  static constexpr float kPShift = F8 ? 4.0f : 0.0f;                // P relative to m_run - shift
  static constexpr float kThreshold = F8 ? 4.0f : 8.0f;             // lazy rescale threshold
};

struct Params {
  int nb;
  int N;
  int npad;
  int ngroups;
  int total_units;
  float scale_log2;
  const uint32_t* ulist;    // [B*H*ngroups*nb] union entries j | members << 16; nullptr: dense
  const int* ucnt;          // [B*H*ngroups]
  const int* head_order;    // [B*H] rank -> bh
  const int* local_order;   // [B*H*ngroups] (bh, rank) -> group
  __nv_bfloat16* out;
  float* lse;
  float* blse;              // nullable [B*H, nb, npad]: per (key block, row) log-sum-exp
  const float* vscale;      // F8: [B*H, 128] per-channel scales of the E4M3 V
  int* status;
  unsigned long long* counter;
};

template <int BN, int HD>
struct __align__(1024) Smem {
  uint8_t q[2][Tile<BN, false, HD>::kQTileBytes];
  uint8_t kv[kRingBytes];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[Tile<BN, false, HD>::kStages];
  uint64_t kv_empty[Tile<BN, false, HD>::kStages];
  uint64_t s_full[2];
  uint64_t p_full[2][2];   // [slot][half of P]
  uint64_t o_full[2];
  uint64_t unit_full[2];
  uint64_t unit_empty[2];
  uint64_t mma_done;
  int unit_box[2];
  uint32_t tmem_base;
  int abort_flag;
};

struct Unit {
  int bh, grp, cnt;
  const uint32_t* list;
  bool slot[2];
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, const Params& P) {
  constexpr int G = Tile<BN>::kGroup;
  Unit x;
  x.bh = 0;
  x.grp = 0;
  x.cnt = 0;
  x.list = nullptr;
  x.slot[0] = x.slot[1] = false;
  if (u < 0 || u >= P.total_units) return x;
  if (P.ulist) {
    const int r = u / P.ngroups;
    const int k = u - r * P.ngroups;
    x.bh = __ldg(P.head_order + r);
    x.grp = __ldg(P.local_order + static_cast<size_t>(x.bh) * P.ngroups + k);
    const size_t row = static_cast<size_t>(x.bh) * P.ngroups + x.grp;
    x.cnt = min(max(__ldg(P.ucnt + row), 1), P.nb);
    x.list = P.ulist + row * P.nb;
  } else {
    x.bh = u / P.ngroups;
    x.grp = u - x.bh * P.ngroups;
    x.cnt = P.nb;
  }
  x.slot[0] = x.grp * G < P.nb;
  x.slot[1] = x.grp * G + G / 2 < P.nb;
  return x;
}

template <int BN>
__device__ __forceinline__ uint32_t entry_at(const Unit& x, int k, const Params& P) {
  constexpr uint32_t kAll = (1u << Tile<BN>::kGroup) - 1u;
  if (!x.list) return static_cast<uint32_t>(k) | (kAll << 16);
  uint32_t e = __ldg(x.list + k);
  if ((e & 0xFFFFu) >= static_cast<uint32_t>(P.nb)) {
    record_status(P.status, FVATTN_ERR_INVALID_ARG);
    e &= 0xFFFF0000u;
  }
  return e;
}

template <int BN, bool F8, int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Params P) {
  using T = Tile<BN, F8, HD>;
  static_assert(HD == 64 || HD == 128, "head dimension 64 or 128");
  static_assert(!F8 || HD == 128, "the E4M3-V path has d = 128");
  constexpr int kStages = T::kStages;
  extern __shared__ uint8_t smem_raw[];
  Smem<BN, HD>& sm = *reinterpret_cast<Smem<BN, HD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    for (int X = 0; X < 2; ++X) {
      mbar_init(&sm.q_full[X], 1);
      mbar_init(&sm.q_empty[X], 1);
      mbar_init(&sm.s_full[X], 1);
      mbar_init(&sm.p_full[X][0], 4);
      mbar_init(&sm.p_full[X][1], 4);
      mbar_init(&sm.o_full[X], 1);
      mbar_init(&sm.unit_full[X], 1);
      mbar_init(&sm.unit_empty[X], 9);   // MMA thread + 4 + 4 softmax warps
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 9) {   // warp-uniform: the whole warp allocates
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
  //
  // Warp-collective tensor-memory instructions (tcgen05.alloc/dealloc/ld/st and
  // wait::ld/st, all .sync.aligned) must be executed by every lane of the warp
  // together. Each call site below states why its control flow is warp-uniform.
  // The %globaltimer bound on the mbarrier waits cannot rescue a warp whose lanes
  // diverged around such an instruction: the lanes that reached it wait there for
  // the others with no limit. (An earlier version rescaled O under a per-row
  // branch around tcgen05.ld/st; a first test run with large logits hung in it
  // until the run was killed. The rescale now branches on a warp vote.)
  auto teardown = [&]() {
    __syncwarp();
    tc_fence_before();
    asm volatile("barrier.sync 1, %0;" ::"n"(kThreads) : "memory");
    if (warp == 9) {   // warp-uniform: every lane of warp 9 passed the barrier above
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  };

  if (warp >= 8) {
    regs_dec<kRegsControl>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- producer
      int it = 0, un = 0;
      int qn[2] = {0, 0};
      bool ok = true;
      while (ok) {
        const int b = un & 1;
        if (!mbar_wait(&sm.unit_empty[b], ((un >> 1) & 1) ^ 1, abort_flag, P.status)) break;
        int u = static_cast<int>(atomicAdd(P.counter, 1ull));
        if (u >= P.total_units) u = -1;
        sm.unit_box[b] = u;
        mbar_arrive(&sm.unit_full[b]);
        ++un;
        const Unit x = decode_unit<BN>(u, P);
        if (x.cnt == 0) break;
        const int row0 = x.bh * P.npad + x.grp * kUnitRows;
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          if (!(X == 0 ? x.slot[0] : x.slot[1])) continue;
          if (!mbar_wait(&sm.q_empty[X], (qn[X] & 1) ^ 1, abort_flag, P.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.q_full[X], T::kQTileBytes);
#pragma unroll
          for (int hq = 0; hq < T::kHalves; ++hq)
            tma_load_2d(sm.q[X] + hq * kQHalfBytes, &tm_q, &sm.q_full[X], 64 * hq, row0 + X * 128);
          ++qn[X];
        }
        const int ns = (x.cnt + T::kBPS - 1) / T::kBPS;
        for (int k = 0; ok && k < ns; ++k) {
          int kvrow[T::kBPS];
#pragma unroll
          for (int h = 0; h < T::kBPS; ++h) {
            // past the list's end (odd count): repeat the step's first block; its
            // half of the S tile is masked by the softmax warps
            const int idx = T::kBPS * k + h < x.cnt ? T::kBPS * k + h : T::kBPS * k;
            kvrow[h] = x.bh * P.npad + static_cast<int>(entry_at<BN>(x, idx, P) & 0xFFFFu) * BN;
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {     // K(k) then V(k)
            const int s = it % kStages;
            if (!mbar_wait(&sm.kv_empty[s], ((it / kStages) & 1) ^ 1, abort_flag, P.status)) { ok = false; break; }
            uint8_t* dst = sm.kv + s * T::kKVBytes;
            if (F8 && t == 1) {
              // E4M3 V: one 128-byte row (all channels) per key, one box per entry
              mbar_arrive_expect_tx(&sm.kv_full[s], T::kVBytes);
#pragma unroll
              for (int h = 0; h < T::kBPS; ++h)
                tma_load_2d(dst + h * T::kSubBytes, &tm_v, &sm.kv_full[s], 0, kvrow[h]);
            } else {
              mbar_arrive_expect_tx(&sm.kv_full[s], T::kKVBytes);
              const CUtensorMap* tm = t == 0 ? &tm_k : &tm_v;
#pragma unroll
              for (int h = 0; h < T::kBPS; ++h) {
#pragma unroll
                for (int hq = 0; hq < T::kHalves; ++hq)
                  tma_load_2d(dst + hq * T::kKVHalf + h * T::kSubBytes, tm, &sm.kv_full[s], 64 * hq, kvrow[h]);
              }
            }
            ++it;
          }
        }
      }
      // Drain: every load this thread armed has landed before the CTA exits.
      for (int o = max(0, it - kStages); o < it; ++o)
        mbar_wait_plain(&sm.kv_full[o % kStages], (o / kStages) & 1);
      for (int X = 0; X < 2; ++X)
        if (qn[X] > 0) mbar_wait_plain(&sm.q_full[X], (qn[X] - 1) & 1);
    } else if (warp == 9) {
      // ---------------------------------------------------------- MMA issuer
      // The whole warp runs this loop: every value in it is warp-uniform, each wait
      // is a warp vote, and one elected lane issues each tcgen05.mma / commit. The
      // shared-memory descriptors are built once; a stage or K slice is a constant
      // added to the start-address field (addresses stay inside the 18-bit window,
      // so the field never carries).
      int base = 0, un = 0;
      int qn[2] = {0, 0};
      int pn[2] = {0, 0};
      const uint64_t dq[2] = {umma_desc_sw128(smem_u32(sm.q[0]), 16, 1024),
                              umma_desc_sw128(smem_u32(sm.q[1]), 16, 1024)};
      const uint64_t dk = umma_desc_sw128(smem_u32(sm.kv), 16, 1024);
      const uint64_t dv = umma_desc_sw128(smem_u32(sm.kv), T::kKVHalf, 1024);
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, P.status));
      };
      bool ok = true;
      while (ok) {
        const int b = un & 1;
        if (!wait(&sm.unit_full[b], (un >> 1) & 1)) break;
        const int u = *reinterpret_cast<volatile int*>(&sm.unit_box[b]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.unit_empty[b]);
        ++un;
        const Unit x = decode_unit<BN>(u, P);
        if (x.cnt == 0) break;
        const int cnt = (x.cnt + T::kBPS - 1) / T::kBPS;   // steps of 128 keys
        auto kv_ready = [&](int o) -> bool { return wait(&sm.kv_full[o % kStages], (o / kStages) & 1); };
        // Member-only MMAs with 64-token blocks: a unit there spans four query blocks,
        // and slot X computes S and P.V for a step only when one of its two query
        // blocks selected one of the step's entries (the softmax warps skip the same
        // steps, decided from the same entries). Per 32 union entries one coalesced
        // load and two ballots give each entry's slot membership; the next window's
        // entries are loaded ahead. With 128-token blocks every slot computes every
        // step: there a skip saves less than the test costs in this warp.
        constexpr int G = T::kGroup;
        constexpr uint32_t kMask0 = (1u << (G / 2)) - 1u, kMask1 = kMask0 << (G / 2);
        uint32_t win[2] = {~0u, ~0u}, prev[2] = {~0u, ~0u};
        int wbase = 0;
        uint32_t ent_next = (BN == 64 && x.list && lane < x.cnt) ? __ldg(x.list + lane) : 0u;
        auto refill = [&]() {
          prev[0] = win[0];
          prev[1] = win[1];
          win[0] = __ballot_sync(0xffffffffu, ((ent_next >> 16) & kMask0) != 0u);
          win[1] = __ballot_sync(0xffffffffu, ((ent_next >> 16) & kMask1) != 0u);
          const int nx = wbase + 32 + lane;
          ent_next = (x.list && nx < x.cnt) ? __ldg(x.list + nx) : 0u;
        };
        if (BN == 64 && x.list) refill();
        // Steps are asked for in the order k-1, k (slot 0), k-1, k (slot 1): never more
        // than one step behind the newest, so the previous window covers the older one.
        auto member = [&](int X, int k) -> bool {
          if (BN != 64 || !x.list) return true;
          const int e0 = k * T::kBPS;
          while (e0 >= wbase + 32) {
            wbase += 32;
            refill();
          }
          const uint32_t w = e0 >= wbase ? win[X] : prev[X];
          const int sh = e0 >= wbase ? e0 - wbase : e0 - wbase + 32;
          return ((w >> sh) & ((1u << T::kBPS) - 1u)) != 0u;
        };
        bool started[2] = {false, false};
        auto s_op = [&](int X, int k) -> bool {   // S_X = Q_X K(k)^T, K(k) already waited on
          if (!member(X, k)) return true;
          if (!started[X]) {
            if (!wait(&sm.q_full[X], qn[X] & 1)) return false;
            ++qn[X];
          }
          tc_fence_after();
          const uint64_t ks = dk + static_cast<uint64_t>(((base + 2 * k) % kStages) * (T::kKVBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            constexpr int kQH = kQHalfBytes;
            const uint32_t qo = ((kk >> 2) * kQH + (kk & 3) * 32) >> 4;
            const uint32_t ko = ((kk >> 2) * T::kKVHalf + (kk & 3) * 32) >> 4;
            umma_ss_elect(tmem + X * 128, dq[X] + qo, ks + ko, T::kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit_elect(&sm.s_full[X]);
          started[X] = true;
          return true;
        };
        bool pv_started[2] = {false, false};
        auto pv_op = [&](int X, int k) -> bool {  // O_X += P_X V(k), V(k) already waited on
          // P arrives in two halves (key columns [0, 64) and [64, 128)); the
          // first half's MMAs run while the softmax warps finish the second.
          if (!member(X, k)) return true;
          const uint64_t vs = dv + static_cast<uint64_t>(((base + 2 * k + 1) % kStages) * (T::kKVBytes >> 4));
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!wait(&sm.p_full[X][h], pn[X] & 1)) return false;
            tc_fence_after();
            constexpr int kPerHalf = T::kStepKeys / 2 / T::kPVK;
#pragma unroll
            for (int kk = h * kPerHalf; kk < (h + 1) * kPerHalf; ++kk) {
              // kk-th K slice of P: 8 TMEM columns (16 bf16 or 32 E4M3 keys); of V:
              // kPVK rows of 128 bytes
              const uint64_t bd = vs + static_cast<uint32_t>((kk * T::kPVK * 128) >> 4);
              if constexpr (F8)
                umma_ts_f8_elect(tmem + 256 + X * 128, tmem + X * 128 + kk * 8, bd, T::kIdescPV,
                                 (pv_started[X] || kk > 0) ? 1u : 0u);
              else
                umma_ts_elect(tmem + 256 + X * 128, tmem + X * 128 + kk * 8, bd, T::kIdescPV,
                              (pv_started[X] || kk > 0) ? 1u : 0u);
            }
          }
          ++pn[X];
          pv_started[X] = true;
          return true;
        };
        const bool two = x.slot[1];
        ok = kv_ready(base) && s_op(0, 0) && (!two || s_op(1, 0));
        if (ok) umma_commit_elect(&sm.kv_empty[base % kStages]);
        for (int k = 1; ok && k < cnt; ++k) {
          ok = kv_ready(base + 2 * k - 1) && pv_op(0, k - 1) && kv_ready(base + 2 * k) && s_op(0, k) &&
               (!two || pv_op(1, k - 1));
          if (!ok) break;
          umma_commit_elect(&sm.kv_empty[(base + 2 * k - 1) % kStages]);
          ok = !two || s_op(1, k);
          if (!ok) break;
          umma_commit_elect(&sm.kv_empty[(base + 2 * k) % kStages]);
        }
        if (ok) ok = kv_ready(base + 2 * cnt - 1) && pv_op(0, cnt - 1) && (!two || pv_op(1, cnt - 1));
        if (ok) umma_commit_elect(&sm.kv_empty[(base + 2 * cnt - 1) % kStages]);
        if (ok) {
          // Q and O of both slots are released once every MMA of the unit is done.
          // (A slot always has a member step: each query block selects at least one
          // key block. Should one have none, its Q phase is still consumed here.)
          for (int X = 0; X < (two ? 2 : 1); ++X) {
            if (!started[X]) {
              if (!wait(&sm.q_full[X], qn[X] & 1)) break;
              ++qn[X];
            }
            umma_commit_elect(&sm.q_empty[X]);
            umma_commit_elect(&sm.o_full[X]);
          }
        }
        base += 2 * cnt;
      }
      // Drain: every MMA this warp issued has completed before TMEM is freed.
      umma_commit_elect(&sm.mma_done);
      mbar_wait_plain(&sm.mma_done, 0);
    }
    teardown();
    return;
  }

  regs_inc<kRegsSoftmax>();
  {
    // ------------------------------------------------------------ softmax / epilogue
    constexpr int NC = T::kStepKeys / 32;   // 32-column chunks of S
    constexpr int BPS = T::kBPS;            // union entries per step
    constexpr int CPE = NC / BPS;           // chunks per entry
    const int X = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int qb = (X * 128 + row) / BN;  // query block of this row within the unit
    const uint32_t kSlotMask = ((1u << (T::kGroup / 2)) - 1u) << (X * (T::kGroup / 2));   // this slot's member bits
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + X * 128;
    const uint32_t tO = tmem + lane_off + 256 + X * 128;
    const int tail = P.N - (P.nb - 1) * BN;  // valid keys in the last block
    const float sl2 = P.scale_log2;
    int n = 0, sn = 0, on = 0;
#pragma unroll 1
    while (true) {
      const int b = n & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.unit_full[b], (n >> 1) & 1, abort_flag, P.status))) break;
      const int u = *reinterpret_cast<volatile int*>(&sm.unit_box[b]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.unit_empty[b]);
      ++n;
      const Unit x = decode_unit<BN>(u, P);
      if (x.cnt == 0) break;
      if (!(X == 0 ? x.slot[0] : x.slot[1])) continue;
      const int ns = (x.cnt + BPS - 1) / BPS;
      const int qrow = x.grp * kUnitRows + X * 128 + row;   // row within the head
      float m_run = -FLT_MAX;
      float l_run = 0.f;
      bool have = false;
      bool ok = true;
      // Entries of the next step, read ahead; past the list's end, 0 (no member).
      uint32_t e_next[BPS];
#pragma unroll
      for (int h = 0; h < BPS; ++h) e_next[h] = h < x.cnt ? entry_at<BN>(x, h, P) : 0u;
#pragma unroll 1
      for (int k = 0; k < ns; ++k) {
        uint32_t e[BPS];
        bool mem[BPS];
        bool any_mem = false;
        bool slot_mem = false;   // one of this slot's query blocks selected an entry of the step
#pragma unroll
        for (int h = 0; h < BPS; ++h) {
          e[h] = e_next[h];
          const int idx = BPS * (k + 1) + h;
          if (k + 1 < ns) e_next[h] = idx < x.cnt ? entry_at<BN>(x, idx, P) : 0u;
          mem[h] = (e[h] >> (16 + qb)) & 1u;     // warp-uniform: a warp's rows share qb
          any_mem |= mem[h];
          slot_mem |= ((e[h] >> 16) & kSlotMask) != 0u;
        }
        // With 64-token blocks the MMA warp computes neither S nor P.V for a step none
        // of the slot's query blocks selected (the same test on the same entries), so
        // there is nothing to wait for. slot_mem is warp-uniform (the entries are).
        if (BN == 64 && !slot_mem) continue;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[X], sn & 1, abort_flag, P.status))) { ok = false; break; }
        ++sn;
        tc_fence_after();
        // any_mem is warp-uniform: it depends only on the step's union entries
        // (the same for every lane) and on qb, which all 32 rows of a warp share
        // (32 divides BN). The S loads and P stores below therefore run on full warps.
        if (any_mem) {
          uint32_t s[NC][32];
#pragma unroll
          for (int c = 0; c < NC; ++c) tmem_ld32(tS + c * 32, s[c]);
          tmem_wait_ld();
          float mx = -FLT_MAX;
          if constexpr (BPS == 1) {
            // One block per step (the row attends it): only the keys past N of the
            // last block are masked.
#pragma unroll
            for (int c = 0; c < NC; ++c) {
              const int kbase = c * 32;
              if (static_cast<int>(e[0] & 0xFFFFu) == P.nb - 1 && tail < kbase + 32) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (kbase + i >= tail) s[c][i] = __float_as_uint(-INFINITY);
              }
            }
            // Row max: 8 independent chains of 3-input max (exact in any order).
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = -FLT_MAX;
#pragma unroll
            for (int c = 0; c < NC; ++c)
#pragma unroll
              for (int i = 0; i < 16; ++i)
                mx8[i & 7] = fmax3(mx8[i & 7], __uint_as_float(s[c][2 * i]), __uint_as_float(s[c][2 * i + 1]));
            mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
          } else {
            // Two 64-key entries per step. Keys this row does not attend:
            //  * the half whose entry the row's query block did not select (or the
            //    pad half of an odd step): it is left out of the row max below and
            //    gets an exponent offset of -inf, so its P is exactly 0;
            //  * the keys past N of the last block: set to -inf one by one. That is
            //    rare and warp-uniform, so it sits behind a vote; written inline,
            //    both maskings compile to selects over all 128 values on every step
            //    (about half again the instructions of a one-block step).
            bool tail_step = false;
#pragma unroll
            for (int h = 0; h < BPS; ++h)
              tail_step |= mem[h] && static_cast<int>(e[h] & 0xFFFFu) == P.nb - 1 && tail < BN;
            if (__any_sync(0xffffffffu, tail_step)) {
#pragma unroll
              for (int c = 0; c < NC; ++c) {
                const int h = c / CPE;
                const int kbase = (c % CPE) * 32;   // first key of the chunk within its block
                const int v = static_cast<int>(e[h] & 0xFFFFu) == P.nb - 1 ? tail - kbase : 32;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (i >= v) s[c][i] = __float_as_uint(-INFINITY);
              }
            }
            // Row max over the attended halves: per half, 8/BPS independent chains
            // of 3-input max (exact in any order).
            constexpr int kChains = 8 / BPS;
#pragma unroll
            for (int h = 0; h < BPS; ++h) {
              float mc[kChains];
#pragma unroll
              for (int i = 0; i < kChains; ++i) mc[i] = -FLT_MAX;
#pragma unroll
              for (int c = h * CPE; c < (h + 1) * CPE; ++c)
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  mc[i % kChains] = fmax3(mc[i % kChains], __uint_as_float(s[c][2 * i]),
                                          __uint_as_float(s[c][2 * i + 1]));
              float mh = mc[0];
#pragma unroll
              for (int i = 1; i < kChains; ++i) mh = fmaxf(mh, mc[i]);
              if (mem[h]) mx = fmaxf(mx, mh);
            }
          }
          const float m_new = mx * sl2;
          if (!have) {
            m_run = m_new;
            have = true;
          } else {
            // The decision is per row but tcgen05.ld/st are warp-collective: when
            // any row of the warp needs a larger max, the whole warp rescales,
            // rows that do not need it with factor 1.
            const bool need = m_new > m_run + T::kThreshold;
            if (__any_sync(0xffffffffu, need)) {   // vote: the O load/store below is warp-uniform
              const float f = need ? ex2_approx(m_run - m_new) : 1.f;
              l_run *= f;
#pragma unroll 1
              for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                tmem_st32(tO + c * 32, o);
              }
              tmem_wait_st();
              if (need) m_run = m_new;
            }
          }
          // x = s * scale*log2(e) - m and the row sums in packed fp32x2 arithmetic.
          // Each half of P is published as soon as it is in TMEM.
          const float2 sl2x2 = make_float2(sl2, sl2);
          const float m_eff = m_run - T::kPShift;
          const float2 negm = make_float2(-m_eff, -m_eff);
          float2 lc[NC];
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            uint32_t pk[16];
            float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            // a half the row does not attend (two entries per step): every x = -inf, so P = 0
            const float2 negc =
                (BPS == 1 || mem[c / CPE]) ? negm : make_float2(-INFINITY, -INFINITY);
            __half2 hs[2] = {__float2half2_rn(0.f), __float2half2_rn(0.f)};
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 xv = __ffma2_rn(
                  make_float2(__uint_as_float(s[c][2 * i]), __uint_as_float(s[c][2 * i + 1])), sl2x2, negc);
              const float p0 = ex2_approx(xv.x);
              const float p1 = ex2_approx(xv.y);
              if constexpr (F8) {
                // four keys per 32-bit word, lowest key in the low byte
                const uint32_t q8 = pack_e4m3x2(p0, p1);
                hs[i & 1] = __hadd2(hs[i & 1], e4m3x2_to_half2(q8));
                pk[i >> 1] = (i & 1) ? (pk[i >> 1] | (q8 << 16)) : q8;
              } else {
                ls[i & 1] = __fadd2_rn(ls[i & 1], make_float2(p0, p1));
                pk[i] = pack_bf16x2(p0, p1);
              }
            }
            if constexpr (F8) {
              lc[c] = __half22float2(__hadd2(hs[0], hs[1]));
              tmem_st8(tS + c * 8, reinterpret_cast<const uint32_t(&)[8]>(pk));
            } else {
              lc[c] = __fadd2_rn(ls[0], ls[1]);
              tmem_st16(tS + c * 16, pk);
            }
            if (c == NC / 2 - 1 || c == NC - 1) {   // c is a compile-time loop index: uniform
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.p_full[X][c == NC - 1 ? 1 : 0]);
            }
          }
#pragma unroll
          for (int h = 0; h < BPS; ++h) {
            float l_blk = 0.f;
#pragma unroll
            for (int c = h * CPE; c < (h + 1) * CPE; ++c) l_blk += lc[c].x + lc[c].y;
            l_run += l_blk;
            // Block log-sum-exp of this row over this key block [GSRS §5.3]: the
            // exponentials are relative to m_run, so it is m_run + log2 of their
            // sum, converted to the natural base.
            if (P.blse && mem[h] && qrow < P.npad)
              P.blse[(static_cast<size_t>(x.bh) * P.nb + (e[h] & 0xFFFFu)) * P.npad + qrow] =
                  (m_eff + __log2f(l_blk)) * kLn2;
          }
        } else {   // the same warp-uniform condition, negated: P = 0 for the whole step
          uint32_t z[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
          for (int c = 0; c < T::kPCols / 16; ++c) tmem_st16(tS + c * 16, z);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&sm.p_full[X][0]);
            mbar_arrive(&sm.p_full[X][1]);
          }
        }
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[X], on & 1, abort_flag, P.status))) break;
      ++on;
      tc_fence_after();
      // Rows past the head's last block (the second half of a 64-token-block
      // tile at the end of a head) are not stored; the TMEM loads stay
      // warp-collective (the loop runs for every lane; `store` only guards the
      // global stores). Every exit above is a warp-wide vote (__all_sync) or a
      // value read from shared memory by all lanes (the unit, its slots).
      const bool store = qrow < P.npad;
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const float* vs = F8 ? P.vscale + static_cast<size_t>(x.bh) * HD : nullptr;
      const size_t grow = static_cast<size_t>(x.bh) * P.npad + qrow;
      uint4* orow = reinterpret_cast<uint4*>(P.out + grow * HD);
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        uint32_t w[16];
        if constexpr (F8) {
          // O of the codes, times 1/l and each channel's scale
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 sc = __ldg(reinterpret_cast<const float4*>(vs + c * 32) + i);
            w[2 * i] = pack_bf16x2(__uint_as_float(o[4 * i]) * (inv_l * sc.x),
                                   __uint_as_float(o[4 * i + 1]) * (inv_l * sc.y));
            w[2 * i + 1] = pack_bf16x2(__uint_as_float(o[4 * i + 2]) * (inv_l * sc.z),
                                       __uint_as_float(o[4 * i + 3]) * (inv_l * sc.w));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        }
        if (!(l_run > 0.f)) {   // a row no processed step reached: O was never written
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = 0u;
        }
        if (store) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            orow[c * 4 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (store && P.lse) P.lse[grow] = (m_run - T::kPShift + __log2f(l_run)) * kLn2;
      tc_fence_before();
    }
  }
  teardown();
}

}  // namespace sm100

// ---------------------------------------------------------------- work order
// plan_union_kernel: per (b, h) and group of G consecutive query blocks, the
// ascending union of their KV lists with one membership bit per query block
// (bitmaps in shared memory; out-of-range entries are dropped and recorded).
template <int G>
__global__ void __launch_bounds__(256)
    plan_union_kernel(const int* __restrict__ kv_idx, const int* __restrict__ kv_cnt, int nb,
                      int ngroups, uint32_t* __restrict__ ulist, int* __restrict__ ucnt,
                      int* status) {
  __shared__ uint32_t bm[G][128];
  __shared__ int base[129];
  const int grp = blockIdx.x;
  const int bh = blockIdx.y;
  const int nwords = (nb + 31) >> 5;
  for (int t = threadIdx.x; t < G * 128; t += blockDim.x) bm[t / 128][t % 128] = 0u;
  __syncthreads();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int i = grp * G + g;
    if (i >= nb) break;
    const size_t row = static_cast<size_t>(bh) * nb + i;
    int c = kv_cnt[row];
    if (c < 1 || c > nb) {
      if (threadIdx.x == 0) record_status(status, FVATTN_ERR_INVALID_ARG);
      c = min(max(c, 1), nb);
    }
    for (int t = threadIdx.x; t < c; t += blockDim.x) {
      const int j = kv_idx[row * nb + t];
      if (j >= 0 && j < nb) atomicOr(&bm[g][j >> 5], 1u << (j & 31));
      else record_status(status, FVATTN_ERR_INVALID_ARG);
    }
  }
  __syncthreads();
  if (threadIdx.x < nwords) {
    uint32_t m = 0u;
#pragma unroll
    for (int g = 0; g < G; ++g) m |= bm[g][threadIdx.x];
    base[threadIdx.x + 1] = __popc(m);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    base[0] = 0;
    for (int w = 1; w <= nwords; ++w) base[w] += base[w - 1];
    ucnt[static_cast<size_t>(bh) * ngroups + grp] = base[nwords];
  }
  __syncthreads();
  if (threadIdx.x < nwords) {
    const int w = threadIdx.x;
    uint32_t m = 0u;
#pragma unroll
    for (int g = 0; g < G; ++g) m |= bm[g][w];
    uint32_t* out = ulist + (static_cast<size_t>(bh) * ngroups + grp) * nb + base[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1u;
      uint32_t members = 0u;
#pragma unroll
      for (int g = 0; g < G; ++g) members |= ((bm[g][w] >> bit) & 1u) << g;
      *out++ = static_cast<uint32_t>(w * 32 + bit) | (members << 16);
    }
  }
}

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

// Within each head: units by descending union length (ties: lower index); the head's total.
__global__ void __launch_bounds__(1024)
    plan_heads_kernel(const int* __restrict__ ucnt, int ngroups, int* __restrict__ local_order,
                      unsigned long long* __restrict__ head_total) {
  __shared__ uint32_t keys[4096];
  __shared__ unsigned long long red[32];
  const int bh = blockIdx.x;
  int n2 = 1;
  while (n2 < ngroups) n2 <<= 1;
  unsigned long long part = 0;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    if (i < ngroups) {
      const int c = ucnt[static_cast<size_t>(bh) * ngroups + i];
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
    for (int w = 0; w < static_cast<int>(blockDim.x + 31) / 32; ++w) t += red[w];
    head_total[bh] = t;
  }
  for (int r = threadIdx.x; r < ngroups; r += blockDim.x)
    local_order[static_cast<size_t>(bh) * ngroups + r] = 0xFFFF - static_cast<int>(keys[r] & 0xFFFFu);
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
template <int BN, bool F8, int HD>
static cudaError_t launch_bn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const sm100::Params& P, int num_sms, cudaStream_t st) {
  const size_t smem = sizeof(sm100::Smem<BN, HD>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(sm100::attn_fwd_sm100_kernel<BN, F8, HD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = max(1, min(num_sms, P.total_units));
  sm100::attn_fwd_sm100_kernel<BN, F8, HD><<<grid, sm100::kThreads, smem, st>>>(tq, tk, tv, P);
  return cudaGetLastError();
}

cudaError_t launch_attn_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              void* out, float* lse, float* blse, const float* vscale,
                              const int* kv_idx, const int* kv_cnt,
                              uint32_t* ulist, int* ucnt, int* local_order,
                              unsigned long long* head_total, int* head_order, int BH, int N,
                              int nb, int bs, int d, float scale, int* status,
                              unsigned long long* counter, int num_sms, cudaStream_t st) {
  const int G = sm100::kUnitRows / bs;
  const int ngroups = (nb + G - 1) / G;
  if (kv_idx) {
    const dim3 g1(ngroups, BH);
    if (G == 2)
      plan_union_kernel<2><<<g1, 256, 0, st>>>(kv_idx, kv_cnt, nb, ngroups, ulist, ucnt, status);
    else
      plan_union_kernel<4><<<g1, 256, 0, st>>>(kv_idx, kv_cnt, nb, ngroups, ulist, ucnt, status);
    plan_heads_kernel<<<BH, 1024, 0, st>>>(ucnt, ngroups, local_order, head_total);
    plan_rank_kernel<<<1, 1024, 0, st>>>(head_total, BH, head_order);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sm100::Params P;
  P.nb = nb;
  P.N = N;
  P.npad = nb * bs;
  P.ngroups = ngroups;
  P.total_units = BH * ngroups;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.ulist = kv_idx ? ulist : nullptr;
  P.ucnt = ucnt;
  P.head_order = head_order;
  P.local_order = local_order;
  P.out = static_cast<__nv_bfloat16*>(out);
  P.lse = lse;
  P.blse = blse;
  P.vscale = vscale;
  P.status = status;
  P.counter = counter;
  if (vscale)
    return bs == 64 ? launch_bn<64, true, 128>(tq, tk, tv, P, num_sms, st)
                    : launch_bn<128, true, 128>(tq, tk, tv, P, num_sms, st);
  if (d == 64)
    return bs == 64 ? launch_bn<64, false, 64>(tq, tk, tv, P, num_sms, st)
                    : launch_bn<128, false, 64>(tq, tk, tv, P, num_sms, st);
  return bs == 64 ? launch_bn<64, false, 128>(tq, tk, tv, P, num_sms, st)
                  : launch_bn<128, false, 128>(tq, tk, tv, P, num_sms, st);
}

}  // namespace fvattn
