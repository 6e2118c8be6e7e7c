// lvsa.cu -- KV block lists of the LVSA static pattern: a local temporal window
// plus rotating equidistant global frames, lifted to blocks of the permuted
// token sequence.
//
// [LVSA §3, attention pattern]  query frame t attends A(t) = G ∪ W(t); G holds
//   one frame every Tper frames, W(t) up to 2W+1 neighbouring frames, clipped
//   at the ends of the video.
// [LVSA §3, budget allocation]  the window is expanded to make up for clipping
//   and for overlap with G, so every frame attends |G| + min(2W+1, T-|G|) frames.
// [LVSA §3, rotating global frames]  at denoising step s, G is shifted by s
//   modulo Tper.
//
// Readings: G_s = { g : g = s (mod Tper) }. Each expansion pass adds exactly the
// current deficit to the window, ceil(deficit/2) frames after t and the rest
// before t, a clipped side handing its share to the other side; passes repeat
// while added frames fall on global frames. Key block j is attended by query
// block i when a valid token of i lies in a frame tq and a valid token of j in
// a frame of A(tq). The pattern is the same for every (b, h); the lists are
// written for every head so that fvattn_sparse_fwd consumes them unchanged.
//
// block_frames_kernel: one CTA per block, the bitmask of the frames its valid
// tokens lie in (at most 1024 frames, 32 words), through the same source map
// (tiles or an explicit order table) as the permutation kernels.
// lvsa_lists_kernel: one CTA per query block: the union of A(tq) over its frames
// as a frame bitmask, then every key block whose frames meet it, in ascending
// order (block-wide ballot scan), copied to all B*H rows.
#include "common.cuh"

namespace fvattn {

constexpr int kLvsaThreads = 256;
constexpr int kLvsaWords = 32;        // frame bitmask words: T <= 1024

__device__ __forceinline__ int floor_div(int a, int b) {   // b > 0
  const int q = a / b;
  return (a % b != 0 && a < 0) ? q - 1 : q;
}

// |G_s ∩ [lo, hi]| for G_s = { g in Z : g = r (mod per) }.
__device__ __forceinline__ int globals_in(int lo, int hi, int r, int per) {
  if (hi < lo) return 0;
  return floor_div(hi - r, per) - floor_div(lo - 1 - r, per);
}

__global__ void __launch_bounds__(kLvsaThreads)
    block_frames_kernel(TileGeom g, int N, int bs, int words, uint32_t* __restrict__ frames) {
  __shared__ uint32_t m[kLvsaWords];
  const int i = blockIdx.x;
  if (threadIdx.x < kLvsaWords) m[threadIdx.x] = 0u;
  __syncthreads();
  const int plane = g.Hh * g.W;
  const int end = min((i + 1) * bs, N);
  for (int pos = i * bs + threadIdx.x; pos < end; pos += blockDim.x) {
    const int src = source_index(pos, N, g);
    if (src < 0) continue;
    const int t = src / plane;
    atomicOr(&m[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  if (threadIdx.x < words) frames[static_cast<size_t>(i) * kLvsaWords + threadIdx.x] = m[threadIdx.x];
}

__global__ void __launch_bounds__(kLvsaThreads)
    lvsa_lists_kernel(const uint32_t* __restrict__ frames, int T, int nb, int words, int window,
                      int per, int r, int BH, int* __restrict__ kv_idx, int* __restrict__ kv_cnt,
                      unsigned long long* __restrict__ head_work) {
  __shared__ uint32_t fi[kLvsaWords];      // frames of this query block
  __shared__ uint32_t allowed[kLvsaWords]; // key frames attended by some frame of it
  __shared__ int warp_cnt[kLvsaThreads / 32];
  __shared__ int total;
  extern __shared__ int list[];            // nb entries: this row's list
  const int i = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < kLvsaWords) {
    fi[threadIdx.x] = threadIdx.x < words ? frames[static_cast<size_t>(i) * kLvsaWords + threadIdx.x] : 0u;
    // G_s bits of this word
    uint32_t gbits = 0u;
    for (int b = 0; b < 32; ++b) {
      const int t = threadIdx.x * 32 + b;
      if (t < T && (t - r) % per == 0 && t >= r) gbits |= 1u << b;
    }
    allowed[threadIdx.x] = gbits;
  }
  if (threadIdx.x == 0) total = 0;
  __syncthreads();
  const int n_glob = globals_in(0, T - 1, r, per);
  const int target = n_glob + min(2 * window + 1, T - n_glob);
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    if (!((fi[t >> 5] >> (t & 31)) & 1u)) continue;
    int lo = max(0, t - window), hi = min(T - 1, t + window);
    for (int pass = 0; pass <= T; ++pass) {       // at most T passes: each adds >= 1 frame
      const int count = (hi - lo + 1) + n_glob - globals_in(lo, hi, r, per);
      const int deficit = target - count;
      if (deficit <= 0) break;
      int right = min(T - 1 - hi, (deficit + 1) / 2);
      const int left = min(lo, deficit - right);
      right = min(T - 1 - hi, deficit - left);
      if (left == 0 && right == 0) break;
      lo -= left;
      hi += right;
    }
    for (int w = lo >> 5; w <= (hi >> 5); ++w) {
      const int a = max(lo, w * 32) - w * 32, b = min(hi, w * 32 + 31) - w * 32;
      const uint32_t bits = (b == 31 ? 0xFFFFFFFFu : ((1u << (b + 1)) - 1u)) & ~((1u << a) - 1u);
      atomicOr(&allowed[w], bits);
    }
  }
  __syncthreads();
  // Ascending compaction of the attended key blocks, 256 candidates per round.
  for (int j0 = 0; j0 < nb; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    bool sel = false;
    if (j < nb) {
      const uint32_t* fj = frames + static_cast<size_t>(j) * kLvsaWords;
      for (int w = 0; w < words; ++w) sel |= (fj[w] & allowed[w]) != 0u;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = total;
    for (int w = 0; w < warp; ++w) before += warp_cnt[w];
    if (sel) list[before + __popc(bal & ((1u << lane) - 1u))] = j;
    __syncthreads();
    if (threadIdx.x == 0) {
      int add = 0;
      for (int w = 0; w < kLvsaThreads / 32; ++w) add += warp_cnt[w];
      total += add;
    }
    __syncthreads();
  }
  const int cnt = total;
  for (int bh = 0; bh < BH; ++bh) {
    int* row = kv_idx + (static_cast<size_t>(bh) * nb + i) * nb;
    for (int t = threadIdx.x; t < cnt; t += blockDim.x) row[t] = list[t];
  }
  for (int bh = threadIdx.x; bh < BH; bh += blockDim.x) {
    kv_cnt[static_cast<size_t>(bh) * nb + i] = cnt;
    atomicAdd(head_work + bh, static_cast<unsigned long long>(cnt));
  }
}

cudaError_t launch_lvsa_lists(const TileGeom& g, int N, int bs, int window, int per, int step,
                              int BH, int* kv_idx, int* kv_cnt, unsigned long long* head_work,
                              uint32_t* frames, cudaStream_t st) {
  const int nb = (N + bs - 1) / bs;
  const int words = (g.T + 31) / 32;
  const int r = ((step % per) + per) % per;
  block_frames_kernel<<<nb, kLvsaThreads, 0, st>>>(g, N, bs, words, frames);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = static_cast<size_t>(nb) * sizeof(int);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(lvsa_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  lvsa_lists_kernel<<<nb, kLvsaThreads, smem, st>>>(frames, g.T, nb, words, window, per, r, BH,
                                                     kv_idx, kv_cnt, head_work);
  return cudaGetLastError();
}

}  // namespace fvattn
