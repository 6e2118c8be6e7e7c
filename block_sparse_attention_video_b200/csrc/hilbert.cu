// hilbert.cu -- the Hilbert-curve token order of a latent video grid, as an
// explicit permutation table for the block-order kernels.
//
// [FVAttn §3.1]  blocks are reordered along a Hilbert curve so that spatial
//   neighbours fall into nearby blocks at every scale. [GSRS §A.6]  a generalized
//   Hilbert curve groups nearby spatio-temporal tokens into compact blocks.
// Reading: tokens are ordered by their index on the 3-D Hilbert curve over
// (t, y, x) of the smallest cube of side 2^b holding the grid (b = bits of the
// largest extent); on the grid this is the cube's curve restricted to the grid.
//
// The index follows J. Skilling, "Programming the Hilbert curve" (AIP Conf.
// Proc. 707, 2004): an in-place transform of the coordinates (undo the excess
// work of the recursion from the top bit down, then Gray-encode) whose bits,
// interleaved from the top with axis 0 first, are the index.
//
// Construction (once per grid): every token gets the 64-bit key
// (index << nbits) | raster index, nbits = bits of N; keys are distinct, so an
// unstable sort is exact. A bitonic network over the next power of two (one
// launch per stage, pad keys = all ones) sorts them, and the table takes the
// low nbits of each sorted key. Keys need 3b + nbits <= 64 bits.
#include "common.cuh"

namespace fvattn {

constexpr int kHilbertThreads = 256;

__device__ __forceinline__ unsigned long long hilbert_key3(uint32_t t, uint32_t y, uint32_t x, int b) {
  uint32_t X[3] = {t, y, x};
  const uint32_t M = 1u << (b - 1);
  for (uint32_t Q = M; Q > 1; Q >>= 1) {
    const uint32_t P = Q - 1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (X[i] & Q) {
        X[0] ^= P;
      } else {
        const uint32_t s = (X[0] ^ X[i]) & P;
        X[0] ^= s;
        X[i] ^= s;
      }
    }
  }
  X[1] ^= X[0];
  X[2] ^= X[1];
  uint32_t flip = 0;
  for (uint32_t Q = M; Q > 1; Q >>= 1)
    if (X[2] & Q) flip ^= Q - 1;
  X[0] ^= flip;
  X[1] ^= flip;
  X[2] ^= flip;
  unsigned long long h = 0;
  for (int q = b - 1; q >= 0; --q) {
#pragma unroll
    for (int i = 0; i < 3; ++i) h = (h << 1) | ((X[i] >> q) & 1u);
  }
  return h;
}

__global__ void __launch_bounds__(kHilbertThreads)
    hilbert_keys_kernel(int T, int Hh, int W, int b, int nbits, int n2,
                        unsigned long long* __restrict__ keys) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n2) return;
  const int N = T * Hh * W;
  if (idx >= N) {
    keys[idx] = ~0ull;
    return;
  }
  const int x = idx % W;
  const int y = (idx / W) % Hh;
  const int t = idx / (W * Hh);
  keys[idx] = (hilbert_key3(t, y, x, b) << nbits) | static_cast<unsigned long long>(idx);
}

// One compare-exchange stage of an ascending bitonic sort.
__global__ void __launch_bounds__(kHilbertThreads)
    bitonic_stage_kernel(unsigned long long* __restrict__ a, int n2, int j, int k) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n2) return;
  const int l = i ^ j;
  if (l <= i) return;
  const bool up = (i & k) == 0;
  const unsigned long long x = a[i], y = a[l];
  if ((x > y) == up) {
    a[i] = y;
    a[l] = x;
  }
}

__global__ void __launch_bounds__(kHilbertThreads)
    hilbert_table_kernel(const unsigned long long* __restrict__ keys, int N, int nbits,
                         int* __restrict__ table) {
  const int pos = blockIdx.x * blockDim.x + threadIdx.x;
  if (pos < N) table[pos] = static_cast<int>(keys[pos] & ((1ull << nbits) - 1ull));
}

int hilbert_bits(int extent) {
  int b = 1;
  while ((1 << b) < extent) ++b;
  return b;
}

int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

cudaError_t launch_hilbert_table(int T, int Hh, int W, int* table, unsigned long long* keys,
                                 cudaStream_t st) {
  const int N = T * Hh * W;
  const int b = hilbert_bits(max(T, max(Hh, W)));
  const int nbits = hilbert_bits(N);
  const int n2 = next_pow2(N);
  const int grid = (n2 + kHilbertThreads - 1) / kHilbertThreads;
  hilbert_keys_kernel<<<grid, kHilbertThreads, 0, st>>>(T, Hh, W, b, nbits, n2, keys);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      bitonic_stage_kernel<<<grid, kHilbertThreads, 0, st>>>(keys, n2, j, k);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  hilbert_table_kernel<<<(N + kHilbertThreads - 1) / kHilbertThreads, kHilbertThreads, 0, st>>>(
      keys, N, nbits, table);
  return cudaGetLastError();
}

}  // namespace fvattn
