// common.cuh -- shared definitions of the fvattn CUDA library: status codes,
// workspace header, the closed-form 3-D tile index map, small helpers.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/fvattn.h"

namespace fvattn {

// First 256 bytes of every workspace.
struct WsHeader {
  int status;                  // first error recorded by a kernel (0 = none)
  int pad0;
  unsigned long long counter;  // dynamic work-unit counter of the attention scheduler
  unsigned long long pad[30];
};
static_assert(sizeof(WsHeader) == 256, "workspace header must be 256 bytes");
constexpr size_t kWsHeaderBytes = 256;

__host__ __device__ __forceinline__ size_t align_up(size_t v, size_t a) {
  return (v + a - 1) / a * a;
}

// Latent video grid with 3-D tiles [FVAttn §3.1 video-aware block organisation,
// read as 3-D tiles]. Tiles are visited in raster order over the tile grid and
// tokens in raster order inside a tile; the last tile along an axis may be
// partial. Because only the last tile of each axis is short, the offset of a
// tile has a closed form and so does the inverse map used here.
struct TileGeom {
  int T, Hh, W, tt, th, tw;
  const int* table;   // non-null: explicit order (table[pos] = raster index), e.g. Hilbert
};

// Original token index n = (t*Hh + y)*W + x of the token at permuted position pos.
__host__ __device__ __forceinline__ int tile_source_index(int pos, const TileGeom& g) {
  const int slab = g.tt * g.Hh * g.W;              // tokens in a full slab of tiles
  const int ti = pos / slab;
  const int r1 = pos - ti * slab;
  const int st = min(g.tt, g.T - ti * g.tt);       // frames in this slab
  const int row = st * g.th * g.W;                 // tokens in a full row of tiles
  const int yi = r1 / row;
  const int r2 = r1 - yi * row;
  const int sy = min(g.th, g.Hh - yi * g.th);      // rows in this row of tiles
  const int full_tile = st * sy * g.tw;
  const int xi = r2 / full_tile;
  const int r3 = r2 - xi * full_tile;
  const int sx = min(g.tw, g.W - xi * g.tw);       // columns in this tile
  const int plane = sy * sx;
  const int dt = r3 / plane;
  const int rem = r3 - dt * plane;
  const int dy = rem / sx;
  const int dx = rem - dy * sx;
  return ((ti * g.tt + dt) * g.Hh + (yi * g.th + dy)) * g.W + (xi * g.tw + dx);
}

// Source row of permuted position pos (< N): the explicit table when there is
// one, else the tile map. A table entry outside [0, N) gives -1 (row skipped).
__device__ __forceinline__ int source_index(int pos, int N, const TileGeom& g) {
  if (!g.table) return tile_source_index(pos, g);
  const int s = __ldg(g.table + pos);
  return (s >= 0 && s < N) ? s : -1;
}

__device__ __forceinline__ void record_status(int* status_word, int code) {
  if (status_word) atomicCAS(status_word, 0, code);
}

}  // namespace fvattn
