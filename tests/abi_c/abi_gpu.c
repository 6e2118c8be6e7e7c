/* A plain C99 program that runs the whole path through the C ABI on the GPU
 * with device memory from cudaMalloc (no Python): route, V permutation,
 * block-sparse attention and the inverse permutation on a small grid. With
 * p = 1 every block is selected [FVAttn §2.1: Top-p keeps the blocks whose
 * cumulative score reaches p], so the sparse output must equal the dense
 * kernel's bit for bit; the lists must hold every block in ascending order. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "fvattn.h"

#define CK(x)                                                                       \
  do {                                                                              \
    if ((x) != cudaSuccess) { fprintf(stderr, "cuda error line %d\n", __LINE__); return 2; } \
  } while (0)
#define FV(x)                                                                       \
  do {                                                                              \
    fvattn_status s_ = (x);                                                         \
    if (s_ != FVATTN_OK) {                                                          \
      fprintf(stderr, "%s: %s (line %d)\n", #x, fvattn_status_string(s_), __LINE__); \
      return 3;                                                                     \
    }                                                                               \
  } while (0)

static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u); /* round to nearest even */
  return (uint16_t)(u >> 16);
}

static float from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static void* dalloc(size_t n) {
  void* p = NULL;
  if (cudaMalloc(&p, n < 256 ? 256 : n) != cudaSuccess) return NULL;
  return p;
}

int main(void) {
  const int B = 1, H = 2, d = 128, block = 128;
  fvattn_grid g;
  memset(&g, 0, sizeof g);
  g.T = 2; g.Hh = 16; g.W = 20; g.tt = 2; g.th = 8; g.tw = 8; g.block = block;
  g.order = FVATTN_ORDER_TILES;
  const int N = g.T * g.Hh * g.W, nb = (N + block - 1) / block, npad = nb * block;
  const size_t elems = (size_t)B * H * N * d, pelems = (size_t)B * H * npad * d;

  /* deterministic inputs: a 32-bit LCG mapped to [-2, 2) */
  uint16_t* h = (uint16_t*)malloc(3 * elems * 2);
  uint32_t state = 12345u;
  size_t i;
  for (i = 0; i < 3 * elems; ++i) {
    state = state * 1664525u + 1013904223u;
    h[i] = to_bf16(((float)(state >> 8) / 16777216.0f) * 4.0f - 2.0f);
  }
  void *q = dalloc(elems * 2), *k = dalloc(elems * 2), *v = dalloc(elems * 2);
  void *qp = dalloc(pelems * 2), *kp = dalloc(pelems * 2), *vp = dalloc(pelems * 2);
  void *ops = dalloc(pelems * 2), *opd = dalloc(pelems * 2), *out = dalloc(elems * 2);
  int32_t* idx = (int32_t*)dalloc((size_t)B * H * nb * nb * 4);
  int32_t* cnt = (int32_t*)dalloc((size_t)B * H * nb * 4);
  int64_t* hw = (int64_t*)dalloc((size_t)B * H * 8);
  size_t wr = fvattn_workspace_bytes(FVATTN_OP_ROUTE, B, H, N, d, block);
  size_t wa = fvattn_workspace_bytes(FVATTN_OP_SPARSE_FWD, B, H, N, d, block);
  void *wsr = dalloc(wr), *wsa = dalloc(wa);
  if (!q || !k || !v || !qp || !kp || !vp || !ops || !opd || !out || !idx || !cnt || !hw || !wsr || !wsa) {
    fprintf(stderr, "cudaMalloc failed\n");
    return 2;
  }
  CK(cudaMemcpy(q, h, elems * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(k, h + elems, elems * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(v, h + 2 * elems, elems * 2, cudaMemcpyHostToDevice));

  const float scale = 1.0f / sqrtf((float)d);
  FV(fvattn_route(q, k, B, H, N, d, FVATTN_BF16, &g, 1.0f, 1, qp, kp, idx, cnt, hw, wsr, wr, NULL));
  FV(fvattn_permute(v, vp, B, H, N, d, FVATTN_BF16, &g, 0, NULL));
  FV(fvattn_sparse_fwd(qp, kp, vp, ops, NULL, NULL, idx, cnt, B, H, N, d, FVATTN_BF16, block, scale, wsa,
                       wa, NULL));
  FV(fvattn_workspace_status(wsa, NULL));
  FV(fvattn_dense_fwd(qp, kp, vp, opd, NULL, NULL, B, H, N, d, FVATTN_BF16, block, scale, wsa, wa, NULL));
  FV(fvattn_workspace_status(wsa, NULL));
  FV(fvattn_permute(ops, out, B, H, N, d, FVATTN_BF16, &g, 1, NULL));
  FV(fvattn_workspace_status(wsr, NULL));
  CK(cudaDeviceSynchronize());

  /* lists: every block, ascending; work = nb * nb per head */
  int32_t* hidx = (int32_t*)malloc((size_t)B * H * nb * nb * 4);
  int32_t* hcnt = (int32_t*)malloc((size_t)B * H * nb * 4);
  int64_t hhw[2];
  CK(cudaMemcpy(hidx, idx, (size_t)B * H * nb * nb * 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hcnt, cnt, (size_t)B * H * nb * 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hhw, hw, sizeof hhw, cudaMemcpyDeviceToHost));
  int r, j;
  for (r = 0; r < B * H * nb; ++r) {
    if (hcnt[r] != nb) { fprintf(stderr, "row %d count %d\n", r, hcnt[r]); return 4; }
    for (j = 0; j < nb; ++j)
      if (hidx[(size_t)r * nb + j] != j) { fprintf(stderr, "row %d entry %d\n", r, j); return 4; }
  }
  for (r = 0; r < B * H; ++r)
    if (hhw[r] != (int64_t)nb * nb) { fprintf(stderr, "head work %d\n", r); return 4; }

  /* sparse with every block == dense, bit for bit, on the valid rows */
  uint16_t* hs = (uint16_t*)malloc(pelems * 2);
  uint16_t* hd = (uint16_t*)malloc(pelems * 2);
  uint16_t* ho = (uint16_t*)malloc(elems * 2);
  CK(cudaMemcpy(hs, ops, pelems * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hd, opd, pelems * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(ho, out, elems * 2, cudaMemcpyDeviceToHost));
  size_t bh, row;
  double amax = 0.0;
  for (bh = 0; bh < (size_t)B * H; ++bh)
    for (row = 0; row < (size_t)N; ++row)
      for (j = 0; j < d; ++j) {
        size_t at = (bh * npad + row) * d + j;
        if (hs[at] != hd[at]) { fprintf(stderr, "sparse != dense at %zu\n", at); return 5; }
        float f = from_bf16(hs[at]);
        if (!isfinite(f)) { fprintf(stderr, "non-finite output\n"); return 5; }
        if (fabs(f) > amax) amax = fabs(f);
      }
  /* an output is a convex combination of V rows: |o| <= max |v| = 2 */
  if (amax > 2.0) { fprintf(stderr, "output outside the range of V: %f\n", amax); return 6; }
  for (i = 0; i < elems; ++i)
    if (!isfinite(from_bf16(ho[i]))) { fprintf(stderr, "non-finite after inverse\n"); return 7; }
  printf("abi_gpu ok: N %d, nb %d, max |o| %.4f\n", N, nb, amax);
  return 0;
}
