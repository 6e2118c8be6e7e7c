/* A plain C99 consumer of libfvattn.so: it includes only include/fvattn.h and
 * calls the entry points that need no GPU (workspace sizing, status strings
 * and the host-side argument checks that reject a call before any launch). */
#include <stdio.h>
#include <string.h>

#include "fvattn.h"

#define CHECK(cond, code)                                   \
  do {                                                      \
    if (!(cond)) {                                          \
      fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
      return (code);                                        \
    }                                                       \
  } while (0)

int main(void) {
  /* Wan-14B 720p shape: B 1, H 40, N 75,600, d 128, blocks of 128 */
  const int B = 1, H = 40, N = 21 * 45 * 80, d = 128, block = 128;
  int op;
  for (op = FVATTN_OP_ROUTE; op <= FVATTN_OP_QUANT_V; ++op) {
    size_t n = fvattn_workspace_bytes((fvattn_op)op, B, H, N, d, block);
    CHECK(n >= 256 && n % 256 == 0, 10 + op);
    printf("workspace op %d: %zu bytes\n", op, n);
  }
  CHECK(fvattn_workspace_bytes(FVATTN_OP_ROUTE, B, H, 0, d, block) == 0, 20);
  CHECK(fvattn_workspace_bytes(FVATTN_OP_ROUTE, B, H, N, 96, block) == 0, 21);
  CHECK(fvattn_workspace_bytes(FVATTN_OP_SPARSE_FWD, B, H, N, d, 100) == 0, 22);

  {
    fvattn_grid g;
    fvattn_status st;
    memset(&g, 0, sizeof g);
    g.T = 21; g.Hh = 45; g.W = 80; g.tt = 2; g.th = 8; g.tw = 8; g.block = block;
    g.order = FVATTN_ORDER_TILES; g.table = NULL;
    /* null tensors */
    st = fvattn_permute(NULL, NULL, B, H, N, d, FVATTN_BF16, &g, 0, NULL);
    CHECK(st == FVATTN_ERR_INVALID_ARG, 30);
    /* grid that does not match N */
    g.W = 81;
    st = fvattn_permute((const void*)0x100000, (void*)0x200000, B, H, N, d, FVATTN_BF16, &g, 0, NULL);
    CHECK(st == FVATTN_ERR_INVALID_ARG, 31);
    g.W = 80;
    /* p outside (0, 1] */
    st = fvattn_route((const void*)0x100000, (const void*)0x200000, B, H, N, d, FVATTN_BF16, &g,
                      1.5f, 8, NULL, NULL, (int32_t*)0x300000, (int32_t*)0x400000,
                      (int64_t*)0x500000, (void*)0x600000, (size_t)1 << 30, NULL);
    CHECK(st == FVATTN_ERR_INVALID_ARG, 32);
    /* the E4M3 path needs d = 128 */
    st = fvattn_quantize_v((const void*)0x100000, B, H, N, 64, block, (uint8_t*)0x10000000,
                           (float*)0x20000000, (void*)0x30000000, (size_t)1 << 20, NULL);
    CHECK(st == FVATTN_ERR_UNSUPPORTED, 33);
    /* missing workspace */
    st = fvattn_dense_fwd((const void*)0x100000, (const void*)0x200000, (const void*)0x300000,
                          (void*)0x400000, NULL, NULL, B, H, N, d, FVATTN_BF16, block, 0.088f,
                          NULL, 0, NULL);
    CHECK(st == FVATTN_ERR_WORKSPACE, 34);
    /* the fused V permutation + quantization: d = 128 only, and null outputs */
    st = fvattn_permute_quantize_v((const void*)0x100000, B, H, N, 64, &g, (uint8_t*)0x10000000,
                                   (float*)0x20000000, (void*)0x30000000, (size_t)1 << 20, NULL);
    CHECK(st == FVATTN_ERR_UNSUPPORTED, 35);
    st = fvattn_permute_quantize_v((const void*)0x100000, B, H, N, d, &g, NULL, NULL, NULL, 0, NULL);
    CHECK(st == FVATTN_ERR_INVALID_ARG, 36);
    /* the bounded-wait self-test needs its result buffer and a workspace */
    st = fvattn_wait_selftest(NULL, (void*)0x30000000, 256, NULL);
    CHECK(st == FVATTN_ERR_INVALID_ARG, 37);
    st = fvattn_wait_selftest((int64_t*)0x100000, NULL, 0, NULL);
    CHECK(st == FVATTN_ERR_WORKSPACE, 38);
  }
  {
    int s;
    for (s = FVATTN_OK; s <= FVATTN_ERR_TIMEOUT; ++s) {
      const char* msg = fvattn_status_string((fvattn_status)s);
      CHECK(msg != NULL && msg[0] != '\0', 40 + s);
    }
  }
  printf("abi_host ok\n");
  return 0;
}
