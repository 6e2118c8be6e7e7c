// noalloc.cu -- fvattn_route_noalloc: the routing front end for callers that
// cannot hand the library a device workspace.
//
// Some callers cannot allocate device memory where they call the router: a
// plugin inside an inference engine that owns all device memory and offers no
// scratch buffer, or a latency-critical loop where cudaMalloc would synchronize
// the device and stall it. This entry point takes no workspace. Its scratch
// (the status word, the pooled q/k block means and the block score matrix that
// fvattn_route keeps in its workspace) lives in the file-scope device array below, which every GPU
// that loads the library holds until the process exits.
//
// Limits and sharing:
//   - At most kScratchBytes (96 MiB) of scratch: sizes whose route workspace
//     (fvattn_workspace_bytes(FVATTN_OP_ROUTE, ...)) is larger are rejected with
//     FVATTN_ERR_WORKSPACE before anything is launched. The Wan-14B 720p shape
//     (40 heads, 591 blocks, d = 128) needs 80.2 MB (block means 24.2 MB, block
//     scores 56.0 MB) and fits.
//   - Every call on a device uses the same array and leaves its contents for
//     the next call. The router clears the status word at the start of each
//     call and overwrites the block means and scores completely, so no stale value is
//     read. Calls whose kernels overlap on the GPU (concurrent streams, or
//     several host threads) race on the array: keep them ordered.
//   - The array's device address is looked up with cudaGetSymbolAddress on the
//     first call on each device (with that device current) and cached; make
//     that first call before capturing a stream into a graph. The cache is
//     keyed on the CUDA context that was current at the lookup: a call under
//     another context (cudaDeviceReset made a new primary context, or the
//     caller made a context of its own current) looks the address up again, so
//     such a first call under a new context should also come before any capture.
//   - Nothing here allocates: no cudaMalloc, no cudaFree, no allocating
//     library routine.
#include <cuda.h>
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(96) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char fvattn_route_scratch[kScratchBytes];

// The driver's cuCtxGetCurrent, looked up once through the runtime (the library
// does not link libcuda directly).
using CtxGetCurrent = CUresult (*)(CUcontext*);
CtxGetCurrent ctx_get_current() {
  static const CtxGetCurrent fn = []() -> CtxGetCurrent {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrent>(p);
    return nullptr;
  }();
  return fn;
}

CUcontext current_context() {
  CUcontext c = nullptr;
  const CtxGetCurrent f = ctx_get_current();
  if (!f || f(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

struct CacheEntry {
  CUcontext ctx;
  void* ptr;
};
std::mutex g_mu;
CacheEntry g_cache[kMaxDevices];

// Device address of the scratch array in the current device's current context
// (nullptr on error). Calls from several host threads are serialised by g_mu.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  CUcontext ctx = current_context();
  if (dev < kMaxDevices && ctx && g_cache[dev].ctx == ctx && g_cache[dev].ptr) return g_cache[dev].ptr;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, fvattn_route_scratch) != cudaSuccess || !ptr) return nullptr;
  ctx = current_context();    // the lookup makes the device's primary context current if none was
  if (dev < kMaxDevices && ctx) g_cache[dev] = CacheEntry{ctx, ptr};
  return ptr;
}

}  // namespace

extern "C" fvattn_status fvattn_route_noalloc(const void* q, const void* k, int B, int H, int N,
                                              int d, fvattn_dtype dtype, const fvattn_grid* grid,
                                              float p, int k_min, void* qp_out, void* kp_out,
                                              int32_t* kv_idx, int32_t* kv_cnt,
                                              int64_t* head_work, void* stream) {
  if (!grid) return FVATTN_ERR_INVALID_ARG;
  const size_t need = fvattn_workspace_bytes(FVATTN_OP_ROUTE, B, H, N, d, grid->block);
  if (need == 0) return FVATTN_ERR_INVALID_ARG;
  if (need > kScratchBytes) return FVATTN_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return FVATTN_ERR_CUDA;
  return fvattn_route(q, k, B, H, N, d, dtype, grid, p, k_min, qp_out, kp_out, kv_idx, kv_cnt,
                      head_work, scratch, kScratchBytes, stream);
}
