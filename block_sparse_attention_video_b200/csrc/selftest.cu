// selftest.cu -- fvattn_wait_selftest: exercises the bounded device waits that
// every kernel of the library uses, without any fault.
//
// The attention kernel's roles hand work to each other through shared-memory
// mbarriers. If an arrival were ever lost, an unbounded wait would spin until
// the GPU is reset; instead every wait (mbar_wait in sm100.cuh) gives up after
// kWaitTimeoutNs of %globaltimer, raises a CTA-wide abort flag that makes every
// other waiter of the CTA return at once, and records FVATTN_ERR_TIMEOUT in the
// workspace status word, so the kernel ends and the host reads the status.
//
// This kernel runs exactly those helpers on mbarriers that nothing ever arrives
// at: one thread waits until the limit runs out, a thread of another warp waits
// on a second such barrier and is released by the abort flag, and the drain-style
// wait (no abort flag) runs out too. It touches no TMA, tensor memory or global
// memory other than its result words and the status word.
#include "common.cuh"
#include "sm100.cuh"

namespace fvattn {

__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(long long* out, int* status) {
  __shared__ __align__(8) uint64_t never[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&never[0], 1);
    mbar_init(&never[1], 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  volatile int* af = &abort_flag;
  if (threadIdx.x == 0) {
    // phase 0 of never[0] never completes: the limit runs out
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = mbar_wait(&never[0], 0, af, status);
    out[0] = ok ? 1 : 0;
    out[1] = static_cast<long long>(globaltimer_ns() - t0);
  } else if (threadIdx.x == 32) {
    // released by the abort flag the first waiter raises (or by its own limit)
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = mbar_wait(&never[1], 0, af, status);
    out[2] = ok ? 1 : 0;
    out[3] = static_cast<long long>(globaltimer_ns() - t0);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the final-drain form of the wait has a limit of its own
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = mbar_wait_plain(&never[0], 0);
    out[4] = ok ? 1 : 0;
    out[5] = static_cast<long long>(globaltimer_ns() - t0);
    out[6] = static_cast<long long>(kWaitTimeoutNs);
    out[7] = *af;
  }
}

cudaError_t launch_wait_selftest(long long* out, int* status, cudaStream_t st) {
  wait_selftest_kernel<<<1, 64, 0, st>>>(out, status);
  return cudaGetLastError();
}

}  // namespace fvattn
