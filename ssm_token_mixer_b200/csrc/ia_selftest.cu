// Self-test of the bounded waits' expiry path (a diagnostic with no
// counterpart in the paper).  Every wait in the library's kernels gives up
// after a limit, sets the device error flag and lets the CTA finish; this
// kernel makes that happen on purpose, with nothing in flight: it waits on
// mbarriers that nobody arrives on, with a short limit, so that a test can
// check that the kernel returns and that ia_check_device_errors reports
// IA_ERR_TIMEOUT once and then clears it.
#include <cstdint>

#include "ia_device.cuh"
#include "ia_internal.h"

namespace ia {
namespace {

// Three single-lane waiters, one per warp:
//   warp 0: mbar_wait with the short limit (expires);
//   warp 1: mbar_wait_or_abort with the short limit (expires, raises the
//           CTA's abort flag);
//   warp 2: mbar_wait_or_abort with the full one-second limit on the same
//           barrier: it must return early, as soon as warp 1 has aborted.
// out[2w] = 1 if waiter w saw its phase complete (never here), out[2w + 1] =
// how long its wait took, in ns.
__global__ void __launch_bounds__(96) wait_expiry_kernel(int* err, unsigned long long limit_ns,
                                                         unsigned long long* out) {
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    volatile int* abort = &abort_flag;
    const unsigned long long t0 = global_ns();
    bool done;
    if (warp == 0)
      done = mbar_wait(&bar[0], 0u, err, limit_ns);
    else if (warp == 1)
      done = mbar_wait_or_abort(&bar[1], 0u, err, abort, limit_ns);
    else
      done = mbar_wait_or_abort(&bar[1], 0u, err, abort);
    out[2 * warp] = done ? 1ull : 0ull;
    out[2 * warp + 1] = global_ns() - t0;
  }
}

}  // namespace
}  // namespace ia

using namespace ia;

extern "C" IA_API ia_status_t ia_selftest_wait_expiry(unsigned long long limit_ns, unsigned long long* out,
                                                      void* stream) {
  if (!out || (reinterpret_cast<uintptr_t>(out) & 7u)) return IA_ERR_INVALID_ARG;
  if (limit_ns < 1000ull || limit_ns > kWaitLimitNs) return IA_ERR_INVALID_ARG;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  int* err = device_error_ptr();
  if (!err) return IA_ERR_CUDA;
  wait_expiry_kernel<<<1, 96, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns, out);
  return map_cuda(cudaGetLastError());
}
