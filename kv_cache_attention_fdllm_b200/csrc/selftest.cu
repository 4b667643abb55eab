// fdllm_bounded_wait_selftest: runs the bounded mbarrier wait that every
// kernel of this library uses, against an mbarrier that nothing completes, with
// a short limit, so that the timeout path can be shown to end cleanly.
//
// One CTA of 64 threads.  Thread 0 initialises an mbarrier that expects one
// arrival which never comes.  Lane 0 of warp 0 waits on it with the caller's
// limit: the wait must give up, record FDLLM_ERR_TIMEOUT in the status word and
// set the CTA's abort flag.  Then lane 0 of warp 1 waits on the same barrier:
// with the abort flag set it must return at once, as every later wait of a
// kernel does after a timeout, so that all threads still reach their barriers.
// Both waits' results and durations (globaltimer ns) go to the workspace.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace fdllm {

namespace {

__global__ void __launch_bounds__(64) bounded_wait_selftest_kernel(int* status, uint64_t limit_ns,
                                                                   unsigned long long* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_ns();
    const bool ok = tc::mbar_wait(&bar, 0u, &abort_flag, status, limit_ns);
    result[0] = ok ? 1ull : 0ull;
    result[1] = global_ns() - t0;
  }
  __syncthreads();
  if (threadIdx.x == 32) {
    const uint64_t t0 = global_ns();
    const bool ok = tc::mbar_wait(&bar, 0u, &abort_flag, status, limit_ns);
    result[2] = ok ? 1ull : 0ull;
    result[3] = global_ns() - t0;
  }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* status, uint64_t limit_ns,
                                         unsigned long long* result, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 64, 0, stream>>>(status, limit_ns, result);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fdllm
