// selftest.cu -- exercises the bounded-wait path without faulting the GPU.
//
// One CTA initialises an mbarrier that nothing ever completes and waits on it
// with a short limit, first with the suspending wait (mbar_wait_sleep_limit, its outcome
// kept in a shared-memory error word), then with the polling one (mbar_wait_limit).  Each
// wait gives up; the second records OB_DEVERR_TIMEOUT in the device error word and the
// kernel returns normally; the host then reads the error word.  Should the suspending wait
// not give up as it must (return true, or no timeout recorded), OB_DEVERR_NAN is recorded
// instead and the second wait skipped, so the host sees another status.  No trap, assert
// or unbounded loop is involved.
#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

__global__ void timeout_selftest_kernel(unsigned* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ unsigned sleep_err;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    sleep_err = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool done = mbar_wait_sleep_limit(&bar, 0, &sleep_err, nullptr, limit_ns);
    if (done || sleep_err != OB_DEVERR_TIMEOUT)
      record_error(err, OB_DEVERR_NAN);
    else
      (void)mbar_wait_limit(&bar, 0, err, &abort_flag, limit_ns);
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(&bar);  // complete the phase before exit
}

}  // namespace

cudaError_t launch_timeout_selftest(uint64_t limit_ns, const LaunchCtx& c) {
  if (limit_ns > 1000000000ull) limit_ns = 1000000000ull;  // never longer than 1 s
  timeout_selftest_kernel<<<1, 32, 0, c.stream>>>(c.err, limit_ns);
  return cudaGetLastError();
}

}  // namespace ob
