// Failure-path self-test: the bounded waits every kernel of the library uses, run against an
// mbarrier that nothing ever signals, with a short limit. Each wait gives up, records the
// timeout in the device error word exactly as a stalled kernel would, and the kernel returns
// normally, so the context stays usable (no trap, no fault, no endless wait).
#include "common.cuh"
#include "internal.h"

namespace svdq {
namespace {

__global__ void k_selftest_wait(uint32_t *err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);  // one arrival expected; none ever comes
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // site 1: the spinning wait; site 2: the parked wait (its error is recorded only if the
    // first one somehow completed, since the error word keeps the first error)
    if (!mbar_wait(smem_u32(&bar), 0, err, KID_SELFTEST, 1, limit_ns)) {
      mbar_wait_parked(smem_u32(&bar), 0, err, KID_SELFTEST, 2, 1000, limit_ns);
    } else {
      record_error(err, KID_SELFTEST, 3);  // a wait on a barrier nobody signals must not succeed
    }
  }
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t *err, uint64_t limit_ns, cudaStream_t st) {
  k_selftest_wait<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace svdq
