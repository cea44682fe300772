// Failure-detection self-test: one kernel whose single mbarrier wait nothing completes.  The
// wait is the same bounded mbar_wait every kernel of the library uses: it gives up after
// kWaitLimitNs, records BQG_DEVERR_TIMEOUT and the kernel returns, so the context stays usable.
// No fault, trap or endless loop is involved.  Part of the single translation unit bqg.cu.
#pragma once

#include "common.cuh"
#include "host_common.h"

namespace bqg {

__global__ void k_wait_selftest() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // phase 0 completes after one arrival, which never comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0u);
}

}  // namespace bqg

extern "C" int bqg_selftest_wait_timeout(void* stream) {
  int dev;
  bqg::DeviceInfo* info;
  const int st = bqg::current_device(&dev, &info);
  if (st != BQG_OK) return st;
  bqg::k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return bqg::launch_status();
}
