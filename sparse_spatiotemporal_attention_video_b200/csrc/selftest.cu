// selftest.cu -- exercises the bounded wait every kernel of this library uses
// (mbar_wait): one CTA waits on an mbarrier phase that nothing completes, with
// a caller-chosen limit, and must give up, raise STA_DEV_TIMEOUT and return.
// The GPU context stays usable afterwards; no trap, no fault.  In the debug
// build, also the index check of every kernel (dcheck) on a caller's index.
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace sta {
namespace {

__global__ void bounded_wait_kernel(uint64_t limit_ns, int32_t* dev_status, int32_t* waited_ok) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none is ever made
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* ab = &abort_flag;
    const bool ok = mbar_wait(&bar, 0, ab, limit_ns);
    *waited_ok = ok ? 1 : 0;
    if (!ok) raise_status(dev_status, STA_DEV_TIMEOUT);
  }
}

// Stores 1 into buf[index] through the debug build's check.  Launched only by
// the debug build (the C ABI refuses it otherwise).
__global__ void index_check_kernel(int32_t* buf, int n, int index, int32_t* dev_status) {
  if (dcheck(index >= 0 && index < n, dev_status)) buf[index] = 1;
}

}  // namespace

cudaError_t launch_index_check_selftest(int32_t* buf, int n, int index, int32_t* dev_status,
                                        cudaStream_t s) {
  index_check_kernel<<<1, 1, 0, s>>>(buf, n, index, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int32_t* dev_status,
                                         int32_t* waited_ok, cudaStream_t s) {
  bounded_wait_kernel<<<1, 32, 0, s>>>(limit_ns, dev_status, waited_ok);
  return cudaGetLastError();
}

}  // namespace sta
