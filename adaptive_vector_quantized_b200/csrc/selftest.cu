// Self-test of the bounded mbarrier wait that every tensor-core kernel uses
// (tc::mbar_wait): one thread waits on an mbarrier that nothing completes;
// the wait must give up after its limit, set the timeout bit of the device
// error word and let the kernel end, so that the context stays usable.  This
// is how a lost copy or MMA completion shows up on the host (AVQ_ERR_TIMEOUT
// from avq_check_device) without faulting or hanging the GPU.
#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace avq {

namespace {

__global__ void wait_probe_kernel(unsigned int* err, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  // phase 0 of a barrier that expects one arrival nobody makes
  if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, timeout_ns)) atomicOr(err, kErrTimeout);
}

}  // namespace

cudaError_t launch_wait_probe(unsigned int* err, unsigned long long timeout_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace avq
