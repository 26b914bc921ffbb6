// Self-test of the bounded mbarrier wait that every tensor-core kernel uses
// (tc::mbar_wait): one thread waits on an mbarrier that nothing completes;
// the wait must give up after its limit, set the timeout bit of the device
// error word and let the kernel end, so that the context stays usable.  This
// is how a lost copy or MMA completion shows up on the host (AVQ_ERR_TIMEOUT
// from avq_check_device) without faulting or hanging the GPU.
//
// Also the evaluation of the FMA-pipe 2^x (fm::exp2_poly2), so that its error
// bound can be checked against exact values.
#include <algorithm>

#include "common.cuh"
#include "fastmath.cuh"
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

__global__ void exp2_probe_kernel(const float2* __restrict__ x, float2* __restrict__ y, long long n2) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += (long long)gridDim.x * blockDim.x)
    y[i] = fm::exp2_poly2(x[i]);
}

}  // namespace

cudaError_t launch_exp2_probe(const float* x, float* y, long long n, cudaStream_t st) {
  const long long n2 = n / 2;
  if (n2 == 0) return cudaSuccess;
  const int blocks = (int)std::min<long long>((n2 + 255) / 256, 4096);
  exp2_probe_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float2*>(x), reinterpret_cast<float2*>(y), n2);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(unsigned int* err, unsigned long long timeout_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace avq
