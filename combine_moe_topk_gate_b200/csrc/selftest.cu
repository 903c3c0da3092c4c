// selftest.cu -- exercises the bounded wait the pipelined kernels use.
//
// Every wait on an mbarrier in the combine, combine-backward and NVFP4
// kernels gives up after a fixed wall time (kWaitLimitNs, read from
// %globaltimer), records MOE_ERR_TIMEOUT in the caller's status word and lets
// the CTA return, so a lost copy never hangs the GPU.  This kernel waits on an
// mbarrier that nothing completes and takes the same path: it is the way to
// check that path without a fault.
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

__global__ void bounded_wait_selftest_kernel(int32_t* d_status) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    mbar_init_fence();
  }
  __syncthreads();
  // nothing arrives on the barrier, so its first phase never completes
  if (threadIdx.x == 0 && !mbar_wait(b, 0)) report_timeout(d_status);
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int32_t* d_status, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(d_status);
  return cudaGetLastError();
}

}  // namespace moe
