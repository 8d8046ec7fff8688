// Self-test of the in-kernel failure path: a kernel whose pipeline wait can
// never complete (an mbarrier that nothing arrives on) must give up after the
// bounded wait, record FA_ERR_PIPELINE_TIMEOUT in the device status word and
// return, leaving the context usable.  Nothing is faulted or trapped.
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

__global__ void __launch_bounds__(64) wait_forever_kernel(unsigned int* status) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(bar, 1);        // one arrival expected; none is ever made
    fence_mbar_init();
  }
  __syncthreads();
  const Abort ab{&abort_flag, status};
  // Both warps wait; the first to time out sets the flag, the other then
  // leaves at once.
  mbar_wait_warp(bar, 0, ab, 0x7F);
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned int* status, cudaStream_t stream) {
  wait_forever_kernel<<<1, 64, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace fa
