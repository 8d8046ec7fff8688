// Self-test of the in-kernel failure path: a kernel whose pipeline wait can
// never complete (an mbarrier that nothing arrives on) must give up after the
// bounded wait, record FA_ERR_PIPELINE_TIMEOUT in the device status word and
// return, leaving the context usable.  Nothing is faulted or trapped.
#include "fa_exp2.cuh"
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

// Evaluates the softmax's exp2 exactly as the attention kernels do (packed
// pairs), so its accuracy can be measured against fp64 on a dense grid.
template <int DEG>
__global__ void __launch_bounds__(256) exp2_eval_kernel(const float2* __restrict__ x, float2* __restrict__ y,
                                                        long long pairs) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < pairs; i += stride) {
    const float2 a = x[i];
    const uint64_t r = DEG == 0 ? exp2_sfu_f2(f2_pack(a.x, a.y)) : exp2_poly_f2<DEG>(f2_pack(a.x, a.y));
    float lo, hi;
    f2_unpack(r, lo, hi);
    y[i] = make_float2(lo, hi);
  }
}

}  // namespace

cudaError_t launch_selftest_exp2(const float* x, float* y, long long n, int degree, cudaStream_t stream) {
  const long long pairs = n / 2;   // n is even (checked by the entry point)
  const long long blocks = (pairs + 255) / 256;
  const unsigned grid = static_cast<unsigned>(blocks < 148 * 8 ? (blocks > 0 ? blocks : 1) : 148 * 8);
  const float2* x2 = reinterpret_cast<const float2*>(x);
  float2* y2 = reinterpret_cast<float2*>(y);
  switch (degree) {
    case 0: exp2_eval_kernel<0><<<grid, 256, 0, stream>>>(x2, y2, pairs); break;
    case 3: exp2_eval_kernel<3><<<grid, 256, 0, stream>>>(x2, y2, pairs); break;
    case 4: exp2_eval_kernel<4><<<grid, 256, 0, stream>>>(x2, y2, pairs); break;
    default: exp2_eval_kernel<5><<<grid, 256, 0, stream>>>(x2, y2, pairs); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(unsigned int* status, cudaStream_t stream) {
  wait_forever_kernel<<<1, 64, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace fa
