// FP8 (E4M3) block quantisation for the FP8 attention forward ("the
// librarian" page, "FA3 -- the Hopper moment", pillar 3: a per-tile scale
// instead of one per tensor, and a pre-multiplication by a random orthogonal
// Hadamard-based matrix that spreads outliers before quantising; lineage
// page, "FA3 (2024)", idea 3).
//
// Per (b, h) and 128-row block of a [B, H, N, d] bf16 tensor:
//   x <- x diag(s) H_d / sqrt(d)       (optional; H_d Sylvester, s given)
//   scale = amax(|x| over the block) / 448   (1 if the block is all zero)
//   code  = e4m3_rn_satfinite(fp32(x) / scale)
// One CTA of 128 threads per block, thread = row.  The rotation is the fast
// Walsh-Hadamard transform (log2 d butterfly stages of a+b, a-b in fp32, in
// registers) followed by one multiply by fp32(1/sqrt(d)); it equals H_d z in
// exact arithmetic and differs from the fp64 product by a few fp32 ulps.
// Memory-bound: 2 bytes read and 1 byte written per element.
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  unsigned short lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <int D, bool ROT>
__global__ void __launch_bounds__(128) quant_fp8_kernel(const uint4* __restrict__ x,
                                                        uint4* __restrict__ x8,
                                                        float* __restrict__ scales,
                                                        const float* __restrict__ signs, int N,
                                                        int nblk) {
  __shared__ float warp_max[4];
  const int bh = blockIdx.x / nblk;
  const int blk = blockIdx.x % nblk;
  const int r = threadIdx.x;
  const int row = blk * 128 + r;
  const bool valid = row < N;
  const size_t row_off = static_cast<size_t>(bh) * N + row;
  float v[D];
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    uint4 w = make_uint4(0, 0, 0, 0);
    if (valid) w = x[row_off * (D / 8) + c8];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * c8 + 2 * k] = __uint_as_float(ww[k] << 16);
      v[8 * c8 + 2 * k + 1] = __uint_as_float(ww[k] & 0xFFFF0000u);
    }
  }
  if constexpr (ROT) {
#pragma unroll
    for (int i = 0; i < D; ++i) v[i] *= signs[i];
    constexpr int kLog2D = (D == 64) ? 6 : 7;
#pragma unroll
    for (int st = 0; st < kLog2D; ++st) {
      const int h = 1 << st;
#pragma unroll
      for (int bf = 0; bf < D / 2; ++bf) {        // butterfly bf of this stage
        const int lo = (bf >> st) * 2 * h + (bf & (h - 1));
        const float a = v[lo], b = v[lo + h];
        v[lo] = a + b;
        v[lo + h] = a - b;
      }
    }
    const float inv_sqrt_d = (D == 64) ? 0.125f : 0.08838834764831845f;
#pragma unroll
    for (int i = 0; i < D; ++i) v[i] *= inv_sqrt_d;
  }
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < D; ++i) am = fmaxf(am, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
  if ((r & 31) == 0) warp_max[r >> 5] = am;
  __syncthreads();
  am = fmaxf(fmaxf(warp_max[0], warp_max[1]), fmaxf(warp_max[2], warp_max[3]));
  const float scale = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
  if (r == 0) scales[static_cast<size_t>(bh) * nblk + blk] = scale;
  if (valid) {
#pragma unroll
    for (int c16 = 0; c16 < D / 16; ++c16) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 16 * c16 + 4 * k;
        w[k] = e4m3x4(__fdiv_rn(v[i], scale), __fdiv_rn(v[i + 1], scale), __fdiv_rn(v[i + 2], scale),
                      __fdiv_rn(v[i + 3], scale));
      }
      x8[row_off * (D / 16) + c16] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <int D, bool ROT>
cudaError_t launch_q(const uint16_t* x, uint8_t* x8, float* scales, const float* signs, int BH, int N,
                     cudaStream_t stream) {
  const int nblk = (N + 127) / 128;
  const unsigned grid = static_cast<unsigned>(BH) * static_cast<unsigned>(nblk);
  quant_fp8_kernel<D, ROT><<<grid, 128, 0, stream>>>(reinterpret_cast<const uint4*>(x),
                                                     reinterpret_cast<uint4*>(x8), scales, signs, N, nblk);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_fp8(const uint16_t* x, uint8_t* x8, float* scales, const float* signs,
                             int BH, int N, int d, cudaStream_t stream) {
  if (d == 64)
    return signs ? launch_q<64, true>(x, x8, scales, signs, BH, N, stream)
                 : launch_q<64, false>(x, x8, scales, signs, BH, N, stream);
  return signs ? launch_q<128, true>(x, x8, scales, signs, BH, N, stream)
               : launch_q<128, false>(x, x8, scales, signs, BH, N, stream);
}

}  // namespace fa
