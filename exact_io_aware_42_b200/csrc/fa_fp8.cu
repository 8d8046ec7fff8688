// FP8 (E4M3) block quantisation for the FP8 attention forward ("the
// librarian" page, "FA3 -- the Hopper moment", pillar 3: a per-tile scale
// instead of one per tensor, and a pre-multiplication by a random orthogonal
// Hadamard-based matrix that spreads outliers before quantising; lineage
// page, "FA3 (2024)", idea 3).
//
// Per (b, h) and 128-row block of a [B, H, N, d] bf16 tensor:
//   x <- x diag(s) H_d / sqrt(d)       (optional; H_d Sylvester, s given)
//   scale = max(amax(|x| over the block) / 448, 2^-126)   (1 if the block is all zero)
//   code  = e4m3_rn_satfinite(fp32(x) / scale)
// One CTA of 128 threads per block, thread = row (d = 128: the block moves
// through shared memory by TMA both ways; d = 64: direct loads).  The rotation is the fast
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

// Smallest block scale: the smallest normal fp32, 2^-126.  A block whose
// amax / 448 would be subnormal takes this scale instead, so that 1 / scale
// stays finite (a subnormal scale has no finite fp32 reciprocal and would
// turn 0 / scale into NaN).  Every quotient is then still at most 448.
constexpr float kMinScale = 1.17549435082228751e-38f;

// x / s rounded to nearest, by Markstein's correction step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with y = RN(1/s),
// q0 = RN(x y), r = x - q0 s (exact by FMA), q = RN(q0 + r y).  This gives
// the correctly rounded quotient for normal operands and results; the only
// quotients here outside that range are below 2^-126 in magnitude, which
// round to E4M3 zero either way.  Checked bit for bit against IEEE division
// by the quantisation tests.
// s > 0, so the quotient has the sign of x; copysignf restores it where the
// correction step's sum of zeros would give +0 for x = -0.
__device__ __forceinline__ float div_rn(float x, float s, float y) {
  const float q0 = x * y;
  const float r = fmaf(-q0, s, x);
  return copysignf(fmaf(r, y, q0), x);
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
  const float scale = am > 0.f ? fmaxf(__fdiv_rn(am, 448.f), kMinScale) : 1.f;
  const float inv = __frcp_rn(scale);
  if (r == 0) scales[static_cast<size_t>(bh) * nblk + blk] = scale;
  if (valid) {
#pragma unroll
    for (int c16 = 0; c16 < D / 16; ++c16) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 16 * c16 + 4 * k;
        w[k] = e4m3x4(div_rn(v[i], scale, inv), div_rn(v[i + 1], scale, inv), div_rn(v[i + 2], scale, inv),
                      div_rn(v[i + 3], scale, inv));
      }
      x8[row_off * (D / 16) + c16] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// d = 128 with TMA: a persistent grid (two CTAs per SM) walks the 128-row
// blocks; each block (128 rows x 256 B, two 128-byte swizzled panels)
// arrives in shared memory by one bulk copy issued while the previous block
// is processed (two input buffers); thread r reads row r chunk by chunk at
// the swizzled position (no bank conflicts); the codes go back through a
// 16 KB swizzled tile and one TMA store, which the next block's codes wait
// for only until it has read the tile.
template <bool ROT>
__global__ void __launch_bounds__(128) quant_fp8_tma_kernel(const __grid_constant__ QuantParams p, int total) {
  constexpr int D = 128;
  // dynamic shared memory only (no static variables ahead of it): two input
  // tiles 2 x 32 KB | code tile 16 KB | 2 mbarriers | abort flag | 2 x 4 warp maxima
  extern __shared__ __align__(1024) uint8_t qsm[];
  const uint32_t sbase = smem_u32(qsm);
  const uint32_t out = sbase + 4 * 16384, bars = sbase + 5 * 16384;
  auto in = [&](int b) -> uint32_t { return sbase + b * 2 * 16384; };
  auto bar = [&](int b) -> uint32_t { return bars + 8 * b; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(qsm + 5 * 16384 + 16);
  float* warp_max = reinterpret_cast<float*>(qsm + 5 * 16384 + 32);   // [2][4]
  const int r = threadIdx.x;
  const int G = static_cast<int>(gridDim.x);
  if (r == 0) {
    *abort_flag = 0;
    mbar_init(bar(0), 1);
    mbar_init(bar(1), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (sbase & 1023u) {                  // swizzled tiles need a 1024-byte aligned base
    if (r == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH);
    return;
  }
  auto load = [&](int blk_id, int b) {  // block blk_id -> input buffer b
    const int bh = blk_id / p.nblk, blk = blk_id % p.nblk;
    mbar_arrive_expect_tx(bar(b), 2 * 16384);
    tma_load_3d(in(b), &p.tm_x, bar(b), 0, blk * 128, bh);
    tma_load_3d(in(b) + 16384, &p.tm_x, bar(b), 64, blk * 128, bh);
  };
  const Abort ab{abort_flag, p.status};
  int issued = 0;                        // loads issued (thread 0)
  if (r == 0 && static_cast<int>(blockIdx.x) < total) {
    load(blockIdx.x, 0);
    issued = 1;
  }
  int k = 0;
  for (int blk_id = blockIdx.x; blk_id < total; blk_id += G, ++k) {
    const int b = k & 1;
    // the next block into the other buffer, which every thread finished
    // reading before the barriers of the previous iteration
    if (r == 0 && blk_id + G < total) {
      load(blk_id + G, b ^ 1);
      ++issued;
    }
    const bool ok = __syncthreads_and(mbar_wait(bar(b), (k >> 1) & 1, ab, 32) ? 1 : 0) != 0;
    if (!ok) break;
    const int bh = blk_id / p.nblk, blk = blk_id % p.nblk;
    float v[D];
#pragma unroll
    for (int c = 0; c < 16; ++c) {      // 16-byte chunk c of the row = elements 8c .. 8c+7
      const uint32_t addr = in(b) + (c / 8) * 16384 + r * 128 + (((c % 8) ^ (r & 7)) << 4);
      uint32_t w0, w1, w2, w3;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3) : "r"(addr));
      const uint32_t ww[4] = {w0, w1, w2, w3};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[8 * c + 2 * q] = __uint_as_float(ww[q] << 16);
        v[8 * c + 2 * q + 1] = __uint_as_float(ww[q] & 0xFFFF0000u);
      }
    }
    if constexpr (ROT) {
#pragma unroll
      for (int i = 0; i < D; ++i) v[i] *= p.signs[i];
#pragma unroll
      for (int st = 0; st < 7; ++st) {
        const int h = 1 << st;
#pragma unroll
        for (int bf = 0; bf < D / 2; ++bf) {
          const int lo = (bf >> st) * 2 * h + (bf & (h - 1));
          const float a = v[lo], c2 = v[lo + h];
          v[lo] = a + c2;
          v[lo + h] = a - c2;
        }
      }
#pragma unroll
      for (int i = 0; i < D; ++i) v[i] *= 0.08838834764831845f;
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) am = fmaxf(am, fabsf(v[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
    if ((r & 31) == 0) warp_max[4 * b + (r >> 5)] = am;
    if (r == 0) tma_store_wait_read_all();   // the previous block's codes have left the code tile
    __syncthreads();
    am = fmaxf(fmaxf(warp_max[4 * b], warp_max[4 * b + 1]), fmaxf(warp_max[4 * b + 2], warp_max[4 * b + 3]));
    const float scale = am > 0.f ? fmaxf(__fdiv_rn(am, 448.f), kMinScale) : 1.f;
    const float inv = __frcp_rn(scale);
    if (r == 0) p.scales[static_cast<size_t>(bh) * p.nblk + blk] = scale;
#pragma unroll
    for (int c = 0; c < 8; ++c) {       // 16 codes per chunk
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = 16 * c + 4 * q;
        w[q] = e4m3x4(div_rn(v[i], scale, inv), div_rn(v[i + 1], scale, inv), div_rn(v[i + 2], scale, inv),
                      div_rn(v[i + 3], scale, inv));
      }
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(out + r * 128 + ((c ^ (r & 7)) << 4)),
                   "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (r == 0) {                        // rows past N are clipped by the store
      tma_store_3d(&p.tm_x8, out, 0, blk * 128, bh);
      tma_store_commit();
    }
  }
  if (r == 0) {
    tma_store_wait_read_all();           // the code tile is read before the CTA exits
    if (*abort_flag) {
      // a wait gave up: let every copy this thread issued land (bounded)
      volatile int never = 0;
      const Abort drain{&never, p.status};
      for (int q = (issued > 2 ? issued - 2 : 0); q < issued; ++q) mbar_wait(bar(q & 1), (q >> 1) & 1, drain, 33);
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

cudaError_t launch_quant_fp8_tma(const QuantParams& q, int BH, cudaStream_t stream) {
  const long long total = static_cast<long long>(BH) * q.nblk;
  if (total > 0x7fffffffLL) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long cap = 2ll * (sms > 0 ? sms : 1);   // two CTAs per SM (80 KB of shared memory each)
  const unsigned grid = static_cast<unsigned>(total < cap ? total : cap);
  const int smem = 5 * 16384 + 64;
  if (grid == 0) return cudaSuccess;
  if (q.signs) {
    e = set_smem_once<quant_fp8_tma_kernel<true>>(smem);
    if (e != cudaSuccess) return e;
    quant_fp8_tma_kernel<true><<<grid, 128, smem, stream>>>(q, static_cast<int>(total));
  } else {
    e = set_smem_once<quant_fp8_tma_kernel<false>>(smem);
    if (e != cudaSuccess) return e;
    quant_fp8_tma_kernel<false><<<grid, 128, smem, stream>>>(q, static_cast<int>(total));
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const uint16_t* x, uint8_t* x8, float* scales, const float* signs,
                             int BH, int N, int d, cudaStream_t stream) {
  if (d == 64)
    return signs ? launch_q<64, true>(x, x8, scales, signs, BH, N, stream)
                 : launch_q<64, false>(x, x8, scales, signs, BH, N, stream);
  return signs ? launch_q<128, true>(x, x8, scales, signs, BH, N, stream)
               : launch_q<128, false>(x, x8, scales, signs, BH, N, stream);
}

}  // namespace fa
