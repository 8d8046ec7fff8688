// Attention backward for sm_100a: dQ, dK, dV of the loss sum(O * dO).
//
// The probabilities are never stored: every tile of P is rebuilt from the
// saved logsumexp, P = exp(S - L) ("FlashAttention" concept note, "How it
// works", recomputation; lineage page, "FA1 (2022)", idea 3).  The gradient
// is the textbook one of softmax(scale Q K^T) V:
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO o O),  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   preprocess  D per row and a zeroed fp32 dQ accumulator (memory-bound)
//   main        one CTA per (b, h, 128-key block j): K_j, V_j stay in shared
//               memory while the 128-query blocks i stream past
//   postprocess dQ = bf16(scale * dQ accumulator) (memory-bound)
//
// Main kernel, per query block i (TMEM lanes are the CTA's 128 keys):
//   S^T  = K_j Q_i^T            tcgen05 SS   -> TMEM [0,128)  (region A)
//   dP^T = V_j dO_i^T           tcgen05 SS   -> TMEM [128,256) (region B)
//   P^T  = 2^(S^T c - L log2 e) softmax warps, bf16 back into TMEM
//   dV  += P^T dO_i             tcgen05 TS   (A = P^T from TMEM)
//   dS^T = P^T o (dP^T - D)     softmax warps, bf16 into TMEM and
//                               into shared memory (MN-major, 128-B swizzle)
//   dK  += dS^T Q_i             tcgen05 TS
//   dQ_i = dS K_j               tcgen05 SS (A = dS, MN-major) -> region B
//   dQ accumulator += dQ_i      dQ warps: TMEM -> shared -> TMA bulk reduce-add
// dV and dK accumulate in TMEM [256,256+d) and [256+d,256+2d) over all i and
// are written once at the end.  dQ accumulation: every key block adds its
// share of a query block's dQ into one fp32 buffer with TMA bulk reductions
// in L2 (the summation order across key blocks is not fixed, so dQ may differ
// in the last bits from run to run; dK and dV are deterministic).
//
// Roles: warps 0-7 P / dS and the dK, dV epilogue (thread = key row; warps
// 0-3 take queries 0..63 of each block, warps 4-7 queries 64..127); warps 8-11
// dQ reduction (thread = query row); warp 12 TMA producer (also stages L and
// D of each query block in shared memory); warp 13 TMEM owner and the single
// MMA-issuing thread.  Every wait is bounded (fa_ptx.cuh).
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

template <int D, bool DQ>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;       // one 128 x D bf16 tile
  // Ring depths: (dO_i, L_i, D_i) and Q_i.  Q_i is read first (S^T) and last
  // (dK), so its ring is one stage deeper where the dS buffer's space is free
  // (no dQ product); the next block's S^T then never waits for its Q tile.
  static constexpr int kStagesD = (D == 128) ? 2 : 3;
  static constexpr int kStagesQ = kStagesD + (DQ ? 0 : 1);
  // 14 warps with the dQ drain warps, 10 without (the roles keep their
  // order: P/dS 0-7, [dQ 8-11], producer, MMA).
  static constexpr int kThreads = DQ ? 448 : 320;
  // All swizzled tiles are 1024-byte aligned offsets from the (1024-aligned)
  // dynamic shared memory base.
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;                        // + s * kTileBytes
  static constexpr int kOffDO = kOffQ + kStagesQ * kTileBytes;        // + s * kTileBytes
  static constexpr int kOffDS = kOffDO + kStagesD * kTileBytes;       // dS^T, 128 x 128 bf16 (dQ only)
  static constexpr int kOffL = kOffDS + (DQ ? 128 * 128 * 2 : 0);     // + s * 512: L log2 e [128], Q ring
  // D_i is staged beside Q_i with dQ (the dO slot is then released as soon
  // as dV has read dO), beside dO_i without dQ (no room for a third D slot)
  static constexpr bool kDWithQ = DQ;
  static constexpr int kDSlots = kDWithQ ? kStagesQ : kStagesD;
  static constexpr int kOffDl = kOffL + kStagesQ * 512;               // + s * 512: D [128]
  static constexpr int kOffBar = kOffDl + kDSlots * 512;
  static constexpr int kNumBars = 1 + 2 * kStagesQ + 2 * kStagesD + 10;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: columns [0,128) hold S^T, then P^T (bf16); [128,256) hold dP^T,
  // then dS^T (bf16), then dQ_i.  S^T of the next block is issued right after
  // dV of this one, so the next P phase overlaps dK, dQ and the dQ drain.
  static constexpr uint32_t kColA = 0;
  static constexpr uint32_t kColB = 128;
  static constexpr uint32_t kColDV = 256;
  static constexpr uint32_t kColDK = 256 + D;
};
static_assert(BwdCfg<128, true>::kSmemBytes <= 232448, "backward d=128 shared memory");
static_assert(BwdCfg<128, false>::kSmemBytes <= 232448, "backward d=128 shared memory");
static_assert(BwdCfg<64, false>::kSmemBytes <= 232448, "backward d=64 shared memory");

enum : unsigned int { kSiteBProd = 16, kSiteBMmaKV, kSiteBMmaQ, kSiteBMmaFree, kSiteBMmaP, kSiteBMmaDS,
                      kSiteBSmS, kSiteBSmDP, kSiteBSmDQ, kSiteBDq, kSiteBEpi, kSiteBDrain, kSiteBAlign };

// ------------------------------------------------------------------ preprocess
// One group of d/8 threads per row (d = 256: a whole warp): 16-byte loads of
// O and dO, fp32 dot product reduced by shuffles; the same threads zero that
// row of dQ_acc.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const uint4* __restrict__ o,
                                                             const uint4* __restrict__ dout,
                                                             float* __restrict__ delta,
                                                             float4* __restrict__ dq_acc,
                                                             long long rows) {
  constexpr int kTpr = D / 8;                       // threads per row (8 or 16)
  constexpr int kRowsPerWarp = 32 / kTpr;
  const int lane = threadIdx.x & 31;
  const int sub = lane % kTpr;
  const long long warp_id = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32;
  const long long nwarps = static_cast<long long>(gridDim.x) * blockDim.x / 32;
  // The loop bound is uniform across the warp so every shuffle sees all lanes.
  for (long long wrow = warp_id * kRowsPerWarp; wrow < rows; wrow += nwarps * kRowsPerWarp) {
    const long long row = wrow + lane / kTpr;
    const bool valid = row < rows;
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    if (valid) {
      a = o[row * kTpr + sub];
      b = dout[row * kTpr + sub];
    }
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      acc = fmaf(__uint_as_float(aw[w] << 16), __uint_as_float(bw[w] << 16), acc);
      acc = fmaf(__uint_as_float(aw[w] & 0xFFFF0000u), __uint_as_float(bw[w] & 0xFFFF0000u), acc);
    }
#pragma unroll
    for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (valid) {
      if (sub == 0) delta[row] = acc;
      if (dq_acc == nullptr) continue;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      dq_acc[row * (D / 4) + 2 * sub] = z;
      dq_acc[row * (D / 4) + 2 * sub + 1] = z;
    }
  }
}

// ------------------------------------------------------------------ postprocess
__global__ void __launch_bounds__(256) bwd_postprocess_kernel(const float4* __restrict__ acc,
                                                              uint2* __restrict__ dq, long long n4,
                                                              float scale) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    const float4 a = acc[i];
    dq[i] = make_uint2(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale));
  }
}

// ------------------------------------------------------------------ split reduction
// dV, dK = bf16(sum over splits s = 0..S-1, in that order, of the fp32
// partials [s][dV, dK][n]); n counts the elements of one of dV, dK.
__global__ void __launch_bounds__(256) bwd_kv_reduce_kernel(const float4* __restrict__ part,
                                                            uint2* __restrict__ dv, uint2* __restrict__ dk,
                                                            long long n4, int splits) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < 2 * n4; i += stride) {
    const long long which = i / n4, e = i % n4;
    float4 a = part[which * n4 + e];
    for (int s = 1; s < splits; ++s) {
      const float4 b = part[(static_cast<long long>(s) * 2 + which) * n4 + e];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    (which ? dk : dv)[e] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
}

// ------------------------------------------------------------------ main
__device__ __forceinline__ void st_shared_v4b(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void st_global_v4(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// NPOLY of every 4 groups of 4 query columns take the FMA-pipe exp2
// (fa_exp2.cuh) in the P phase, the rest the SFU.  DQ = false builds the
// kernel without its dQ product (dK and dV only; the deterministic dQ
// kernel computes dQ): no dS staging in shared memory, no dQ warps' work,
// and the MMA issuer waits on nothing of dQ.
template <int D, bool CAUSAL, int NPOLY, bool DQ>
__global__ void __launch_bounds__(BwdCfg<D, DQ>::kThreads, 1) bwd_main_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D, DQ>;
  constexpr int NQ = C::kStagesQ;
  constexpr int ND = C::kStagesD;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {   // the swizzled layouts below need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH | (kSiteBAlign << 8));
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  const int B_KV = 0;
  auto B_QF = [](int s) { return 1 + s; };             // Q_i landed (L_i written)
  auto B_QE = [](int s) { return 1 + NQ + s; };        // Q_i's slot free
  auto B_DF = [](int s) { return 1 + 2 * NQ + s; };    // dO_i landed (D_i written)
  auto B_DE = [](int s) { return 1 + 2 * NQ + ND + s; };
  // B_DS: dS^T is in TMEM (for dK); B_DSSM: dS is in shared memory (for dQ);
  // B_DQFREE: dQ_i has left TMEM (its region may take the next dP^T);
  // B_DQSMEM: the dS buffer, used to stage dQ_i, is free again.
  const int B_S = 1 + 2 * NQ + 2 * ND, B_DP = B_S + 1, B_P = B_S + 2, B_DS = B_S + 3, B_DQ = B_S + 4,
            B_DQFREE = B_S + 5, B_FINAL = B_S + 6, B_DRAIN = B_S + 7, B_DQSMEM = B_S + 8,
            B_DSSM = B_S + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kWarpProd = DQ ? 12 : 8;
  constexpr int kWarpMma = kWarpProd + 1;
  // Head-major order: the CTAs resident at any time cover a few heads, so
  // their dQ accumulators (and K, V, Q, dO) stay in L2.  Within a head the
  // key blocks with the most query blocks (small j, causal) go first.
  // kvh is the K/V head (flattened [B * H_kv]); with grouped K/V heads the
  // CTA visits the query blocks of its G query heads one head after the
  // other, so dK and dV sum over the group in TMEM.
  // With kv_split = S > 1 (few K/V heads) the G query heads of a group are
  // shared out over S CTAs per key block, G / S heads each; their dK, dV go
  // to fp32 partials that a reduction kernel sums in split order.
  // Causal: longest first within groups of K/V heads (causal_kv_order).
  int kvh, split, j;
  if (CAUSAL) {
    causal_kv_order(static_cast<int>(blockIdx.x), p.n_kv, p.kv_split, p.group_kv, p.BH / p.kv_group, kvh, split, j);
  } else {
    kvh = blockIdx.x / (p.n_kv * p.kv_split);
    split = (blockIdx.x / p.n_kv) % p.kv_split;
    j = blockIdx.x % p.n_kv;
  }
  const int g_per = p.kv_group / p.kv_split;   // query heads of this CTA
  const int i0 = CAUSAL ? j : 0;
  // Sliding window (causal): the last query block that sees a key of block j.
  const int i_last = CAUSAL ? min(p.n_q - 1, (j * 128 + 127 + p.window) / 128) : p.n_q - 1;
  const int n_i = i_last - i0 + 1;          // query blocks per query head (>= 1)
  const int n_it = n_i * g_per;
  auto q_block = [&](int idx) { return i0 + idx % n_i; };
  auto q_head = [&](int idx) { return kvh * p.kv_group + split * g_per + idx / n_i; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar(B_QF(s)), 1);
      mbar_init(bar(B_QE(s)), 1);
    }
    for (int s = 0; s < ND; ++s) {
      mbar_init(bar(B_DF(s)), 1);
      mbar_init(bar(B_DE(s)), 1);
    }
    mbar_init(bar(B_S), 1);
    mbar_init(bar(B_DP), 1);
    mbar_init(bar(B_P), 256);
    mbar_init(bar(B_DS), 256);
    mbar_init(bar(B_DSSM), 256);
    mbar_init(bar(B_DQ), 1);
    mbar_init(bar(B_DQFREE), 128);
    mbar_init(bar(B_DQSMEM), 128);
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag, p.status};
  const uint32_t kAddr = sbase + C::kOffK, vAddr = sbase + C::kOffV, dsAddr = sbase + C::kOffDS;
  auto qAddr = [&](int s) -> uint32_t { return sbase + C::kOffQ + s * C::kTileBytes; };
  auto doAddr = [&](int s) -> uint32_t { return sbase + C::kOffDO + s * C::kTileBytes; };

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    int issued_q = 0, issued_d = 0;
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_do);
      mbar_arrive_expect_tx(bar(B_KV), 2 * C::kTileBytes);
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_3d(kAddr + pn * C::kPanelBytes, &p.tm_k, bar(B_KV), pn * 64, j * 128, kvh);
        tma_load_3d(vAddr + pn * C::kPanelBytes, &p.tm_v, bar(B_KV), pn * 64, j * 128, kvh);
      }
    }
    // Per query block: L_i (log2 units, +inf past N) and D_i (0 past N) beside
    // Q_i (the Q slot is held until dK, after the dS phase has read them; the
    // dO slot is released as soon as dV has read dO); both are written by
    // the warp before the arrive that publishes the slot.  The values of the next block are loaded into
    // registers right after this block's copies are issued, so the load
    // latency runs while the warp waits for the next free slots instead of
    // delaying the next copies.
    auto fetch_rows = [&](int idx, float4& l4, float4& d4) {
      const int i = q_block(idx), qh = q_head(idx);
      float lv[4], dv[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int q = i * 128 + lane * 4 + t;
        const size_t g = static_cast<size_t>(qh) * p.N + q;
        lv[t] = q < p.N ? p.lse[g] * 1.4426950408889634f : INFINITY;
        dv[t] = q < p.N ? p.delta[g] : 0.f;
      }
      l4 = make_float4(lv[0], lv[1], lv[2], lv[3]);
      d4 = make_float4(dv[0], dv[1], dv[2], dv[3]);
    };
    float4 l_next = make_float4(0.f, 0.f, 0.f, 0.f), d_next = l_next;
    if (n_it > 0) fetch_rows(0, l_next, d_next);
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx), qh = q_head(idx);
      const int sq = idx % NQ, sd = idx % ND;
      bool w = true;
      if (lane == 0) w = mbar_wait(bar(B_QE(sq)), ((idx / NQ) & 1) ^ 1, ab, kSiteBProd);
      if (!(ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0)) break;
      reinterpret_cast<float4*>(smem + C::kOffL + sq * 512)[lane] = l_next;
      if constexpr (C::kDWithQ) reinterpret_cast<float4*>(smem + C::kOffDl + sq * 512)[lane] = d_next;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_QF(sq)), C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(qAddr(sq) + pn * C::kPanelBytes, &p.tm_q, bar(B_QF(sq)), pn * 64, i * 128, qh);
        ++issued_q;
        w = mbar_wait(bar(B_DE(sd)), ((idx / ND) & 1) ^ 1, ab, kSiteBProd);
      }
      if (!(ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0)) break;
      if constexpr (!C::kDWithQ) {
        reinterpret_cast<float4*>(smem + C::kOffDl + sd * 512)[lane] = d_next;
        __syncwarp();
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_DF(sd)), C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(doAddr(sd) + pn * C::kPanelBytes, &p.tm_do, bar(B_DF(sd)), pn * 64, i * 128, qh);
        ++issued_d;
      }
      if (idx + 1 < n_it) fetch_rows(idx + 1, l_next, d_next);
    }
    if (lane == 0 && *abort_flag) {   // let the copies in flight land before the CTA leaves
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_KV), 0, drain, kSiteBDrain);
      for (int q = (issued_q > NQ ? issued_q - NQ : 0); q < issued_q; ++q)
        mbar_wait(bar(B_QF(q % NQ)), (q / NQ) & 1, drain, kSiteBDrain);
      for (int q = (issued_d > ND ? issued_d - ND : 0); q < issued_d; ++q)
        mbar_wait(bar(B_DF(q % ND)), (q / ND) & 1, drain, kSiteBDrain);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t kIdescTS = idesc_bf16_f32(128, D, false, true);      // dV, dK
      constexpr uint32_t kIdescQ = idesc_bf16_f32(128, D, true, true);        // dQ
      auto gemm_kk = [&](uint32_t dcol, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
          mma_f16_ss(tmem + dcol, smem_desc_sw128(a_addr + off, 16, 1024),
                     smem_desc_sw128(b_addr + off, 16, 1024), kIdescKK, kk > 0 ? 1u : 0u);
        }
      };
      auto gemm_ts = [&](uint32_t dcol, uint32_t a_col, uint32_t b_addr, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // packed queries 0..63 at a_col, 64..127 at a_col + 64
          mma_f16_ts(tmem + dcol, tmem + a_col + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                     smem_desc_sw128(b_addr + kk * 2048, C::kPanelBytes, 1024), kIdescTS,
                     (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(B_KV), 0, ab, kSiteBMmaKV);
      if (ok && n_it > 0 && (ok = mbar_wait(bar(B_QF(0)), 0, ab, kSiteBMmaQ))) {
        tc_fence_after();
        gemm_kk(C::kColA, kAddr, qAddr(0));                      // S^T(0) = K Q^T
        tc_commit(bar(B_S));
      }
      for (int idx = 0; idx < n_it && ok; ++idx) {
        const int sq = idx % NQ, sd = idx % ND;
        if (DQ && idx > 0) {   // dQ of the previous block has left region B
          if (!(ok = mbar_wait(bar(B_DQFREE), (idx - 1) & 1, ab, kSiteBMmaFree))) break;
        }
        if (!(ok = mbar_wait(bar(B_DF(sd)), (idx / ND) & 1, ab, kSiteBMmaQ))) break;
        tc_fence_after();
        gemm_kk(C::kColB, vAddr, doAddr(sd));                    // dP^T = V dO^T
        tc_commit(bar(B_DP));
        if (!(ok = mbar_wait(bar(B_P), idx & 1, ab, kSiteBMmaP))) break;
        tc_fence_after();
        gemm_ts(C::kColDV, C::kColA, doAddr(sd), idx > 0);       // dV += P^T dO
        if constexpr (C::kDWithQ) tc_commit(bar(B_DE(sd)));   // dP^T and dV, dO_i's readers, are done
        // S^T of the next block goes to region A right behind dV, which is
        // the last reader of P^T there (the dS phase keeps its own copy of P
        // in registers), so the next P phase overlaps dK and dP.
        if (idx + 1 < n_it) {
          const int s1 = (idx + 1) % NQ;
          if (!(ok = mbar_wait(bar(B_QF(s1)), ((idx + 1) / NQ) & 1, ab, kSiteBMmaQ))) break;
          tc_fence_after();
          gemm_kk(C::kColA, kAddr, qAddr(s1));
          tc_commit(bar(B_S));
        }
        if (!(ok = mbar_wait(bar(B_DS), idx & 1, ab, kSiteBMmaDS))) break;
        tc_fence_after();
        gemm_ts(C::kColDK, C::kColB, qAddr(sq), idx > 0);        // dK += dS^T Q
        if constexpr (DQ) {
          if (!(ok = mbar_wait(bar(B_DSSM), idx & 1, ab, kSiteBMmaDS))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)                         // dQ_i = dS K  -> region B
            mma_f16_ss(tmem + C::kColB, smem_desc_sw128(dsAddr + kk * 2048, C::kPanelBytes, 1024),
                       smem_desc_sw128(kAddr + kk * 2048, C::kPanelBytes, 1024), kIdescQ,
                       kk > 0 ? 1u : 0u);
          tc_commit(bar(B_DQ));
        }
        // Without dQ, region B takes dP^T of the next block after this dK in
        // issue order, and its completion (B_DP) implies dK has read dS^T.
        // dK is the last reader of Q_i, and it follows the dS phase, the last
        // reader of L_i and D_i: the Q slot (and without dQ the dO slot, which
        // holds D_i) is free once it completes.
        tc_commit(bar(B_QE(sq)));
        if constexpr (!C::kDWithQ) tc_commit(bar(B_DE(sd)));
      }
      tc_commit(bar(B_FINAL));
      tc_commit(bar(B_DRAIN));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_DRAIN), 0, drain, kSiteBDrain);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P, dS (thread = key row)
    // Two warpgroups split the 128 query columns: wg 0 takes queries 0..63,
    // wg 1 queries 64..127.  Each writes its packed P and dS over the first
    // half of its own fp32 columns (cols 64 wg .. 64 wg + 31), so neither
    // touches a column the other still reads.
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;
    const int key = j * 128 + r;
    const bool key_ok = key < p.N;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col_half = 64u * wg;
    const float cs = p.scale_log2;
    bool ok = true;
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx);
      const float4* L4 = reinterpret_cast<const float4*>(smem + C::kOffL + (idx % NQ) * 512) + 16 * wg;
      const float4* D4 = reinterpret_cast<const float4*>(smem + C::kOffDl + (idx % (C::kDWithQ ? NQ : ND)) * 512) + 16 * wg;
      // Visible query columns of this thread's key: c_lo <= column <= c_hi
      // (column c is query i * 128 + c): after the key on the diagonal block,
      // within the sliding window, and none at all for a key past N.
      const int c_lo = (CAUSAL && i == j) ? r : 0;
      const int c_hi = !key_ok ? -1 : (CAUSAL ? min(127, key + p.window - i * 128) : 127);
      const bool all_visible = c_lo == 0 && c_hi == 127;   // no mask in this block for this key
      // ALiBi: -slope log2(e) |query - key| for this block's query head
      const float sl2 = p.alibi ? p.alibi[q_head(idx) % p.H] * 1.4426950408889634f : 0.f;
      const float dq0 = static_cast<float>(i * 128 + static_cast<int>(col_half) - key);
      const uint32_t tS = tmem + C::kColA + lane_off + col_half;
      const uint32_t tDP = tmem + C::kColB + lane_off + col_half;
      if (!(ok = mbar_wait_warp(bar(B_S), idx & 1, ab, kSiteBSmS))) break;
      tc_fence_after();
      uint32_t pp[32];   // this thread's P^T row, packed bf16: the dS phase reads it here
      {
        uint32_t u[64];
        tmem_ld64(tS, u);
        // one uniform branch on ALiBi outside the unrolled loop
        auto p_rows = [&](auto alibi_on) {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l4 = L4[c4];
          const float lq[4] = {l4.x, l4.y, l4.z, l4.w};
          float pv[4];
          float nl[4] = {-lq[0], -lq[1], -lq[2], -lq[3]};
          if constexpr (decltype(alibi_on)::value) {
#pragma unroll
            for (int t = 0; t < 4; ++t) nl[t] -= sl2 * fabsf(dq0 + static_cast<float>(4 * c4 + t));
          }
          const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(u[4 * c4]), __uint_as_float(u[4 * c4 + 1])),
                                      f2_pack(cs, cs), f2_pack(nl[0], nl[1]));
          const uint64_t x23 = f2_fma(f2_pack(__uint_as_float(u[4 * c4 + 2]), __uint_as_float(u[4 * c4 + 3])),
                                      f2_pack(cs, cs), f2_pack(nl[2], nl[3]));
          const bool poly = (c4 & 3) < NPOLY;
          const uint64_t p01 = poly ? exp2_poly_f2<3>(x01) : exp2_sfu_f2(x01);
          const uint64_t p23 = poly ? exp2_poly_f2<3>(x23) : exp2_sfu_f2(x23);
          f2_unpack(p01, pv[0], pv[1]);
          f2_unpack(p23, pv[2], pv[3]);
          if (!CAUSAL || !all_visible) {   // non-causal: unbranched (fewer spills)
#pragma unroll
            for (int t = 0; t < 4; ++t) {                // query 64 wg + 4 c4 + t
              const int col = static_cast<int>(col_half) + 4 * c4 + t;
              pv[t] = (col < c_lo || col > c_hi) ? 0.f : pv[t];
            }
          }
          u[2 * c4] = pack_bf16x2(pv[0], pv[1]);
          u[2 * c4 + 1] = pack_bf16x2(pv[2], pv[3]);
        }
        };
        if (p.alibi)
          p_rows(std::true_type{});
        else
          p_rows(std::false_type{});
#pragma unroll
        for (int c = 0; c < 32; ++c) pp[c] = u[c];
        tmem_st32(tS, pp);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_P));
      if (!(ok = mbar_wait_warp(bar(B_DP), idx & 1, ab, kSiteBSmDP))) break;
      tc_fence_after();
      uint32_t ds[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {                      // 32 dP^T columns at a time
        uint32_t dp[32];
        tmem_ld32(tDP + 32 * h, dp);
#pragma unroll
        for (int c4 = 8 * h; c4 < 8 * h + 8; ++c4) {
          const float4 d4 = D4[c4];
          const float dq[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int t2 = 0; t2 < 2; ++t2) {
            const int c2 = 2 * c4 + t2;                  // packed pair index
            const float p0 = __uint_as_float(pp[c2] << 16), p1 = __uint_as_float(pp[c2] & 0xFFFF0000u);
            float d0, d1;
            if constexpr (CAUSAL) {
              // dS = P (dP - D), two columns per fp32x2 operation (dP + (-D)
              // is dP - D exactly); the non-causal build measured faster with
              // scalar operations (fewer spills)
              const uint64_t g2 =
                  f2_add(f2_pack(__uint_as_float(dp[2 * c2 - 32 * h]), __uint_as_float(dp[2 * c2 + 1 - 32 * h])),
                         f2_pack(-dq[2 * t2], -dq[2 * t2 + 1]));
              f2_unpack(f2_mul(f2_pack(p0, p1), g2), d0, d1);
            } else {
              d0 = p0 * (__uint_as_float(dp[2 * c2 - 32 * h]) - dq[2 * t2]);
              d1 = p1 * (__uint_as_float(dp[2 * c2 + 1 - 32 * h]) - dq[2 * t2 + 1]);
            }
            ds[c2] = pack_bf16x2(d0, d1);
          }
        }
      }
      tmem_st32(tDP, ds);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
      if constexpr (!DQ) continue;
      // the dS buffer doubles as the dQ staging area: wait until the dQ
      // reduction of the previous block has left it
      if (idx > 0 && !(ok = mbar_wait_warp(bar(B_DQSMEM), (idx - 1) & 1, ab, kSiteBSmDQ))) break;
      {
        const uint32_t row = dsAddr + wg * C::kPanelBytes + r * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_shared_v4b(row + ((q ^ (r & 7)) << 4), ds[4 * q], ds[4 * q + 1], ds[4 * q + 2], ds[4 * q + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(B_DSSM));
    }
    if (ok) ok = mbar_wait_warp(bar(B_FINAL), 0, ab, kSiteBEpi);
    ok = named_bar_and(1, 256, ok);
    if (ok) {
      // Every lane takes part in the warp-collective TMEM loads; only the
      // global stores depend on the key being inside the sequence.  wg 0
      // writes head-dim columns [0, d/2), wg 1 [d/2, d).
      tc_fence_after();
      const size_t g = (static_cast<size_t>(kvh) * p.N + (key_ok ? key : 0)) * D;
      const size_t kv_elems = static_cast<size_t>(p.BH / p.kv_group) * p.N * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {      // 0: dV, 1: dK (times scale)
        const uint32_t src = tmem + (which ? C::kColDK : C::kColDV) + lane_off;
        uint16_t* dst = (which ? p.dk : p.dv) + g;
        const float mul = which ? p.scale : 1.f;
        // split partials: [split][dV, dK][B * H_kv, N, d] fp32
        float* part = p.kv_part + (static_cast<size_t>(split) * 2 + which) * kv_elems + g;
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          const int ch = wg * (D / 64) + cc;
          uint32_t u[32];
          tmem_ld32(src + 32 * ch, u);
          if (p.kv_split > 1) {
            if (key_ok) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                st_global_v4(part + 32 * ch + 4 * q, __float_as_uint(__uint_as_float(u[4 * q]) * mul),
                             __float_as_uint(__uint_as_float(u[4 * q + 1]) * mul),
                             __float_as_uint(__uint_as_float(u[4 * q + 2]) * mul),
                             __float_as_uint(__uint_as_float(u[4 * q + 3]) * mul));
            }
            continue;
          }
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t)
            pk[t] = pack_bf16x2(__uint_as_float(u[2 * t]) * mul, __uint_as_float(u[2 * t + 1]) * mul);
          if (key_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_global_v4(dst + 32 * ch + 8 * q, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
    }
  } else if (DQ && warp < 12) {
    // ------------------------------------------------------------ dQ reduction (thread = query row)
    // dQ_i leaves TMEM at once: head-dim columns [0, 64) go to the dS buffer
    // (free once the dQ MMA has read it) as two 128-byte swizzled boxes of 32
    // fp32 columns, columns [64, d) into registers; then the TMEM region is
    // released (the next dP^T may start), the staged half is added into the
    // fp32 accumulator by TMA bulk reductions, the register half is staged and
    // reduced the same way, and finally the dS buffer is released.
    const int r = threadIdx.x - 256;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx), qh = q_head(idx);
      ok = mbar_wait_warp(bar(B_DQ), idx & 1, ab, kSiteBDq);
      // all four warps agree before any of them enters the named barriers below
      if (!(ok = named_bar_and(2, 128, ok))) break;
      tc_fence_after();
      const uint32_t src = tmem + C::kColB + lane_off;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t u[32];
        tmem_ld32(src + 32 * b, u);
        const uint32_t srow = dsAddr + b * 16384 + r * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_shared_v4b(srow + ((q ^ (r & 7)) << 4), u[4 * q], u[4 * q + 1], u[4 * q + 2], u[4 * q + 3]);
      }
      uint32_t hi[D > 64 ? D - 64 : 1];
      if constexpr (D > 64) {
        tmem_ld32(src + 64, *reinterpret_cast<uint32_t(*)[32]>(&hi[0]));
        tmem_ld32(src + 96, *reinterpret_cast<uint32_t(*)[32]>(&hi[32]));
      }
      tc_fence_before();
      mbar_arrive(bar(B_DQFREE));
      fence_proxy_async_smem();
      named_bar_sync(2, 128);
      if (r == 0) {
#pragma unroll
        for (int b = 0; b < 2; ++b) tma_reduce_add_3d(&p.tm_dqacc, dsAddr + b * 16384, 32 * b, i * 128, qh);
        tma_store_commit();
      }
      if constexpr (D > 64) {
        if (r == 0) tma_store_wait_read_all();
        named_bar_sync(2, 128);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint32_t srow = dsAddr + b * 16384 + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_shared_v4b(srow + ((q ^ (r & 7)) << 4), hi[32 * b + 4 * q], hi[32 * b + 4 * q + 1],
                          hi[32 * b + 4 * q + 2], hi[32 * b + 4 * q + 3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (r == 0) {
#pragma unroll
          for (int b = 0; b < 2; ++b)
            tma_reduce_add_3d(&p.tm_dqacc, dsAddr + b * 16384, 64 + 32 * b, i * 128, qh);
          tma_store_commit();
        }
      }
      if (r == 0) tma_store_wait_read_all();   // staging buffer may be rewritten
      named_bar_sync(2, 128);
      mbar_arrive(bar(B_DQSMEM));
    }
    if (r == 0) tma_store_wait_all();      // every reduction has landed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool CAUSAL, int NPOLY, bool DQ>
cudaError_t launch_main_impl(const BwdParams& p, cudaStream_t stream) {
  using C = BwdCfg<D, DQ>;
  auto kern = bwd_main_kernel<D, CAUSAL, NPOLY, DQ>;
  cudaError_t e = set_smem_once<bwd_main_kernel<D, CAUSAL, NPOLY, DQ>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.n_kv) * static_cast<unsigned>(p.BH / p.kv_group) *
                        static_cast<unsigned>(p.kv_split);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

unsigned elementwise_grid(long long items) {
  const long long blocks = (items + 255) / 256;
  return static_cast<unsigned>(blocks < 148LL * 16 ? (blocks > 0 ? blocks : 1) : 148LL * 16);
}

}  // namespace

cudaError_t launch_bwd_preprocess(const uint16_t* o, const uint16_t* dout, float* delta,
                                  float* dq_acc, long long rows, int d, cudaStream_t stream) {
  const unsigned grid = elementwise_grid(rows * (d / 8));
  if (d == 64)
    bwd_preprocess_kernel<64><<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(o),
                                                        reinterpret_cast<const uint4*>(dout), delta,
                                                        reinterpret_cast<float4*>(dq_acc), rows);
  else if (d == 256)
    bwd_preprocess_kernel<256><<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(o),
                                                         reinterpret_cast<const uint4*>(dout), delta,
                                                         reinterpret_cast<float4*>(dq_acc), rows);
  else
    bwd_preprocess_kernel<128><<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(o),
                                                         reinterpret_cast<const uint4*>(dout), delta,
                                                         reinterpret_cast<float4*>(dq_acc), rows);
  return cudaGetLastError();
}

template <int D, bool CAUSAL>
cudaError_t launch_main_np(const BwdParams& p, bool with_dq, cudaStream_t stream) {
  if (!with_dq) return launch_main_impl<D, CAUSAL, 0, false>(p, stream);
  switch (p.poly_groups) {
    case 1: return launch_main_impl<D, CAUSAL, 1, true>(p, stream);
    case 2: return launch_main_impl<D, CAUSAL, 2, true>(p, stream);
    default: return launch_main_impl<D, CAUSAL, 0, true>(p, stream);
  }
}

cudaError_t launch_bwd_main(const BwdParams& p, int d, bool causal, bool with_dq, cudaStream_t stream) {
  if (d == 64)
    return causal ? launch_main_np<64, true>(p, with_dq, stream) : launch_main_np<64, false>(p, with_dq, stream);
  return causal ? launch_main_np<128, true>(p, with_dq, stream) : launch_main_np<128, false>(p, with_dq, stream);
}

cudaError_t launch_bwd_kv_reduce(const float* part, uint16_t* dv, uint16_t* dk, long long n, int splits,
                                 cudaStream_t stream) {
  const long long n4 = n / 4;
  bwd_kv_reduce_kernel<<<elementwise_grid(2 * n4), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(part), reinterpret_cast<uint2*>(dv), reinterpret_cast<uint2*>(dk), n4,
      splits);
  return cudaGetLastError();
}

cudaError_t launch_bwd_postprocess(const float* dq_acc, uint16_t* dq, long long n, float scale,
                                   cudaStream_t stream) {
  const long long n4 = n / 4;
  bwd_postprocess_kernel<<<elementwise_grid(n4), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(dq_acc), reinterpret_cast<uint2*>(dq), n4, scale);
  return cudaGetLastError();
}

}  // namespace fa
