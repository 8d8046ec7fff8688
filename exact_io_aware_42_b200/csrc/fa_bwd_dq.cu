// Deterministic dQ for sm_100a: one CTA per (b, h, 128-query block i).
//
// The atomic backward adds every key block's share of dQ_i into an fp32
// buffer from many CTAs, in an order that is not fixed.  Here dQ_i has a
// single owner instead: the CTA keeps Q_i and dO_i in shared memory, streams
// the key blocks j in ascending order and rebuilds, per tile,
//   S    = Q_i K_j^T            tcgen05 SS   -> TMEM (two buffers)
//   dP   = dO_i V_j^T           tcgen05 SS   -> TMEM
//   P    = 2^(S c - L log2 e)   (recomputation from the saved logsumexp,
//                                "FlashAttention" concept note, "How it works")
//   dS   = P o (dP - D)         dS warps, bf16 over S in TMEM
//   dQ  += dS K_j               tcgen05 TS   (A = dS from TMEM, B = K_j MN-major)
// and writes bf16(scale * dQ) once.  The summation order over j is fixed,
// so dQ is bitwise reproducible; dK and dV come from the main backward
// kernel built without its dQ product.  The price is the recomputation of S
// and dP (three products per tile here against the one dQ product saved in
// the main kernel); the gain is that no CTA issues reductions to memory.
//
// Roles (320 threads): warps 0-7 dS and the epilogue (thread = query row;
// warps 0-3 take keys 0..63 of each tile, warps 4-7 keys 64..127), warp 8
// TMA producer, warp 9 TMEM owner and the single MMA-issuing thread.  K and V
// have separate rings so that K_j, which the dQ product reads last, does not
// hold back the next V.  Every wait is bounded (fa_ptx.cuh).
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

template <int D>
struct DqCfg {
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;       // one 128 x D bf16 tile
  static constexpr int kStagesK = (D == 128) ? 3 : 4;
  static constexpr int kStagesV = (D == 128) ? 2 : 3;
  static constexpr int kThreads = 320;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTileBytes;
  static constexpr int kOffK = 2 * kTileBytes;                       // + s * kTileBytes
  static constexpr int kOffV = kOffK + kStagesK * kTileBytes;        // + s * kTileBytes
  static constexpr int kOffBar = kOffV + kStagesV * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 6;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: S in [0,128) and [128,256) alternately (then dS, packed bf16, over
  // the first half of each warpgroup's columns), dP in [256,384), dQ in
  // [384, 384 + d).
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = 256;
  static constexpr uint32_t kColDQ = 384;
};
static_assert(DqCfg<128>::kSmemBytes <= 232448, "dQ kernel d=128 shared memory");
static_assert(DqCfg<64>::kSmemBytes <= 232448, "dQ kernel d=64 shared memory");

enum : unsigned int { kSiteDProd = 40, kSiteDMmaQ, kSiteDMmaK, kSiteDMmaV, kSiteDMmaDS, kSiteDSmS,
                      kSiteDSmDP, kSiteDEpi, kSiteDDrain, kSiteDAlign };

__device__ __forceinline__ void st_global_v4_dq(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// NPOLY of every 8 column pairs take the FMA-pipe exp2 (fa_exp2.cuh), the
// rest the SFU (d = 64 only, FA_DQ_POLY; measured on B200 the SFU-only
// variant was fastest: the phase is bound by instruction latency, not by
// the SFU's throughput).
template <int D, bool CAUSAL, int NPOLY>
__global__ void __launch_bounds__(320, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = DqCfg<D>;
  constexpr int NK = C::kStagesK;
  constexpr int NV = C::kStagesV;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH | (kSiteDAlign << 8));
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  const int B_QDO = 0;
  auto B_KF = [](int s) { return 1 + s; };
  auto B_KE = [](int s) { return 1 + NK + s; };
  auto B_VF = [](int s) { return 1 + 2 * NK + s; };
  auto B_VE = [](int s) { return 1 + 2 * NK + NV + s; };
  const int B_S0 = 1 + 2 * NK + 2 * NV;            // + t, t = 0, 1
  const int B_DP = B_S0 + 2, B_DS = B_S0 + 3, B_FINAL = B_S0 + 4, B_DRAIN = B_S0 + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Head-major non-causal.  Causal: within each group of group_kv K/V heads
  // (their query heads), query blocks with the most key blocks first across
  // the group's heads (the hardware hands CTAs out in index order: a
  // longest-first schedule whose working set stays in L2).
  int bh, i;
  if (CAUSAL) {
    causal_q_order(static_cast<int>(blockIdx.x), p.n_q, p.group_kv * p.kv_group, p.BH, bh, i);
  } else {
    bh = blockIdx.x / p.n_q;
    i = static_cast<int>(blockIdx.x % p.n_q);
  }
  // Sliding window (causal): key blocks wholly left of the window are skipped.
  const int j_start = CAUSAL ? max(0, i * 128 - p.window) / 128 : 0;
  const int n_j = (CAUSAL ? i + 1 : p.n_kv) - j_start;   // iterations; block = j_start + j
  const int kvh = bh / p.kv_group;   // grouped K/V heads: see the forward kernel

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QDO), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(bar(B_KF(s)), 1);
      mbar_init(bar(B_KE(s)), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar(B_VF(s)), 1);
      mbar_init(bar(B_VE(s)), 1);
    }
    mbar_init(bar(B_S0), 1);
    mbar_init(bar(B_S0 + 1), 1);
    mbar_init(bar(B_DP), 1);
    mbar_init(bar(B_DS), 256);
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag, p.status};
  const uint32_t qAddr = sbase + C::kOffQ, doAddr = sbase + C::kOffDO;
  auto kAddr = [&](int s) -> uint32_t { return sbase + C::kOffK + s * C::kTileBytes; };
  auto vAddr = [&](int s) -> uint32_t { return sbase + C::kOffV + s * C::kTileBytes; };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar(B_QDO), 2 * C::kTileBytes);
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_3d(qAddr + pn * C::kPanelBytes, &p.tm_q, bar(B_QDO), pn * 64, i * 128, bh);
        tma_load_3d(doAddr + pn * C::kPanelBytes, &p.tm_do, bar(B_QDO), pn * 64, i * 128, bh);
      }
      int nk = 0, nv = 0;
      bool ok = true;
      for (int j = 0; j < n_j && ok; ++j) {
        // K_j waits for the dQ product of j - NK, V_j for the dP product of j - NV
        const int sk = j % NK, sv = j % NV;
        if (!(ok = mbar_wait(bar(B_KE(sk)), ((j / NK) & 1) ^ 1, ab, kSiteDProd))) break;
        mbar_arrive_expect_tx(bar(B_KF(sk)), C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(kAddr(sk) + pn * C::kPanelBytes, &p.tm_k, bar(B_KF(sk)), pn * 64, (j_start + j) * 128, kvh);
        ++nk;
        if (!(ok = mbar_wait(bar(B_VE(sv)), ((j / NV) & 1) ^ 1, ab, kSiteDProd))) break;
        mbar_arrive_expect_tx(bar(B_VF(sv)), C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(vAddr(sv) + pn * C::kPanelBytes, &p.tm_v, bar(B_VF(sv)), pn * 64, (j_start + j) * 128, kvh);
        ++nv;
      }
      if (*abort_flag) {   // let the copies in flight land before the CTA leaves
        volatile int never = 0;
        const Abort drain{&never, p.status};
        mbar_wait(bar(B_QDO), 0, drain, kSiteDDrain);
        for (int q = (nk > NK ? nk - NK : 0); q < nk; ++q)
          mbar_wait(bar(B_KF(q % NK)), (q / NK) & 1, drain, kSiteDDrain);
        for (int q = (nv > NV ? nv - NV : 0); q < nv; ++q)
          mbar_wait(bar(B_VF(q % NV)), (q / NV) & 1, drain, kSiteDDrain);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, false, false);   // S, dP
      constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, D, false, true);      // dQ (K MN-major)
      auto gemm_kk = [&](uint32_t dcol, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
          mma_f16_ss(tmem + dcol, smem_desc_sw128(a_addr + off, 16, 1024),
                     smem_desc_sw128(b_addr + off, 16, 1024), kIdescKK, kk > 0 ? 1u : 0u);
        }
      };
      auto wait_k = [&](int j) { return mbar_wait(bar(B_KF(j % NK)), (j / NK) & 1, ab, kSiteDMmaK); };
      auto wait_v = [&](int j) { return mbar_wait(bar(B_VF(j % NV)), (j / NV) & 1, ab, kSiteDMmaV); };
      auto issue_s = [&](int j) {          // S_j -> buffer j % 2
        gemm_kk(C::kColS + 128 * (j & 1), qAddr, kAddr(j % NK));
        tc_commit(bar(B_S0 + (j & 1)));
      };
      auto issue_dp = [&](int j) {         // dP_j; V_j is then free
        gemm_kk(C::kColDP, doAddr, vAddr(j % NV));
        tc_commit(bar(B_DP));
        tc_commit(bar(B_VE(j % NV)));
      };
      bool ok = mbar_wait(bar(B_QDO), 0, ab, kSiteDMmaQ);
      if (ok && (ok = wait_k(0) && wait_v(0))) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        if (n_j > 1 && (ok = wait_k(1))) {
          tc_fence_after();
          issue_s(1);
        }
      }
      for (int j = 0; j < n_j && ok; ++j) {
        // dS_j is in TMEM and dP_j has been read: the dP buffer takes
        // dP_{j+1}, then dQ += dS_j K_j, then S_{j+2} reuses dS_j's buffer
        // (the tensor pipe executes these in issue order).
        if (!(ok = mbar_wait(bar(B_DS), j & 1, ab, kSiteDMmaDS))) break;
        tc_fence_after();
        if (j + 1 < n_j) {
          if (!(ok = wait_v(j + 1))) break;
          tc_fence_after();
          issue_dp(j + 1);
        }
        const uint32_t a_col = C::kColS + 128 * (j & 1);
        const uint32_t k_addr = kAddr(j % NK);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // packed keys 0..63 at a_col, 64..127 at a_col + 64
          mma_f16_ts(tmem + C::kColDQ, tmem + a_col + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                     smem_desc_sw128(k_addr + kk * 2048, C::kPanelBytes, 1024), kIdescDQ,
                     (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_KE(j % NK)));
        if (j + 2 < n_j) {
          if (!(ok = wait_k(j + 2))) break;
          tc_fence_after();
          issue_s(j + 2);
        }
      }
      // Every MMA issued above must be finished before TMEM is released,
      // also when a role gave up part-way.
      tc_commit(bar(B_FINAL));
      tc_commit(bar(B_DRAIN));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_DRAIN), 0, drain, kSiteDDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS, epilogue (thread = query row)
    // Warpgroup wg takes keys [64 wg, 64 wg + 64) of every tile and writes its
    // packed dS over the first 32 of its own 64 fp32 S columns, which the
    // other warpgroup never reads.
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;
    const int q = i * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const size_t grow = static_cast<size_t>(bh) * p.N + (q < p.N ? q : 0);
    const float l2 = q < p.N ? p.lse[grow] * 1.4426950408889634f : INFINITY;   // rows past N: P = 0
    const float dlt = q < p.N ? p.delta[grow] : 0.f;
    const float cs = p.scale_log2;
    // ALiBi: -slope log2(e) |key - query| for this query head
    const float sl2 = p.alibi ? p.alibi[bh % p.H] * 1.4426950408889634f : 0.f;
    bool ok = true;
    for (int j = 0; j < n_j && ok; ++j) {
      const int t = j & 1;
      const uint32_t tS = tmem + C::kColS + 128 * t + lane_off + 64 * wg;
      const uint32_t tDP = tmem + C::kColDP + lane_off + 64 * wg;
      const int jb = j_start + j;
      const int kbase = jb * 128 + 64 * wg;
      // warp-uniform: a key past N, after the query (diagonal) or left of the window
      const bool edge = (CAUSAL && (jb == i || kbase < i * 128 + 127 - p.window)) || kbase + 64 > p.N;
      if (!(ok = mbar_wait_warp(bar(B_S0 + t), (j >> 1) & 1, ab, kSiteDSmS))) break;
      tc_fence_after();
      uint32_t u[64];
      tmem_ld64(tS, u);
      const float dk0 = static_cast<float>(kbase - q);
      // one uniform branch on ALiBi outside the unrolled loop
      auto p_row = [&](auto alibi_on) {
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float n0 = -l2, n1 = -l2;
        if constexpr (decltype(alibi_on)::value) {
          n0 -= sl2 * fabsf(dk0 + static_cast<float>(c));
          n1 -= sl2 * fabsf(dk0 + static_cast<float>(c + 1));
        }
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(u[c]), __uint_as_float(u[c + 1])), f2_pack(cs, cs),
                                  f2_pack(n0, n1));
        float p0, p1;
        f2_unpack(((c / 2) % 8 < NPOLY) ? exp2_poly_f2<3>(x) : exp2_sfu_f2(x), p0, p1);
        u[c] = __float_as_uint(p0);
        u[c + 1] = __float_as_uint(p1);
      }
      };
      if (p.alibi)
        p_row(std::true_type{});
      else
        p_row(std::false_type{});
      if (edge) {   // keys past N, and (diagonal tile) keys after the query
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = kbase + c;
          if (key >= p.N || (CAUSAL && (key > q || key < q - p.window))) u[c] = 0u;
        }
      }
      if (!(ok = mbar_wait_warp(bar(B_DP), j & 1, ab, kSiteDSmDP))) break;
      tc_fence_after();
      uint32_t ds[32];
      {
        uint32_t dp[64];
        tmem_ld64(tDP, dp);
        // dS = P (dP - D), two columns per fp32x2 operation (dP + (-D) is dP - D exactly)
        const uint64_t nd2 = f2_pack(-dlt, -dlt);
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(u[2 * c2]), __uint_as_float(u[2 * c2 + 1])),
                           f2_add(f2_pack(__uint_as_float(dp[2 * c2]), __uint_as_float(dp[2 * c2 + 1])), nd2)),
                    d0, d1);
          ds[c2] = pack_bf16x2(d0, d1);
        }
      }
      tmem_st32(tS, ds);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
    }
    if (ok) ok = mbar_wait_warp(bar(B_FINAL), 0, ab, kSiteDEpi);
    ok = named_bar_and(1, 256, ok);
    if (ok) {
      // Every lane takes part in the warp-collective TMEM loads; only the
      // global stores depend on the row being inside the sequence.  wg 0
      // writes head-dim columns [0, d/2), wg 1 [d/2, d).
      tc_fence_after();
      uint16_t* dst = p.dq + grow * D;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int ch = wg * (D / 64) + cc;
        uint32_t v[32];
        tmem_ld32(tmem + C::kColDQ + lane_off + 32 * ch, v);
        uint32_t pk[16];
#pragma unroll
        for (int t2 = 0; t2 < 16; ++t2)
          pk[t2] = pack_bf16x2(__uint_as_float(v[2 * t2]) * p.scale, __uint_as_float(v[2 * t2 + 1]) * p.scale);
        if (q < p.N) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            st_global_v4_dq(dst + 32 * ch + 8 * w, pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool CAUSAL, int NPOLY>
cudaError_t launch_dq_impl(const BwdParams& p, cudaStream_t stream) {
  using C = DqCfg<D>;
  cudaError_t e = set_smem_once<bwd_dq_kernel<D, CAUSAL, NPOLY>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.n_q) * static_cast<unsigned>(p.BH);
  bwd_dq_kernel<D, CAUSAL, NPOLY><<<grid, C::kThreads, C::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq(const BwdParams& p, int d, bool causal, cudaStream_t stream) {
  // d = 64: poly_groups (FA_BWD_POLY) of 4 selects 0, 2 or 4 of 8 pairs on the polynomial
  if (d == 64) {
    const int np = p.dq_poly;
    if (np == 4) return causal ? launch_dq_impl<64, true, 4>(p, stream) : launch_dq_impl<64, false, 4>(p, stream);
    if (np == 2) return causal ? launch_dq_impl<64, true, 2>(p, stream) : launch_dq_impl<64, false, 2>(p, stream);
    return causal ? launch_dq_impl<64, true, 0>(p, stream) : launch_dq_impl<64, false, 0>(p, stream);
  }
  return causal ? launch_dq_impl<128, true, 0>(p, stream) : launch_dq_impl<128, false, 0>(p, stream);
}

}  // namespace fa
