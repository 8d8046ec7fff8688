// dK, dV of the attention backward on CTA pairs (cta_group::2), d = 128.
//
// Same gradient as the single-CTA main kernel (fa_bwd.cu, built without its
// dQ product): P = 2^(S c - L log2 e) is recomputed from the saved
// logsumexp ("FlashAttention" concept note, "How it works", recomputation),
// dV = P^T dO, dS = P o (dP - D), dK = scale dS^T Q.  dQ comes from the
// query-block-major dQ kernel (fa_bwd_dq.cu), so the result is the
// deterministic backward.
//
// What changes is the unit of work: a cluster of two CTAs owns 256
// consecutive keys, 128 per CTA, and every product is one cta_group::2
// tcgen05.mma issued by a single thread of the rank-0 CTA ("the lineage
// page", "FA4 (2026)", change 4: 2-CTA MMA in the backward for a larger
// effective tile; "the librarian" page, "FA4", idea 3):
//   S^T  = K Q_i^T    M = 256 keys (each CTA's own 128 rows of K), N = 128
//                     queries, each CTA holding 64 of the query rows of Q_i
//   dP^T = V dO_i^T   likewise with V and dO_i
//   dV  += P^T dO_i   A = P^T from each CTA's TMEM, N = d: each CTA holds
//                     one 64-column panel of dO_i (all 128 queries)
//   dK  += dS^T Q_i   likewise with dS^T and a 64-column panel of Q_i
// Each CTA therefore keeps 64 rows of Q_i and dO_i for the S^T / dP^T
// products plus one d-panel of each for dK / dV: the B operands a CTA
// reads from shared memory per query block are half those of the
// single-CTA kernel, and the TMA engine of each SM moves 64 KB per block.
// TMEM per CTA (512 columns): S^T / P^T [0,128), dP^T / dS^T [128,256),
// dV [256,384), dK [384,512).
//
// Synchronisation across the pair (all waits bounded, fa_ptx.cuh):
//  - operand loads: each CTA loads its own operands on its own full
//    barriers; in the rank-1 CTA one thread (warp 9) forwards each
//    completed stage to a barrier of rank 0, where the issuing thread waits
//    for both;
//  - P^T and dS^T ready: lane 0 of each of the 8 P/dS warps of both CTAs
//    arrives on rank 0's barrier (16 arrivals);
//  - product completion: tcgen05.commit multicast to the same barrier in
//    both CTAs (S^T, dP^T ready; operand slots free; final);
//  - L and D rows are staged in each CTA by its own producer warp, behind a
//    local barrier.
// A CTA that gives up marks the peer's abort flag too, so both leave their
// loops; the pair meets at a cluster barrier before TMEM is released.
//
// Roles (320 threads per CTA): warps 0-7 P / dS and the dK, dV epilogue
// (thread = key row; warps 0-3 query columns 0..63, warps 4-7 64..127),
// warp 8 producer, warp 9 TMEM owner (rank 0: the MMA-issuing thread).
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

struct PairCfg {
  static constexpr int D = 128;
  static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes
  static constexpr int kHalfPanelBytes = 64 * 128;     // 64 rows x 128 bytes
  static constexpr int kTileBytes = 128 * D * 2;       // K or V of this CTA
  static constexpr int kStageBytes = 32768;            // rows half (16 KB) + d-panel (16 KB)
  static constexpr int kStagesQ = 3;
  static constexpr int kStagesD = 2;
  static constexpr int kThreads = 320;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;                        // + s * kStageBytes
  static constexpr int kOffDO = kOffQ + kStagesQ * kStageBytes;       // + s * kStageBytes
  static constexpr int kOffL = kOffDO + kStagesD * kStageBytes;       // + s * 512
  static constexpr int kOffDl = kOffL + kStagesQ * 512;               // + s * 512
  static constexpr int kOffBar = kOffDl + kStagesD * 512;
  static constexpr int kNumBars = 2 + 4 * kStagesQ + 4 * kStagesD + 6;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColA = 0;
  static constexpr uint32_t kColB = 128;
  static constexpr uint32_t kColDV = 256;
  static constexpr uint32_t kColDK = 384;
};
static_assert(PairCfg::kSmemBytes <= 232448, "pair backward shared memory");

enum : unsigned int { kSitePProd = 80, kSitePMmaKV, kSitePMmaQ, kSitePMmaP, kSitePMmaDS, kSitePSmS, kSitePSmDP,
                      kSitePSmL, kSitePEpi, kSitePDrain, kSitePAlign };

__device__ __forceinline__ void st_global_v4_pair(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

template <bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    bwd_pair_kernel(const __grid_constant__ BwdParams p) {
  using C = PairCfg;
  constexpr int D = C::D;
  constexpr int NQ = C::kStagesQ;
  constexpr int ND = C::kStagesD;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  // local barriers (each CTA) and the rank-0 barriers that rank 1 forwards
  // its completed loads to (suffix P)
  const int B_KV = 0, B_KVP = 1;
  auto B_QF = [](int s) { return 2 + s; };                  // Q stage s landed (own CTA)
  auto B_QFP = [](int s) { return 2 + NQ + s; };            // ... in rank 1 (rank 0 only)
  auto B_QE = [](int s) { return 2 + 2 * NQ + s; };         // Q stage s free (each CTA)
  auto B_LQ = [](int s) { return 2 + 3 * NQ + s; };         // L rows of stage s staged (each CTA)
  auto B_DF = [](int s) { return 2 + 4 * NQ + s; };
  auto B_DFP = [](int s) { return 2 + 4 * NQ + ND + s; };
  auto B_DE = [](int s) { return 2 + 4 * NQ + 2 * ND + s; };
  auto B_LD = [](int s) { return 2 + 4 * NQ + 3 * ND + s; };
  const int B_S = 2 + 4 * NQ + 4 * ND, B_DP = B_S + 1, B_P = B_S + 2, B_DS = B_S + 3, B_FINAL = B_S + 4,
            B_DRAIN = B_S + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair index -> (K/V head, split, 256-key block J); this CTA's keys are
  // [256 J + 128 rank, 256 J + 128 rank + 128), key block j = 2 J + rank.
  // Head-major non-causal; causal: longest first within groups of K/V heads
  // (causal_kv_order over 256-key blocks).
  const int n_kv2 = (p.N + 255) / 256;
  const int pair = blockIdx.x >> 1;
  int kvh, split, J;
  if (CAUSAL) {
    causal_kv_order(pair, n_kv2, p.kv_split, p.group_kv, p.BH / p.kv_group, kvh, split, J);
  } else {
    kvh = pair / (n_kv2 * p.kv_split);
    split = (pair / n_kv2) % p.kv_split;
    J = pair % n_kv2;
  }
  const int j = 2 * J + static_cast<int>(rank);
  const int g_per = p.kv_group / p.kv_split;
  // query blocks of the pair: causal from the first block that sees key
  // 256 J; with a window, up to the last block that sees the pair's last key
  const int i0 = CAUSAL ? 2 * J : 0;
  const int i_last = CAUSAL ? min(p.n_q - 1, (J * 256 + 255 + p.window) / 128) : p.n_q - 1;
  const int n_i = i_last - i0 + 1;
  const int n_it = n_i * g_per;
  auto q_block = [&](int idx) { return i0 + idx % n_i; };
  auto q_head = [&](int idx) { return kvh * p.kv_group + split * g_per + idx / n_i; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    mbar_init(bar(B_KVP), 1);
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar(B_QF(s)), 1);
      mbar_init(bar(B_QFP(s)), 1);
      mbar_init(bar(B_QE(s)), 1);
      mbar_init(bar(B_LQ(s)), 1);
    }
    for (int s = 0; s < ND; ++s) {
      mbar_init(bar(B_DF(s)), 1);
      mbar_init(bar(B_DFP(s)), 1);
      mbar_init(bar(B_DE(s)), 1);
      mbar_init(bar(B_LD(s)), 1);
    }
    mbar_init(bar(B_S), 1);
    mbar_init(bar(B_DP), 1);
    mbar_init(bar(B_P), 16);      // lane 0 of the 8 P/dS warps of both CTAs
    mbar_init(bar(B_DS), 16);
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers exist before any load or arrive targets them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag, p.status};
  const uint32_t peer_flag = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  auto lead_bar = [&](int i) -> uint32_t { return mapa_shared(bar(i), 0); };
  const uint32_t kAddr = sbase + C::kOffK, vAddr = sbase + C::kOffV;
  auto qAddr = [&](int s) -> uint32_t { return sbase + C::kOffQ + s * C::kStageBytes; };
  auto doAddr = [&](int s) -> uint32_t { return sbase + C::kOffDO + s * C::kStageBytes; };

  if (sbase & 1023u) {   // the swizzled layouts below need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH | (kSitePAlign << 8));
    *abort_flag = 1;
  } else if (warp == 8) {
    // ------------------------------------------------------------ producer
    int issued_q = 0, issued_d = 0;
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_do);
      // K, V of this CTA's 128 keys (both 64-column panels each)
      mbar_arrive_expect_tx(bar(B_KV), 2 * C::kTileBytes);
      for (int pn = 0; pn < 2; ++pn) {
        tma_load_3d(kAddr + pn * C::kPanelBytes, &p.tm_k, bar(B_KV), pn * 64, j * 128, kvh);
        tma_load_3d(vAddr + pn * C::kPanelBytes, &p.tm_v, bar(B_KV), pn * 64, j * 128, kvh);
      }
    }
    // L_i (log2 units, +inf past N) and D_i (0 past N) rows of a query block
    auto stage_rows = [&](float* dst, const float* src, int qh, int i, float mul, float pad) {
      float v4[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int q = i * 128 + lane * 4 + t;
        v4[t] = q < p.N ? src[static_cast<size_t>(qh) * p.N + q] * mul : pad;
      }
      reinterpret_cast<float4*>(dst)[lane] = make_float4(v4[0], v4[1], v4[2], v4[3]);
      __syncwarp();
    };
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx), qh = q_head(idx);
      const int sq = idx % NQ, sd = idx % ND;
      bool w = true;
      if (lane == 0) w = mbar_wait(bar(B_QE(sq)), ((idx / NQ) & 1) ^ 1, ab, kSitePProd);
      if (!(ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0)) break;
      stage_rows(reinterpret_cast<float*>(smem + C::kOffL + sq * 512), p.lse, qh, i, 1.4426950408889634f, INFINITY);
      if (lane == 0) {
        mbar_arrive(bar(B_LQ(sq)));
        mbar_arrive_expect_tx(bar(B_QF(sq)), C::kStageBytes);
        // rows [64 rank, 64 rank + 64) of Q_i, both d-panels (B of S^T)
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d(qAddr(sq) + pn * C::kHalfPanelBytes, &p.tm_q64, bar(B_QF(sq)), pn * 64,
                      i * 128 + 64 * static_cast<int>(rank), qh);
        // d-panel ``rank`` of all 128 rows of Q_i (B of dK)
        tma_load_3d(qAddr(sq) + 2 * C::kHalfPanelBytes, &p.tm_q, bar(B_QF(sq)), 64 * static_cast<int>(rank),
                    i * 128, qh);
        ++issued_q;
        w = mbar_wait(bar(B_DE(sd)), ((idx / ND) & 1) ^ 1, ab, kSitePProd);
      }
      if (!(ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0)) break;
      stage_rows(reinterpret_cast<float*>(smem + C::kOffDl + sd * 512), p.delta, qh, i, 1.f, 0.f);
      if (lane == 0) {
        mbar_arrive(bar(B_LD(sd)));
        mbar_arrive_expect_tx(bar(B_DF(sd)), C::kStageBytes);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d(doAddr(sd) + pn * C::kHalfPanelBytes, &p.tm_do64, bar(B_DF(sd)), pn * 64,
                      i * 128 + 64 * static_cast<int>(rank), qh);
        tma_load_3d(doAddr(sd) + 2 * C::kHalfPanelBytes, &p.tm_do, bar(B_DF(sd)), 64 * static_cast<int>(rank),
                    i * 128, qh);
        ++issued_d;
      }
    }
    if (lane == 0 && *abort_flag) {
      st_shared_cluster_u32(peer_flag, 1u);
      // let the copies this CTA started land before it leaves (bounded)
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_KV), 0, drain, kSitePDrain);
      for (int q = (issued_q > NQ ? issued_q - NQ : 0); q < issued_q; ++q)
        mbar_wait(bar(B_QF(q % NQ)), (q / NQ) & 1, drain, kSitePDrain);
      for (int q = (issued_d > ND ? issued_d - ND : 0); q < issued_d; ++q)
        mbar_wait(bar(B_DF(q % ND)), (q / ND) & 1, drain, kSitePDrain);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (leader && lane == 0) {
      constexpr uint32_t kIdescKK = idesc_bf16_f32(256, 128, false, false);   // S^T, dP^T
      constexpr uint32_t kIdescTS = idesc_bf16_f32(256, D, false, true);      // dV, dK
      constexpr uint16_t kBoth = 0x3;
      // A = 128 rows (this CTA's keys) x d, both CTAs; B = 64 query rows x d per CTA
      auto gemm_kk = [&](uint32_t dcol, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_f16_ss_pair(tmem + dcol,
                          smem_desc_sw128(a_addr + (kk / 4) * C::kPanelBytes + (kk % 4) * 32, 16, 1024),
                          smem_desc_sw128(b_addr + (kk / 4) * C::kHalfPanelBytes + (kk % 4) * 32, 16, 1024),
                          kIdescKK, kk > 0 ? 1u : 0u);
        }
      };
      // A = packed P^T / dS^T (queries 0..63 at a_col, 64..127 at a_col + 64),
      // B = one 64-column d-panel of all 128 queries per CTA (MN-major)
      auto gemm_ts = [&](uint32_t dcol, uint32_t a_col, uint32_t b_addr, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts_pair(tmem + dcol, tmem + a_col + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                          smem_desc_sw128(b_addr + kk * 2048, C::kPanelBytes, 1024), kIdescTS,
                          (acc || kk > 0) ? 1u : 0u);
      };
      // an operand stage is ready when both CTAs' copies have landed
      auto both = [&](int own, int fwd, uint32_t parity, unsigned int site) -> bool {
        return mbar_wait(bar(own), parity, ab, site) && mbar_wait_cluster(bar(fwd), parity, ab, site);
      };
      bool ok = both(B_KV, B_KVP, 0, kSitePMmaKV);
      if (ok && n_it > 0 && (ok = both(B_QF(0), B_QFP(0), 0, kSitePMmaQ))) {
        tc_fence_after();
        gemm_kk(C::kColA, kAddr, qAddr(0));                       // S^T(0) = K Q^T
        tc_commit_pair(bar(B_S), kBoth);
      }
      for (int idx = 0; idx < n_it && ok; ++idx) {
        const int sq = idx % NQ, sd = idx % ND;
        if (!(ok = both(B_DF(sd), B_DFP(sd), (idx / ND) & 1, kSitePMmaQ))) break;
        tc_fence_after();
        gemm_kk(C::kColB, vAddr, doAddr(sd));                     // dP^T = V dO^T
        tc_commit_pair(bar(B_DP), kBoth);
        if (!(ok = mbar_wait_cluster(bar(B_P), idx & 1, ab, kSitePMmaP))) break;
        tc_fence_after();
        gemm_ts(C::kColDV, C::kColA, doAddr(sd) + 2 * C::kHalfPanelBytes, idx > 0);   // dV += P^T dO
        if (idx + 1 < n_it) {                                     // next S^T right behind dV
          const int s1 = (idx + 1) % NQ;
          if (!(ok = both(B_QF(s1), B_QFP(s1), ((idx + 1) / NQ) & 1, kSitePMmaQ))) break;
          tc_fence_after();
          gemm_kk(C::kColA, kAddr, qAddr(s1));
          tc_commit_pair(bar(B_S), kBoth);
        }
        if (!(ok = mbar_wait_cluster(bar(B_DS), idx & 1, ab, kSitePMmaDS))) break;
        tc_fence_after();
        gemm_ts(C::kColDK, C::kColB, qAddr(sq) + 2 * C::kHalfPanelBytes, idx > 0);    // dK += dS^T Q
        // dK is the last reader of Q_i and (after the dS phase) of L_i, D_i
        tc_commit_pair(bar(B_QE(sq)), kBoth);
        tc_commit_pair(bar(B_DE(sd)), kBoth);
      }
      tc_commit_pair(bar(B_FINAL), kBoth);
      tc_commit_pair(bar(B_DRAIN), kBoth);
      if (*abort_flag) st_shared_cluster_u32(peer_flag, 1u);
    } else if (!leader && lane == 0) {
      // rank 1: forward each of this CTA's completed operand stages to rank 0
      const uint32_t kvp = lead_bar(B_KVP);
      bool ok = mbar_wait(bar(B_KV), 0, ab, kSitePMmaKV);
      if (ok) mbar_arrive_cluster(kvp);
      for (int idx = 0; idx < n_it && ok; ++idx) {
        const int sq = idx % NQ, sd = idx % ND;
        if (!(ok = mbar_wait(bar(B_QF(sq)), (idx / NQ) & 1, ab, kSitePMmaQ))) break;
        mbar_arrive_cluster(lead_bar(B_QFP(sq)));
        if (!(ok = mbar_wait(bar(B_DF(sd)), (idx / ND) & 1, ab, kSitePMmaQ))) break;
        mbar_arrive_cluster(lead_bar(B_DFP(sd)));
      }
      if (*abort_flag) st_shared_cluster_u32(peer_flag, 1u);
    }
    __syncwarp();
    // both CTAs: every product of the pair done before TMEM is released
    if (lane == 0) {
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_DRAIN), 0, drain, kSitePDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P, dS (thread = key row)
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;
    const int key = j * 128 + r;
    const bool key_ok = key < p.N;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col_half = 64u * wg;
    const float cs = p.scale_log2;
    const uint32_t p_bar = lead_bar(B_P), ds_bar = lead_bar(B_DS);
    bool ok = true;
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx);
      const int sq = idx % NQ, sd = idx % ND;
      const float4* L4 = reinterpret_cast<const float4*>(smem + C::kOffL + sq * 512) + 16 * wg;
      const float4* D4 = reinterpret_cast<const float4*>(smem + C::kOffDl + sd * 512) + 16 * wg;
      // visible query columns c_lo <= c <= c_hi of this key (column c is
      // query i * 128 + c): at or after the key (causal), within the window,
      // none for a key past N
      const int c_lo = CAUSAL ? min(128, max(0, key - i * 128)) : 0;
      const int c_hi = !key_ok ? -1 : (CAUSAL ? min(127, key + p.window - i * 128) : 127);
      const float sl2 = p.alibi ? p.alibi[q_head(idx) % p.H] * 1.4426950408889634f : 0.f;
      const float dq0 = static_cast<float>(i * 128 + static_cast<int>(col_half) - key);
      const uint32_t tS = tmem + C::kColA + lane_off + col_half;
      const uint32_t tDP = tmem + C::kColB + lane_off + col_half;
      if (!(ok = mbar_wait_warp(bar(B_LQ(sq)), (idx / NQ) & 1, ab, kSitePSmL))) break;
      if (!(ok = mbar_wait_warp(bar(B_S), idx & 1, ab, kSitePSmS))) break;
      tc_fence_after();
      uint32_t pp[32];   // this thread's packed P^T row, kept for the dS phase
      {
        uint32_t u[64];
        tmem_ld64(tS, u);
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
            f2_unpack(exp2_sfu_f2(x01), pv[0], pv[1]);
            f2_unpack(exp2_sfu_f2(x23), pv[2], pv[3]);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int col = static_cast<int>(col_half) + 4 * c4 + t;
              pv[t] = (col < c_lo || col > c_hi) ? 0.f : pv[t];
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
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_bar);
      if (!(ok = mbar_wait_warp(bar(B_LD(sd)), (idx / ND) & 1, ab, kSitePSmL))) break;
      if (!(ok = mbar_wait_warp(bar(B_DP), idx & 1, ab, kSitePSmDP))) break;
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
            const float d0 = p0 * (__uint_as_float(dp[2 * c2 - 32 * h]) - dq[2 * t2]);
            const float d1 = p1 * (__uint_as_float(dp[2 * c2 + 1 - 32 * h]) - dq[2 * t2 + 1]);
            ds[c2] = pack_bf16x2(d0, d1);
          }
        }
      }
      tmem_st32(tDP, ds);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ds_bar);
    }
    if (ok) ok = mbar_wait_warp(bar(B_FINAL), 0, ab, kSitePEpi);
    ok = named_bar_and(1, 256, ok);
    if (ok) {
      // dV and dK of this CTA's 128 keys: wg 0 head-dim columns [0, 64), wg 1 [64, 128)
      tc_fence_after();
      const size_t g = (static_cast<size_t>(kvh) * p.N + (key_ok ? key : 0)) * D;
      const size_t kv_elems = static_cast<size_t>(p.BH / p.kv_group) * p.N * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {      // 0: dV, 1: dK (times scale)
        const uint32_t src = tmem + (which ? C::kColDK : C::kColDV) + lane_off;
        uint16_t* dst = (which ? p.dk : p.dv) + g;
        const float mul = which ? p.scale : 1.f;
        float* part = p.kv_part + (static_cast<size_t>(split) * 2 + which) * kv_elems + g;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ch = wg * 2 + cc;
          uint32_t u[32];
          tmem_ld32(src + 32 * ch, u);
          if (p.kv_split > 1) {
            if (key_ok) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                st_global_v4_pair(part + 32 * ch + 4 * q, __float_as_uint(__uint_as_float(u[4 * q]) * mul),
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
              st_global_v4_pair(dst + 32 * ch + 8 * q, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
    }
    if (threadIdx.x == 0 && *abort_flag) st_shared_cluster_u32(peer_flag, 1u);
  }

  tc_fence_before();
  cluster_sync_all();          // the pair's products, arrivals and copies are done in both CTAs
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kTmemCols);
  }
}

template <bool CAUSAL>
cudaError_t launch_pair_impl(const BwdParams& p, cudaStream_t stream) {
  cudaError_t e = set_smem_once<bwd_pair_kernel<CAUSAL>>(PairCfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  const unsigned pairs = static_cast<unsigned>((p.N + 255) / 256) * static_cast<unsigned>(p.BH / p.kv_group) *
                         static_cast<unsigned>(p.kv_split);
  bwd_pair_kernel<CAUSAL><<<2 * pairs, PairCfg::kThreads, PairCfg::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_pair(const BwdParams& p, bool causal, cudaStream_t stream) {
  return causal ? launch_pair_impl<true>(p, stream) : launch_pair_impl<false>(p, stream);
}

}  // namespace fa
