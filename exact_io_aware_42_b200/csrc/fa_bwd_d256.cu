// Attention backward for head dim 256 on sm_100a: dQ, dK, dV.
//
// The gradient is the one of the d <= 128 kernels (fa_bwd.cu): P is rebuilt
// from the saved logsumexp, P = 2^(S c - L log2 e) ("FlashAttention"
// concept note, "How it works", recomputation), dV = P^T dO,
// dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q.
//
// At d = 256 a 128-key CTA cannot hold dK and dV side by side in TMEM
// (2 x 256 of its 512 columns) next to the S^T and dP^T tiles, and 128-row
// Q, dO, K, V tiles are 64 KB each.  So the work is split three ways; every
// kernel sums in a fixed order, and the result is reproducible:
//
//   kv kernel   two CTAs per (K/V head, key block of 128): role r = 0
//               computes dV, role r = 1 dK, each over the full d (N = 256
//               products, one 256-column TMEM accumulator).  Query blocks of
//               64 rows stream past; per block both roles compute S^T
//               (M = 128 keys, N = 64 queries, K_j resident); the dV role
//               then dV += P^T dO, the dK role dP^T = V dO^T (V_j resident
//               in that role only), dS and dK += dS^T Q.  TMEM: S^T 64,
//               dP^T 64 (dK role), accumulator 256 columns.  S^T is computed
//               twice: 1.25x the minimal tensor work of dK, dV.
//   dq kernel   one CTA per (query head, query block of 128): Q_i, dO_i
//               resident (64 KB each); key blocks of 64 stream past; per
//               block S and dP (N = 64 keys), dQ += dS K_j (N = 256).
//               TMEM: two S buffers of 64, dP 64, dQ 256 columns.
//   D           D = rowsum(dO o O) by the shared preprocessing kernel.
//
// Roles (320 threads) as in the d <= 128 kernels: warps 0-7 the P / dS
// phases and the epilogue (thread = TMEM lane; the two warpgroups split the
// 64 columns of a tile), warp 8 TMA producer, warp 9 TMEM owner and the
// MMA-issuing thread.  Every wait is bounded (fa_ptx.cuh).
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kD2 = 256;
constexpr int kP128 = 128 * 128;   // 128-row panel (64 elements x 128 rows), bytes
constexpr int kP64 = 64 * 128;     // 64-row panel

__device__ __forceinline__ void st_global_v4_d2(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// ================================================================== dq kernel
struct Dq256 {
  static constexpr int kTileQ = 4 * kP128;     // Q_i or dO_i: 128 rows x 256, 64 KB
  static constexpr int kTileK = 4 * kP64;      // K_j or V_j: 64 rows x 256, 32 KB
  static constexpr int kStagesK = 2;
  static constexpr int kStagesV = 1;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTileQ;
  static constexpr int kOffK = 2 * kTileQ;                       // + s * kTileK
  static constexpr int kOffV = kOffK + kStagesK * kTileK;        // + s * kTileK
  static constexpr int kOffBar = kOffV + kStagesV * kTileK;
  static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 6;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;     // + 64 * buffer
  static constexpr uint32_t kColDP = 128;
  static constexpr uint32_t kColDQ = 256;
};
static_assert(Dq256::kSmemBytes <= 232448, "d = 256 dQ kernel shared memory");

enum : unsigned int { kQ2Prod = 100, kQ2MmaQ, kQ2MmaK, kQ2MmaV, kQ2MmaDS, kQ2SmS, kQ2SmDP, kQ2Epi, kQ2Drain, kQ2Align };

template <bool CAUSAL>
__global__ void __launch_bounds__(320, 1) bwd_dq256_kernel(const __grid_constant__ BwdParams p) {
  using C = Dq256;
  constexpr int NK = C::kStagesK;
  constexpr int NV = C::kStagesV;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH | (kQ2Align << 8));
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
  // head-major non-causal; causal: longest first within groups of heads
  // (causal_q_order)
  int bh, i;
  if (CAUSAL) {
    causal_q_order(static_cast<int>(blockIdx.x), p.n_q, p.group_kv * p.kv_group, p.BH, bh, i);
  } else {
    bh = blockIdx.x / p.n_q;
    i = static_cast<int>(blockIdx.x % p.n_q);
  }
  const int n_kb = (p.N + 63) / 64;                   // 64-key blocks
  const int j_start = CAUSAL ? max(0, i * 128 - p.window) / 64 : 0;
  const int n_j = (CAUSAL ? min(2 * i + 2, n_kb) : n_kb) - j_start;
  const int kvh = bh / p.kv_group;

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
  auto kAddr = [&](int s) -> uint32_t { return sbase + C::kOffK + s * C::kTileK; };
  auto vAddr = [&](int s) -> uint32_t { return sbase + C::kOffV + s * C::kTileK; };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k64);
      tma_prefetch_desc(&p.tm_v64);
      mbar_arrive_expect_tx(bar(B_QDO), 2 * C::kTileQ);
      for (int pn = 0; pn < 4; ++pn) {
        tma_load_3d(qAddr + pn * kP128, &p.tm_q, bar(B_QDO), pn * 64, i * 128, bh);
        tma_load_3d(doAddr + pn * kP128, &p.tm_do, bar(B_QDO), pn * 64, i * 128, bh);
      }
      int nk = 0, nv = 0;
      bool ok = true;
      auto load_k = [&](int j) {
        const int sk = j % NK;
        if (!mbar_wait(bar(B_KE(sk)), ((j / NK) & 1) ^ 1, ab, kQ2Prod)) return false;
        mbar_arrive_expect_tx(bar(B_KF(sk)), C::kTileK);
        for (int pn = 0; pn < 4; ++pn)
          tma_load_3d(kAddr(sk) + pn * kP64, &p.tm_k64, bar(B_KF(sk)), pn * 64, (j_start + j) * 64, kvh);
        ++nk;
        return true;
      };
      auto load_v = [&](int j) {
        const int sv = j % NV;
        if (!mbar_wait(bar(B_VE(sv)), ((j / NV) & 1) ^ 1, ab, kQ2Prod)) return false;
        mbar_arrive_expect_tx(bar(B_VF(sv)), C::kTileK);
        for (int pn = 0; pn < 4; ++pn)
          tma_load_3d(vAddr(sv) + pn * kP64, &p.tm_v64, bar(B_VF(sv)), pn * 64, (j_start + j) * 64, kvh);
        ++nv;
        return true;
      };
      // V_j's slot is freed by dP_{j-1}, K_j's by dQ_{j-2}, which the MMA
      // issuer runs after it: past the first ring of K, V goes out first.
      for (int j = 0; j < n_j && ok; ++j) {
        if (j < NK) ok = load_k(j) && load_v(j);
        else ok = load_v(j) && load_k(j);
      }
      if (*abort_flag) {   // let the copies in flight land before the CTA leaves
        volatile int never = 0;
        const Abort drain{&never, p.status};
        mbar_wait(bar(B_QDO), 0, drain, kQ2Drain);
        for (int q = (nk > NK ? nk - NK : 0); q < nk; ++q) mbar_wait(bar(B_KF(q % NK)), (q / NK) & 1, drain, kQ2Drain);
        for (int q = (nv > NV ? nv - NV : 0); q < nv; ++q) mbar_wait(bar(B_VF(q % NV)), (q / NV) & 1, drain, kQ2Drain);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 64, false, false);    // S, dP: 64 keys
      constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, kD2, false, true);    // dQ: N = 256, K MN-major
      // 128 query rows (A, 16 KB panels) x 64 key rows (B, 8 KB panels), K = 256
      auto gemm_kk = [&](uint32_t dcol, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
        for (int kk = 0; kk < kD2 / 16; ++kk)
          mma_f16_ss(tmem + dcol, smem_desc_sw128(a_addr + (kk / 4) * kP128 + (kk % 4) * 32, 16, 1024),
                     smem_desc_sw128(b_addr + (kk / 4) * kP64 + (kk % 4) * 32, 16, 1024), kIdescKK,
                     kk > 0 ? 1u : 0u);
      };
      auto wait_k = [&](int j) { return mbar_wait(bar(B_KF(j % NK)), (j / NK) & 1, ab, kQ2MmaK); };
      auto wait_v = [&](int j) { return mbar_wait(bar(B_VF(j % NV)), (j / NV) & 1, ab, kQ2MmaV); };
      auto issue_s = [&](int j) {
        gemm_kk(C::kColS + 64 * (j & 1), qAddr, kAddr(j % NK));
        tc_commit(bar(B_S0 + (j & 1)));
      };
      auto issue_dp = [&](int j) {
        gemm_kk(C::kColDP, doAddr, vAddr(j % NV));
        tc_commit(bar(B_DP));
        tc_commit(bar(B_VE(j % NV)));
      };
      bool ok = mbar_wait(bar(B_QDO), 0, ab, kQ2MmaQ);
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
        if (!(ok = mbar_wait(bar(B_DS), j & 1, ab, kQ2MmaDS))) break;
        tc_fence_after();
        if (j + 1 < n_j) {
          if (!(ok = wait_v(j + 1))) break;
          tc_fence_after();
          issue_dp(j + 1);
        }
        const uint32_t a_col = C::kColS + 64 * (j & 1);
        const uint32_t k_addr = kAddr(j % NK);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // packed keys 0..31 at a_col, 32..63 at a_col + 32
          mma_f16_ts(tmem + C::kColDQ, tmem + a_col + (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8),
                     smem_desc_sw128(k_addr + kk * 2048, kP64, 1024), kIdescDQ, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_KE(j % NK)));
        if (j + 2 < n_j) {
          if (!(ok = wait_k(j + 2))) break;
          tc_fence_after();
          issue_s(j + 2);
        }
      }
      tc_commit(bar(B_FINAL));
      tc_commit(bar(B_DRAIN));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_DRAIN), 0, drain, kQ2Drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS, epilogue (thread = query row)
    // warpgroup wg takes keys [32 wg, 32 wg + 32) of every 64-key tile
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;
    const int q = i * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const size_t grow = static_cast<size_t>(bh) * p.N + (q < p.N ? q : 0);
    const float l2 = q < p.N ? p.lse[grow] * 1.4426950408889634f : INFINITY;   // rows past N: P = 0
    const float dlt = q < p.N ? p.delta[grow] : 0.f;
    const float cs = p.scale_log2;
    const float sl2 = p.alibi ? p.alibi[bh % p.H] * 1.4426950408889634f : 0.f;
    bool ok = true;
    for (int j = 0; j < n_j && ok; ++j) {
      const int t = j & 1;
      const uint32_t tS = tmem + C::kColS + 64 * t + lane_off + 32 * wg;
      const uint32_t tDP = tmem + C::kColDP + lane_off + 32 * wg;
      const int jb = j_start + j;
      const int kbase = jb * 64 + 32 * wg;
      // warp-uniform: some key of this strip past N, after a query of the
      // tile, or left of the window
      const bool edge = (CAUSAL && (kbase + 31 > i * 128 || kbase < i * 128 + 127 - p.window)) || kbase + 32 > p.N;
      if (!(ok = mbar_wait_warp(bar(B_S0 + t), (j >> 1) & 1, ab, kQ2SmS))) break;
      tc_fence_after();
      uint32_t u[32];
      tmem_ld32(tS, u);
      const float dk0 = static_cast<float>(kbase - q);
      auto p_row = [&](auto alibi_on) {
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float n0 = -l2, n1 = -l2;
          if constexpr (decltype(alibi_on)::value) {
            n0 -= sl2 * fabsf(dk0 + static_cast<float>(c));
            n1 -= sl2 * fabsf(dk0 + static_cast<float>(c + 1));
          }
          const uint64_t x = f2_fma(f2_pack(__uint_as_float(u[c]), __uint_as_float(u[c + 1])), f2_pack(cs, cs),
                                    f2_pack(n0, n1));
          float p0, p1;
          f2_unpack(exp2_sfu_f2(x), p0, p1);
          u[c] = __float_as_uint(p0);
          u[c + 1] = __float_as_uint(p1);
        }
      };
      if (p.alibi)
        p_row(std::true_type{});
      else
        p_row(std::false_type{});
      if (edge) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int key = kbase + c;
          if (key >= p.N || (CAUSAL && (key > q || key < q - p.window))) u[c] = 0u;
        }
      }
      if (!(ok = mbar_wait_warp(bar(B_DP), j & 1, ab, kQ2SmDP))) break;
      tc_fence_after();
      uint32_t ds[16];
      {
        uint32_t dp[32];
        tmem_ld32(tDP, dp);
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) {
          const float d0 = __uint_as_float(u[2 * c2]) * (__uint_as_float(dp[2 * c2]) - dlt);
          const float d1 = __uint_as_float(u[2 * c2 + 1]) * (__uint_as_float(dp[2 * c2 + 1]) - dlt);
          ds[c2] = pack_bf16x2(d0, d1);
        }
      }
      tmem_st16(tS, ds);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
    }
    if (ok) ok = mbar_wait_warp(bar(B_FINAL), 0, ab, kQ2Epi);
    ok = named_bar_and(1, 256, ok);
    if (ok) {
      // wg 0 writes head-dim columns [0, 128), wg 1 [128, 256)
      tc_fence_after();
      uint16_t* dst = p.dq + grow * kD2;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int ch = wg * 4 + cc;
        uint32_t v[32];
        tmem_ld32(tmem + C::kColDQ + lane_off + 32 * ch, v);
        uint32_t pk[16];
#pragma unroll
        for (int t2 = 0; t2 < 16; ++t2)
          pk[t2] = pack_bf16x2(__uint_as_float(v[2 * t2]) * p.scale, __uint_as_float(v[2 * t2 + 1]) * p.scale);
        if (q < p.N) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            st_global_v4_d2(dst + 32 * ch + 8 * w, pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
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

// ================================================================== kv kernel
struct Kv256 {
  static constexpr int kTileKV = 4 * kP128;    // K_j or V_j: 128 rows x 256, 64 KB
  static constexpr int kTileQ = 4 * kP64;      // Q_i or dO_i: 64 rows x 256, 32 KB
  static constexpr int kStagesQ = 2;
  static constexpr int kStagesD = 1;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileKV;
  static constexpr int kOffQ = 2 * kTileKV;                      // + s * kTileQ
  static constexpr int kOffDO = kOffQ + kStagesQ * kTileQ;       // + s * kTileQ
  static constexpr int kOffL = kOffDO + kStagesD * kTileQ;       // + s * 256: L log2 e of 64 queries
  static constexpr int kOffDl = kOffL + kStagesQ * 256;          // + s * 256: D (with the Q stage)
  static constexpr int kOffBar = kOffDl + kStagesQ * 256;
  // The dV role has no V tile: its 64 KB hold two more dO stages (three in
  // all); the dK role keeps one.
  static constexpr int kStagesDV = 3;
  static constexpr int kNumBars = 1 + 2 * kStagesQ + 2 * kStagesDV + 6;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColA = 0;      // S^T / P^T (64 query columns)
  static constexpr uint32_t kColB = 64;     // dP^T / dS^T
  static constexpr uint32_t kColAcc = 128;  // dV (role 0) or dK (role 1): 256 columns
};
static_assert(Kv256::kSmemBytes <= 232448, "d = 256 dK/dV kernel shared memory");

enum : unsigned int { kK2Prod = 110, kK2MmaKV, kK2MmaQ, kK2MmaP, kK2MmaDS, kK2SmS, kK2SmDP, kK2Epi, kK2Drain,
                      kK2Align };

template <bool CAUSAL>
__global__ void __launch_bounds__(320, 1) bwd_kv256_kernel(const __grid_constant__ BwdParams p) {
  using C = Kv256;
  constexpr int NQ = C::kStagesQ;
  constexpr int NDB = C::kStagesDV;   // dO barrier pairs (the deepest ring)
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH | (kK2Align << 8));
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  const int B_KV = 0;
  auto B_QF = [](int s) { return 1 + s; };
  auto B_QE = [](int s) { return 1 + NQ + s; };
  auto B_DF = [](int s) { return 1 + 2 * NQ + s; };
  auto B_DE = [](int s) { return 1 + 2 * NQ + NDB + s; };
  const int B_S = 1 + 2 * NQ + 2 * NDB, B_DP = B_S + 1, B_P = B_S + 2, B_DS = B_S + 3, B_FINAL = B_S + 4,
            B_DRAIN = B_S + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA -> (K/V head, split, key block j, role h: 0 dV, 1 dK); head-major
  // non-causal; causal: longest first within groups of K/V heads
  // (causal_kv_order), the two roles of a key block adjacent
  const int h = blockIdx.x & 1;
  const int rest = blockIdx.x >> 1;
  int kvh, split, j;
  if (CAUSAL) {
    causal_kv_order(rest, p.n_kv, p.kv_split, p.group_kv, p.BH / p.kv_group, kvh, split, j);
  } else {
    kvh = rest / (p.n_kv * p.kv_split);
    split = (rest / p.n_kv) % p.kv_split;
    j = rest % p.n_kv;
  }
  const int g_per = p.kv_group / p.kv_split;
  const int n_qb = (p.N + 63) / 64;                          // 64-query blocks
  const int i0 = CAUSAL ? 2 * j : 0;
  const int i_last = CAUSAL ? min(n_qb - 1, (j * 128 + 127 + p.window) / 64) : n_qb - 1;
  const int n_i = i_last - i0 + 1;
  const int n_it = n_i * g_per;
  auto q_block = [&](int idx) { return i0 + idx % n_i; };
  auto q_head = [&](int idx) { return kvh * p.kv_group + split * g_per + idx / n_i; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    for (int s = 0; s < NQ; ++s) {
      mbar_init(bar(B_QF(s)), 1);
      mbar_init(bar(B_QE(s)), 1);
    }
    for (int s = 0; s < NDB; ++s) {
      mbar_init(bar(B_DF(s)), 1);
      mbar_init(bar(B_DE(s)), 1);
    }
    mbar_init(bar(B_S), 1);
    mbar_init(bar(B_DP), 1);
    mbar_init(bar(B_P), 256);
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
  const uint32_t kAddr = sbase + C::kOffK, vAddr = sbase + C::kOffV;
  auto qAddr = [&](int s) -> uint32_t { return sbase + C::kOffQ + s * C::kTileQ; };
  // dO stages: 1 in the dK role; 3 in the dV role, stages 1 and 2 in the V region
  const int ND = h ? C::kStagesD : C::kStagesDV;
  auto doAddr = [&](int s) -> uint32_t {
    return sbase + (s == 0 ? C::kOffDO : C::kOffV + (s - 1) * C::kTileQ);
  };
  static_assert(2 * Kv256::kTileQ <= Kv256::kTileKV, "two dO stages fit in the V tile");

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    int issued_q = 0, issued_d = 0;
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q64);
      tma_prefetch_desc(&p.tm_do64);
      // V_j only in the dK role (dP^T = V dO^T)
      mbar_arrive_expect_tx(bar(B_KV), (h ? 2 : 1) * C::kTileKV);
      for (int pn = 0; pn < 4; ++pn) {
        tma_load_3d(kAddr + pn * kP128, &p.tm_k, bar(B_KV), pn * 64, j * 128, kvh);
        if (h) tma_load_3d(vAddr + pn * kP128, &p.tm_v, bar(B_KV), pn * 64, j * 128, kvh);
      }
    }
    // L (log2 units, +inf past N) and D (0 past N) of the 64 queries of
    // block idx, two per lane.  The next block's values are loaded into
    // registers right after this block's copies are issued, so their latency
    // runs while the warp waits for the next free slots instead of delaying
    // the next copies.
    auto fetch_rows = [&](int idx, float2& l2, float2& d2) {
      const int i = q_block(idx), qh = q_head(idx);
      float lv[2], dv[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int q = i * 64 + lane * 2 + t;
        const size_t g = static_cast<size_t>(qh) * p.N + q;
        lv[t] = q < p.N ? p.lse[g] * 1.4426950408889634f : INFINITY;
        dv[t] = q < p.N ? p.delta[g] : 0.f;
      }
      l2 = make_float2(lv[0], lv[1]);
      d2 = make_float2(dv[0], dv[1]);
    };
    float2 l_next = make_float2(0.f, 0.f), d_next = l_next;
    if (n_it > 0) fetch_rows(0, l_next, d_next);
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx), qh = q_head(idx);
      const int sq = idx % NQ, sd = idx % ND;
      bool w = true;
      if (lane == 0) w = mbar_wait(bar(B_QE(sq)), ((idx / NQ) & 1) ^ 1, ab, kK2Prod);
      if (!(ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0)) break;
      // L and D of the block live with the Q stage: both are read before
      // the dS phase ends, and the stage is released after dK, which follows it
      reinterpret_cast<float2*>(smem + C::kOffL + sq * 256)[lane] = l_next;
      reinterpret_cast<float2*>(smem + C::kOffDl + sq * 256)[lane] = d_next;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_QF(sq)), C::kTileQ);
        for (int pn = 0; pn < 4; ++pn)
          tma_load_3d(qAddr(sq) + pn * kP64, &p.tm_q64, bar(B_QF(sq)), pn * 64, i * 64, qh);
        ++issued_q;
        w = mbar_wait(bar(B_DE(sd)), ((idx / ND) & 1) ^ 1, ab, kK2Prod);
      }
      if (!(ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_DF(sd)), C::kTileQ);
        for (int pn = 0; pn < 4; ++pn)
          tma_load_3d(doAddr(sd) + pn * kP64, &p.tm_do64, bar(B_DF(sd)), pn * 64, i * 64, qh);
        ++issued_d;
      }
      if (idx + 1 < n_it) fetch_rows(idx + 1, l_next, d_next);
    }
    if (lane == 0 && *abort_flag) {
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_KV), 0, drain, kK2Drain);
      for (int q = (issued_q > NQ ? issued_q - NQ : 0); q < issued_q; ++q)
        mbar_wait(bar(B_QF(q % NQ)), (q / NQ) & 1, drain, kK2Drain);
      for (int q = (issued_d > ND ? issued_d - ND : 0); q < issued_d; ++q)
        mbar_wait(bar(B_DF(q % ND)), (q / ND) & 1, drain, kK2Drain);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 64, false, false);    // S^T, dP^T: 64 queries
      constexpr uint32_t kIdescTS = idesc_bf16_f32(128, kD2, false, true);    // dV, dK: N = 256
      // A = 128 key rows (16 KB panels), B = 64 query rows (8 KB panels), K = 256
      auto gemm_kk = [&](uint32_t dcol, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
        for (int kk = 0; kk < kD2 / 16; ++kk)
          mma_f16_ss(tmem + dcol, smem_desc_sw128(a_addr + (kk / 4) * kP128 + (kk % 4) * 32, 16, 1024),
                     smem_desc_sw128(b_addr + (kk / 4) * kP64 + (kk % 4) * 32, 16, 1024), kIdescKK,
                     kk > 0 ? 1u : 0u);
      };
      // A = packed P^T / dS^T (queries 0..31 at a_col, 32..63 at a_col + 32),
      // B = all four head-dim panels of the 64 query rows (MN-major)
      auto gemm_ts = [&](uint32_t dcol, uint32_t a_col, uint32_t b_addr, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ts(tmem + dcol, tmem + a_col + (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8),
                     smem_desc_sw128(b_addr + kk * 2048, kP64, 1024), kIdescTS,
                     (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(B_KV), 0, ab, kK2MmaKV);
      if (ok && n_it > 0 && (ok = mbar_wait(bar(B_QF(0)), 0, ab, kK2MmaQ))) {
        tc_fence_after();
        gemm_kk(C::kColA, kAddr, qAddr(0));
        tc_commit(bar(B_S));
      }
      for (int idx = 0; idx < n_it && ok; ++idx) {
        const int sq = idx % NQ, sd = idx % ND;
        if (!(ok = mbar_wait(bar(B_DF(sd)), (idx / ND) & 1, ab, kK2MmaQ))) break;
        tc_fence_after();
        if (h) {
          gemm_kk(C::kColB, vAddr, doAddr(sd));                  // dP^T = V dO^T
          tc_commit(bar(B_DP));
          tc_commit(bar(B_DE(sd)));                              // dO_i is read for the last time
        }
        // dV role: P^T is in region A; dK role: the P phase has read S^T
        if (!(ok = mbar_wait(bar(B_P), idx & 1, ab, kK2MmaP))) break;
        tc_fence_after();
        if (!h) {
          gemm_ts(C::kColAcc, C::kColA, doAddr(sd), idx > 0);    // dV += P^T dO
          tc_commit(bar(B_DE(sd)));                              // dO_i is read for the last time
          tc_commit(bar(B_QE(sq)));                              // Q_i (S^T) and its L rows (P phase) too
        }
        if (idx + 1 < n_it) {                                    // next S^T into region A
          const int s1 = (idx + 1) % NQ;
          if (!(ok = mbar_wait(bar(B_QF(s1)), ((idx + 1) / NQ) & 1, ab, kK2MmaQ))) break;
          tc_fence_after();
          gemm_kk(C::kColA, kAddr, qAddr(s1));
          tc_commit(bar(B_S));
        }
        if (h) {
          if (!(ok = mbar_wait(bar(B_DS), idx & 1, ab, kK2MmaDS))) break;
          tc_fence_after();
          gemm_ts(C::kColAcc, C::kColB, qAddr(sq), idx > 0);     // dK += dS^T Q
          tc_commit(bar(B_QE(sq)));
        }
      }
      tc_commit(bar(B_FINAL));
      tc_commit(bar(B_DRAIN));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(B_DRAIN), 0, drain, kK2Drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P, dS (thread = key row)
    // warpgroup wg takes query columns [32 wg, 32 wg + 32) of each block
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;
    const int key = j * 128 + r;
    const bool key_ok = key < p.N;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col_half = 32u * wg;
    const float cs = p.scale_log2;
    bool ok = true;
    for (int idx = 0; idx < n_it && ok; ++idx) {
      const int i = q_block(idx);
      const float2* L2 = reinterpret_cast<const float2*>(smem + C::kOffL + (idx % NQ) * 256) + 16 * wg;
      const float2* D2 = reinterpret_cast<const float2*>(smem + C::kOffDl + (idx % NQ) * 256) + 16 * wg;
      // visible query columns c_lo <= c <= c_hi (column c is query 64 i + c)
      const int c_lo = CAUSAL ? min(64, max(0, key - i * 64)) : 0;
      const int c_hi = !key_ok ? -1 : (CAUSAL ? min(63, key + p.window - i * 64) : 63);
      const float sl2 = p.alibi ? p.alibi[q_head(idx) % p.H] * 1.4426950408889634f : 0.f;
      const float dq0 = static_cast<float>(i * 64 + static_cast<int>(col_half) - key);
      const uint32_t tS = tmem + C::kColA + lane_off + col_half;
      const uint32_t tDP = tmem + C::kColB + lane_off + col_half;
      if (!(ok = mbar_wait_warp(bar(B_S), idx & 1, ab, kK2SmS))) break;
      tc_fence_after();
      uint32_t pp[16];   // packed P^T row, kept for the dS phase
      {
        uint32_t u[32];
        tmem_ld32(tS, u);
        auto p_rows = [&](auto alibi_on) {
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            const float2 l2 = L2[c2];
            float n0 = -l2.x, n1 = -l2.y;
            if constexpr (decltype(alibi_on)::value) {
              n0 -= sl2 * fabsf(dq0 + static_cast<float>(2 * c2));
              n1 -= sl2 * fabsf(dq0 + static_cast<float>(2 * c2 + 1));
            }
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(u[2 * c2]), __uint_as_float(u[2 * c2 + 1])),
                                      f2_pack(cs, cs), f2_pack(n0, n1));
            float p0, p1;
            f2_unpack(exp2_sfu_f2(x), p0, p1);
            const int col = static_cast<int>(col_half) + 2 * c2;
            p0 = (col < c_lo || col > c_hi) ? 0.f : p0;
            p1 = (col + 1 < c_lo || col + 1 > c_hi) ? 0.f : p1;
            pp[c2] = pack_bf16x2(p0, p1);
          }
        };
        if (p.alibi)
          p_rows(std::true_type{});
        else
          p_rows(std::false_type{});
        if (!h) tmem_st16(tS, pp);   // P^T for dV; the dK role keeps P in registers only
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_P));
      if (!h) continue;
      if (!(ok = mbar_wait_warp(bar(B_DP), idx & 1, ab, kK2SmDP))) break;
      tc_fence_after();
      uint32_t ds[16];
      {
        uint32_t dp[32];
        tmem_ld32(tDP, dp);
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) {
          const float2 d2 = D2[c2];
          const float p0 = __uint_as_float(pp[c2] << 16), p1 = __uint_as_float(pp[c2] & 0xFFFF0000u);
          ds[c2] = pack_bf16x2(p0 * (__uint_as_float(dp[2 * c2]) - d2.x), p1 * (__uint_as_float(dp[2 * c2 + 1]) - d2.y));
        }
      }
      tmem_st16(tDP, ds);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_DS));
    }
    if (ok) ok = mbar_wait_warp(bar(B_FINAL), 0, ab, kK2Epi);
    ok = named_bar_and(1, 256, ok);
    if (ok) {
      // dV (role 0) or dK (role 1, times scale) of this CTA's keys: wg 0
      // columns [0, 128), wg 1 [128, 256)
      tc_fence_after();
      const size_t g = (static_cast<size_t>(kvh) * p.N + (key_ok ? key : 0)) * kD2;
      const size_t kv_elems = static_cast<size_t>(p.BH / p.kv_group) * p.N * kD2;
      {
        const int which = h;
        const uint32_t src = tmem + C::kColAcc + lane_off;
        uint16_t* dst = (which ? p.dk : p.dv) + g;
        const float mul = which ? p.scale : 1.f;
        float* part = p.kv_part + (static_cast<size_t>(split) * 2 + which) * kv_elems + g;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int ch = wg * 4 + cc;
          uint32_t u[32];
          tmem_ld32(src + 32 * ch, u);
          if (p.kv_split > 1) {
            if (key_ok) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                st_global_v4_d2(part + 32 * ch + 4 * q, __float_as_uint(__uint_as_float(u[4 * q]) * mul),
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
              st_global_v4_d2(dst + 32 * ch + 8 * q, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
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

}  // namespace

cudaError_t launch_bwd_kv256(const BwdParams& p, bool causal, cudaStream_t stream) {
  const unsigned grid = 2u * static_cast<unsigned>(p.n_kv) * static_cast<unsigned>(p.BH / p.kv_group) *
                        static_cast<unsigned>(p.kv_split);
  cudaError_t e;
  if (causal) {
    if ((e = set_smem_once<bwd_kv256_kernel<true>>(Kv256::kSmemBytes)) != cudaSuccess) return e;
    bwd_kv256_kernel<true><<<grid, 320, Kv256::kSmemBytes, stream>>>(p);
  } else {
    if ((e = set_smem_once<bwd_kv256_kernel<false>>(Kv256::kSmemBytes)) != cudaSuccess) return e;
    bwd_kv256_kernel<false><<<grid, 320, Kv256::kSmemBytes, stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq256(const BwdParams& p, bool causal, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(p.n_q) * static_cast<unsigned>(p.BH);
  cudaError_t e;
  if (causal) {
    if ((e = set_smem_once<bwd_dq256_kernel<true>>(Dq256::kSmemBytes)) != cudaSuccess) return e;
    bwd_dq256_kernel<true><<<grid, 320, Dq256::kSmemBytes, stream>>>(p);
  } else {
    if ((e = set_smem_once<bwd_dq256_kernel<false>>(Dq256::kSmemBytes)) != cudaSuccess) return e;
    bwd_dq256_kernel<false><<<grid, 320, Dq256::kSmemBytes, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fa
