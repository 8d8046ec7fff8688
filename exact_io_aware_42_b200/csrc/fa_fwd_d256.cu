// Fused exact attention forward for head dim 256 on sm_100a (bf16 in, fp32
// accumulate).  Computes the same O and logsumexp L as the d <= 128 kernel
// (fa_fwd_tile.cu) by the same online softmax ("FlashAttention v1/v2/v3/v4: the
// librarian who never clears the desk", online softmax section, eq. 2;
// deferred normalisation, lineage page "FA2 (2023)", refinement 2); the
// librarian page lists d = 256 among the head dims FlashAttention serves
// ("Cases where FlashAttention does not help").
//
// What changes at d = 256 is the on-chip budget.  A 128-row O accumulator
// takes 256 of the 512 TMEM columns, so a CTA holds ONE query tile, and the
// other 256 columns hold two score buffers: S(j + 1) is computed while the
// softmax works on S(j), and P(j) V runs while the softmax works on S(j + 1).
// A 128 x 256 bf16 tile is 64 KB, so K and V stream through a ring of
// 16 KB panels (128 keys x 64 head-dim elements, one 128-byte swizzle
// panel each): S(j) = sum over the 4 panels p of Q_p K_{j,p}^T, and
// O[:, 64 p .. 64 p + 63] += P(j) V_{j,p} (N = 64 per product).
//
// Roles (320 threads):
//   warps 0-7  softmax and the epilogue: thread = query row = TMEM lane;
//              warpgroup wg takes key columns [64 wg, 64 wg + 64) of every
//              score tile and O columns [128 wg, 128 wg + 128).  The two
//              warps of a row exchange partial row maxima through shared
//              memory, so both take the same max and rescale decision, and
//              keep partial row sums that are added at the epilogue.
//   warp  8    TMA producer: Q (4 panels), then the key blocks' panels in
//              the order the products consume them: K(0), K(1), V(0), K(2),
//              V(1), ... into the panel ring (full/empty mbarriers)
//   warp  9    allocates TMEM; one thread issues every tcgen05.mma
// TMEM: [0,128) and [128,256) score buffers (each warpgroup packs its 64
// P values as bf16 pairs over the first 32 of its own 64 columns),
// [256,512) O.
//
// The grid is persistent: one CTA per SM walks its share of the (b, h,
// query tile) items, longest first when causal, in snake order.  Causal
// tiles above the diagonal are never loaded; the diagonal block, key tails
// past N, window edges and ALiBi take the masked path, as at d <= 128.
// Conditional rescaling with the stale-max threshold kRescaleTau as in
// fa_fwd_tile.cu.  Every wait is bounded (fa_ptx.cuh).
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

struct F256 {
  static constexpr int D = 256;
  static constexpr int kPanels = 4;                  // 64-element panels of a row
  static constexpr int kPanelBytes = 128 * 128;      // 128 rows x 128 bytes
  static constexpr int kStages = 10;                 // panel ring
  static constexpr int kThreads = 320;
  static constexpr int kOffQ = 0;                    // 4 panels
  static constexpr int kOffRing = kPanels * kPanelBytes;
  static constexpr int kOffBar = kOffRing + kStages * kPanelBytes;
  static constexpr int kNumBars = 10 + 2 * kStages;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffRed = kOffMisc + 16;      // partial row maxima / sums: [2 slots][2 wg][128] fp32
  static constexpr int kSmemBytes = kOffRed + 2 * 2 * 128 * 4;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;      // + 128 * buffer
  static constexpr uint32_t kColO = 256;
};
static_assert(F256::kSmemBytes <= 232448, "d = 256 forward shared memory");

// barrier slots
constexpr int kBarQ = 0, kBarQFree = 1, kBarP = 2, kBarPV = 4, kBarOFree = 5, kBarDrain = 6;   // slot 3 unused
__device__ __forceinline__ int bar_s256(int b) { return 7 + b; }                 // S buffer b written
__device__ __forceinline__ int bar_full256(int s) { return 10 + s; }
__device__ __forceinline__ int bar_empty256(int s) { return 10 + F256::kStages + s; }

enum : unsigned int { kS2ProdEmpty = 60, kS2ProdQ, kS2MmaQ, kS2MmaFull, kS2MmaP, kS2MmaO, kS2SmS, kS2SmPv,
                      kS2EpiPv, kS2Drain, kS2Align };

__device__ __forceinline__ void st_global_v4_256(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

struct Item256 {
  int bh, kvh, qt, j_start, n;
};

// Work item o: one 128-row query tile.  Causal: the longest tiles of every
// head first; non-causal: head-major.
template <bool CAUSAL>
__device__ __forceinline__ Item256 item256_at(const FwdParams& p, int o) {
  const int n_qt = p.n_kv;          // query tiles = key blocks (N_q = N_k)
  Item256 it;
  it.bh = CAUSAL ? o % p.BH : o / n_qt;
  it.qt = CAUSAL ? n_qt - 1 - o / p.BH : o % n_qt;
  it.kvh = it.bh / p.kv_group;
  it.j_start = CAUSAL ? max(0, it.qt * kBlockM - p.window) / kBlockN : 0;
  it.n = (CAUSAL ? min(it.qt + 1, p.n_kv) : p.n_kv) - it.j_start;
  return it;
}

__device__ __forceinline__ int my_item256(int k) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  return k * G + ((k & 1) ? G - 1 - c : c);
}

template <bool CAUSAL, int NPOLY, int DEG>
__global__ void __launch_bounds__(F256::kThreads, 1) fwd256_kernel(const __grid_constant__ FwdParams p) {
  using C = F256;
  constexpr int NS = C::kStages;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {   // the swizzled layouts need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(p.status, 0u, FA_ERR_LAUNCH | (kS2Align << 8));
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = p.n_kv * p.BH;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    mbar_init(bar(kBarQFree), 1);
    mbar_init(bar(kBarP), 256);
    mbar_init(bar(kBarPV), 1);
    mbar_init(bar(kBarOFree), 256);
    mbar_init(bar(kBarDrain), 1);
    for (int b = 0; b < 2; ++b) mbar_init(bar(bar_s256(b)), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(bar_full256(s)), 1);
      mbar_init(bar(bar_empty256(s)), 1);
    }
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

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      int seq = 0, q_loads = 0;
      bool ok = true;
      // the 4 panels of K (w = 0) or V (w = 1) of key block jb into the ring
      auto load_block = [&](const CUtensorMap* m, int jb, int kvh) -> bool {
        for (int pn = 0; pn < C::kPanels; ++pn) {
          const int s = seq % NS;
          if (!mbar_wait(bar(bar_empty256(s)), ((seq / NS) & 1) ^ 1, ab, kS2ProdEmpty)) return false;
          mbar_arrive_expect_tx(bar(bar_full256(s)), C::kPanelBytes);
          tma_load_3d(sbase + C::kOffRing + s * C::kPanelBytes, m, bar(bar_full256(s)), pn * 64, jb * kBlockN, kvh);
          ++seq;
        }
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int o = my_item256(k);
        if (o >= n_items) break;
        const Item256 it = item256_at<CAUSAL>(p, o);
        if (k > 0 && !(ok = mbar_wait(bar(kBarQFree), (k - 1) & 1, ab, kS2ProdQ))) break;
        mbar_arrive_expect_tx(bar(kBarQ), C::kPanels * C::kPanelBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(sbase + C::kOffQ + pn * C::kPanelBytes, &p.tm_q, bar(kBarQ), pn * 64, it.qt * kBlockM, it.bh);
        ++q_loads;
        // consumption order of the products: K(0), K(1), V(0), K(2), V(1), ...
        ok = load_block(&p.tm_k, it.j_start, it.kvh);
        for (int j = 0; j < it.n && ok; ++j) {
          if (j + 1 < it.n) ok = load_block(&p.tm_k, it.j_start + j + 1, it.kvh);
          if (ok) ok = load_block(&p.tm_v, it.j_start + j, it.kvh);
        }
      }
      if (*abort_flag) {   // let every copy this thread started land before the CTA exits
        volatile int never = 0;
        const Abort drain{&never, p.status};
        if (q_loads > 0) mbar_wait(bar(kBarQ), (q_loads - 1) & 1, drain, kS2Drain);
        const int first = seq > NS ? seq - NS : 0;
        for (int q = first; q < seq; ++q) mbar_wait(bar(bar_full256(q % NS)), (q / NS) & 1, drain, kS2Drain);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, 64, false, true);   // one 64-column O panel
      int seq = 0;      // ring slots consumed
      int gS = 0;       // S products issued (all items): buffer gS % 2
      int gP = 0;       // P V products issued (all items)
      bool ok = true;
      // S(gS) = Q K_j^T over the 4 head-dim panels into buffer gS % 2; the K
      // panels' slots are released when the products are done.
      auto issue_s = [&]() -> bool {
        const int b = gS & 1;
        int slot[C::kPanels];
        for (int pn = 0; pn < C::kPanels; ++pn) {
          slot[pn] = seq % NS;
          if (!mbar_wait(bar(bar_full256(slot[pn])), (seq / NS) & 1, ab, kS2MmaFull)) return false;
          ++seq;
        }
        tc_fence_after();
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          const uint32_t qa = sbase + C::kOffQ + pn * C::kPanelBytes;
          const uint32_t ka = sbase + C::kOffRing + slot[pn] * C::kPanelBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmem + C::kColS + 128 * b, smem_desc_sw128(qa + kk * 32, 16, 1024),
                       smem_desc_sw128(ka + kk * 32, 16, 1024), kIdescS, (pn > 0 || kk > 0) ? 1u : 0u);
          // this panel's slot is free once its 4 products are done, so the
          // next block's panels can load while the rest of S(j) runs
          tc_commit(bar(bar_empty256(slot[pn])));
        }
        tc_commit(bar(bar_s256(b)));
        ++gS;
        return true;
      };
      // O += P(gP) V_j once both warpgroups have stored their P and
      // rescaled their O columns: keys [64 h, 64 h + 64) from warpgroup h's
      // packed P, each half over the 4 V panels (64 O columns each).
      auto issue_pv = [&](bool acc) -> bool {
        const int b = gP & 1;
        int slot[C::kPanels];
        for (int pn = 0; pn < C::kPanels; ++pn) {
          slot[pn] = seq % NS;
          if (!mbar_wait(bar(bar_full256(slot[pn])), (seq / NS) & 1, ab, kS2MmaFull)) return false;
          ++seq;
        }
        if (!mbar_wait(bar(kBarP), gP & 1, ab, kS2MmaP)) return false;
        tc_fence_after();
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn) {
            const uint32_t va = sbase + C::kOffRing + slot[pn] * C::kPanelBytes;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              const int kk = 4 * h + kq;     // 16 keys per product
              mma_f16_ts(tmem + C::kColO + 64 * pn, tmem + C::kColS + 128 * b + 64 * h + 8 * kq,
                         smem_desc_sw128(va + kk * 16 * 128, C::kPanelBytes, 1024), kIdescO,
                         (acc || kk > 0) ? 1u : 0u);
            }
            if (h == 1) tc_commit(bar(bar_empty256(slot[pn])));   // V panel read by both halves
          }
        }
        tc_commit(bar(kBarPV));
        ++gP;
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int o = my_item256(k);
        if (o >= n_items) break;
        const Item256 it = item256_at<CAUSAL>(p, o);
        if (!(ok = mbar_wait(bar(kBarQ), k & 1, ab, kS2MmaQ))) break;
        // S(0); the previous item's last P V precedes it on the tensor pipe
        if (!(ok = issue_s())) break;
        if (it.n == 1) tc_commit(bar(kBarQFree));
        for (int j = 0; j < it.n && ok; ++j) {
          if (j + 1 < it.n) {
            if (!(ok = issue_s())) break;               // S(j + 1) while the softmax works on S(j)
            if (j + 2 == it.n) tc_commit(bar(kBarQFree));
          }
          if (j == 0 && k > 0 && !(ok = mbar_wait(bar(kBarOFree), (k - 1) & 1, ab, kS2MmaO))) break;
          ok = issue_pv(j > 0);
        }
      }
      tc_commit(bar(kBarDrain));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(kBarDrain), 0, drain, kS2Drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int wg = warp >> 2;
    const int r = threadIdx.x & 127;            // query row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + C::kColO + lane_off + 128u * wg;   // this warpgroup's O columns
    const uint32_t pair_bar = 2 + (warp & 3);   // warps w and w + 4 share rows
    float* red = reinterpret_cast<float*>(smem + C::kOffRed);
    auto red_at = [&](int slot, int w) -> float& { return red[(slot * 2 + w) * 128 + r]; };
    int g = 0;         // score tiles over all items: buffer g % 2, barrier phases
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int o = my_item256(k);
      if (o >= n_items) break;
      const Item256 it = item256_at<CAUSAL>(p, o);
      const int bh = it.bh;
      const int qi = it.qt;
      const int row = qi * kBlockM + r;
      const float c = p.scale_log2;
      float m_use = -INFINITY;
      float l = 0.f;    // this warpgroup's share of the row sum
      for (int j = 0; j < it.n; ++j) {
        const int jb = it.j_start + j;
        const int gj = g + j;
        const int b = gj & 1;
        const uint32_t tS = tmem + C::kColS + 128 * b + 64u * wg + lane_off;
        const bool masked = (CAUSAL && (jb == qi || jb * kBlockN < qi * kBlockM + kBlockM - 1 - p.window)) ||
                            ((jb + 1) * kBlockN > p.N) || p.alibi != nullptr;
        uint32_t u[64];
        float mt = -INFINITY;
        const bool ws = mbar_wait_warp(bar(bar_s256(b)), (gj >> 1) & 1, ab, kS2SmS);
        if (ws) {
          tc_fence_after();
          tmem_ld64(tS, u);
          if (masked) {
            const int key0 = jb * kBlockN + 64 * wg;
            const int hi = (CAUSAL ? min(row + 1, p.N) : p.N) - key0;
            const int lo = CAUSAL ? row - p.window - key0 : 0;
            if (p.alibi != nullptr) {
              const float sl2 = p.alibi[bh % p.H] * 1.4426950408889634f;
              const float dk = static_cast<float>(key0 - row);
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const bool vis = i >= lo && i < hi;
                const float bias = -sl2 * fabsf(dk + static_cast<float>(i));
                u[i] = __float_as_uint(vis ? fmaf(__uint_as_float(u[i]), c, bias) : -INFINITY);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const bool vis = i >= lo && i < hi;
                u[i] = __float_as_uint(vis ? __uint_as_float(u[i]) * c : -INFINITY);
              }
            }
          }
          float a8[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) a8[q] = fmaxf(__uint_as_float(u[q]), __uint_as_float(u[8 + q]));
#pragma unroll
          for (int i = 16; i < 64; i += 16) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              a8[q] = max3f(a8[q], __uint_as_float(u[i + q]), __uint_as_float(u[i + 8 + q]));
          }
          mt = max3f(max3f(a8[0], a8[1], a8[2]), max3f(a8[3], a8[4], a8[5]), fmaxf(a8[6], a8[7]));
          if (!masked) mt *= c;
          red_at(b, wg) = mt;
        }
        // both warps of the row pair leave together if either wait failed
        if (!(ok = named_bar_and(pair_bar, 64, ws))) break;
        const float m_new = fmaxf(m_use, fmaxf(mt, red_at(b, wg ^ 1)));
        const bool need = m_new > m_use + kRescaleTau;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_sfu(m_use - m_new);
          m_use = m_new;
        }
        const float neg_m = m_use == -INFINITY ? 0.f : -m_use;
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        const uint64_t c2 = f2_pack(c, c);
        const uint64_t nm2 = f2_pack(neg_m, neg_m);
        if (masked) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2_sfu(__uint_as_float(u[2 * i]) + neg_m);
            const float p1 = ex2_sfu(__uint_as_float(u[2 * i + 1]) + neg_m);
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
            u[i] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])), c2, nm2);
            const uint64_t p2 = ((i & 7) < NPOLY) ? exp2_poly_f2<DEG>(x2) : exp2_sfu_f2(x2);
            acc[i & 3] = f2_add(acc[i & 3], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            u[i] = pack_bf16x2(p0, p1);
          }
        }
        tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        bool wpv = true;
        if (j > 0) {
          // P(j-1) V must be done before O is rescaled or P(j) is released
          wpv = mbar_wait_warp(bar(kBarPV), (gj - 1) & 1, ab, kS2SmPv);
          if (wpv) {
            tc_fence_after();
            if (__any_sync(0xffffffffu, need)) {
#pragma unroll
              for (int ch = 0; ch < 4; ++ch) {
                uint32_t w[32];
                tmem_ld32(tO + ch * 32, w);
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
                tmem_st32(tO + ch * 32, w);
              }
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        if (wpv) mbar_arrive(bar(kBarP));
        float sum4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float lo, hi;
          f2_unpack(acc[q], lo, hi);
          sum4[q] = lo + hi;
        }
        l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
        // a failed wait ends the loop at the next pair barrier or the epilogue's
        ok = wpv;
      }
      g += it.n;
      if (ok) ok = mbar_wait_warp(bar(kBarPV), (g - 1) & 1, ab, kS2EpiPv);
      ok = named_bar_and(1, 256, ok);
      if (!ok) break;
      tc_fence_after();
      // row sum over both halves; the slot of the item's last tile is free
      // (both warps read its maxima before the barrier above)
      const int ls = (g - 1) & 1;
      red_at(ls, wg) = l;
      named_bar_sync(pair_bar, 64);
      const float l_all = red_at(ls, 0) + red_at(ls, 1);
      // epilogue: this warpgroup's 128 O columns / l from TMEM to global memory
      const float inv_l = 1.f / l_all;
      uint16_t* orow = p.o + (static_cast<size_t>(bh) * p.N + (row < p.N ? row : 0)) * D + 128 * wg;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t w[32];
        tmem_ld32(tO + ch * 32, w);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(w[2 * i]) * inv_l, __uint_as_float(w[2 * i + 1]) * inv_l);
        if (row < p.N) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_global_v4_256(orow + ch * 32 + 8 * q, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kBarOFree));
      if (wg == 0 && row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + row] = (m_use + log2f(l_all)) * 0.69314718055994531f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <bool CAUSAL, int NPOLY, int DEG>
cudaError_t launch256(const FwdParams& p, cudaStream_t stream) {
  cudaError_t e = set_smem_once<fwd256_kernel<CAUSAL, NPOLY, DEG>>(F256::kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>(p.n_kv) * p.BH;
  const unsigned grid = static_cast<unsigned>(p.persistent && items > p.sms ? p.sms : items);
  fwd256_kernel<CAUSAL, NPOLY, DEG><<<grid, F256::kThreads, F256::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

template <bool CAUSAL>
cudaError_t launch256_np(const FwdParams& p, cudaStream_t stream) {
  const bool deg4 = p.poly_deg == 4;
  switch (p.poly_pairs) {
    case 0: return launch256<CAUSAL, 0, 3>(p, stream);
    case 4: return deg4 ? launch256<CAUSAL, 4, 4>(p, stream) : launch256<CAUSAL, 4, 3>(p, stream);
    default: return deg4 ? launch256<CAUSAL, 2, 4>(p, stream) : launch256<CAUSAL, 2, 3>(p, stream);
  }
}

}  // namespace

cudaError_t launch_fwd_d256(const FwdParams& p, bool causal, cudaStream_t stream) {
  return causal ? launch256_np<true>(p, stream) : launch256_np<false>(p, stream);
}

}  // namespace fa
