// Fused exact attention forward for sm_100a (bf16 in, fp32 accumulate), one
// 128-row query tile per work item with two score buffers.
//
// What it computes: O = softmax(scale * Q K^T [causal]) V and the per-row
// logsumexp L, as the standard definition ("FlashAttention" concept note,
// "How it works"), reached by the online softmax of "FlashAttention
// v1/v2/v3/v4: the librarian who never clears the desk" (online softmax
// section, eq. 2) with the division by l deferred to the end (lineage page,
// "FA2 (2023)", refinement 2) and conditional rescaling (librarian page,
// "FA4", idea 2; threshold kRescaleTau in log2 units).
//
// Why a second design: with two query tiles per CTA (fa_fwd_tile.cu) the
// tensor memory holds S_0, S_1, O_0, O_1 and nothing else at d = 128, so
// P is stored over the consumed scores and the next S of a tile cannot start
// before its P V product has read P: each tile's own two products sit between
// the end of its softmax and the start of the next one.  Here a CTA holds one
// query tile, so tensor memory has room for two score buffers and P in
// columns of its own:
//   [0,128)        S buffer 0       [128,256)   S buffer 1
//   [256,256+d)    O accumulator    [384,448)   P (packed bf16)
// S(j+2) is issued into the buffer of S(j) as soon as the softmax has read
// S(j) out, so the next scores are always ready when the softmax finishes a
// tile; the tensor core runs S(j+2) and P V(j) behind it.  The price is that
// every K/V tile is fetched from L2 for 128 query rows instead of 256 (L2 has
// the bandwidth: the two-tile kernel uses about an eighth of it).
//
// Persistent grid: one CTA per SM walks its share of the work items (causal:
// longest first, dealt out in rounds with every other round in reverse CTA
// order); the next item's Q load and first two S products run while the
// softmax warps write the current item's O.
// Roles (192 threads): warps 0-3 softmax and epilogue (thread r owns query
// row r = TMEM lane r; one softmax warp per SM sub-partition), warp 4 TMA
// producer, warp 5 TMEM owner and the single MMA-issuing thread.
//
// Measured on B200: slower than the two-tile kernel whenever that kernel has
// at least one work item per SM (B4 H16 N4096 d128 causal 776 vs 926
// TFLOPS: one softmax warp per sub-partition hides less latency than two,
// and splitting each row over two warps costs a row-maximum exchange per
// tile, 688), faster when it has fewer (B2 H8 N1024 d64 causal 105 vs 87:
// twice the CTAs); the library picks it for those problems.
//
// Causal: key j visible to query i iff j <= i; key tiles entirely above the
// diagonal are never loaded; the diagonal tile, the ragged key tail (zero
// filled by TMA) and the sliding-window edge are masked to -inf.
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

template <int D>
struct Q1Cfg {
  static constexpr int kPanels = D / 64;               // 128-byte swizzle panels per row (bf16)
  static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBlockM * D * 2;   // one 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 6 : 8;   // K/V ring
  static constexpr int kThreads = 192;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kTileBytes;
  static constexpr int kOffBar = kOffRing + kStages * kTileBytes;
  static constexpr int kNumBars = 10 + 2 * kStages;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // + base alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;      // + 128 * buffer
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColP = 384;
};
static_assert(Q1Cfg<128>::kSmemBytes <= 232448, "one-tile forward shared memory (d = 128)");
static_assert(Q1Cfg<64>::kSmemBytes <= 232448, "one-tile forward shared memory (d = 64)");

// barrier slots
constexpr int kBarQ = 0;        // Q landed
constexpr int kBarQFree = 1;    // the item's last S product is done (Q may be reloaded)
constexpr int kBarP = 2;        // P stored (128 arrivals)
constexpr int kBarPV = 3;       // P V done
constexpr int kBarOFree = 4;    // O read out by the epilogue (128 arrivals)
constexpr int kBarDrain = 5;
__device__ __forceinline__ int bar_s(int b) { return 6 + b; }       // S buffer b ready
__device__ __forceinline__ int bar_sfree(int b) { return 8 + b; }   // S buffer b read out (128 arrivals)
__device__ __forceinline__ int bar_full(int s) { return 10 + s; }
template <int NS> __device__ __forceinline__ int bar_empty(int s) { return 10 + NS + s; }

// wait-site codes reported in bits 8..15 of the status word
enum : unsigned int { kSiteQProd = 40, kSiteQProdQ, kSiteQMmaQ, kSiteQMmaFull, kSiteQMmaSfree, kSiteQMmaP,
                      kSiteQMmaO, kSiteQSmS, kSiteQSmPv, kSiteQEpi, kSiteQDrain };

struct Q1Item {
  int bh, kvh, qi, j_start, n;
};

// Work item o: query tile qi of flattened head bh.  Causal: the tiles with
// the most key tiles first over all heads; non-causal: head-major.
template <bool CAUSAL>
__device__ __forceinline__ Q1Item q1_item(const FwdParams& p, int n_q, int o) {
  Q1Item it;
  if constexpr (CAUSAL) {
    it.bh = o % p.BH;
    it.qi = n_q - 1 - o / p.BH;
  } else {
    it.bh = o / n_q;
    it.qi = o % n_q;
  }
  it.kvh = it.bh / p.kv_group;
  // sliding window (causal only): key blocks wholly left of the window are skipped
  it.j_start = CAUSAL ? max(0, it.qi * kBlockM - p.window) / kBlockN : 0;
  it.n = (CAUSAL ? min(it.qi + 1, p.n_kv) : p.n_kv) - it.j_start;
  return it;
}

// The k-th item of this CTA: rounds of gridDim.x items, every other round in
// reverse CTA order, so that with longest-first items the totals even out.
__device__ __forceinline__ int q1_my_item(int k) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// Ring order of one item's K/V tiles, shared by producer and MMA issuer:
// K(0), K(1), then per key tile j: K(j+2) (if any), V(j).
// Position q of an item with n key tiles -> (is_v, tile index).
__device__ __forceinline__ void q1_ring_tile(int n, int q, bool& is_v, int& jt) {
  const int pre = n < 2 ? n : 2;
  if (q < pre) {
    is_v = false;
    jt = q;
    return;
  }
  q -= pre;
  // per j: [K(j+2) if j + 2 < n] V(j); the first n - 2 key tiles carry a K
  const int with_k = n > 2 ? n - 2 : 0;
  if (q < 2 * with_k) {
    is_v = (q & 1) != 0;
    jt = is_v ? q / 2 : q / 2 + 2;
    return;
  }
  is_v = true;
  jt = with_k + (q - 2 * with_k);
}

template <int D, bool CAUSAL, int NPOLY, int DEG>
__global__ void __launch_bounds__(192, 1) fwd_q1_kernel(const __grid_constant__ FwdParams p) {
  using C = Q1Cfg<D>;
  constexpr int NS = C::kStages;
  constexpr int kWarpProd = 4;
  constexpr int kWarpMma = 5;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_q = p.n_kv;                       // query tiles per head (N_q = N_k)
  const int n_items = n_q * p.BH;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    mbar_init(bar(kBarQFree), 1);
    mbar_init(bar(kBarP), 128);
    mbar_init(bar(kBarPV), 1);
    mbar_init(bar(kBarOFree), 128);
    mbar_init(bar(kBarDrain), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(bar_s(b)), 1);
      mbar_init(bar(bar_sfree(b)), 128);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(bar_full(s)), 1);
      mbar_init(bar(bar_empty<NS>(s)), 1);
    }
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

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      int seq = 0, q_loads = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int o = q1_my_item(k);
        if (o >= n_items) break;
        const Q1Item it = q1_item<CAUSAL>(p, n_q, o);
        // Q of the previous item is free once its last S product is done
        if (k > 0 && !(ok = mbar_wait(bar(kBarQFree), (k - 1) & 1, ab, kSiteQProdQ))) break;
        mbar_arrive_expect_tx(bar(kBarQ), C::kTileBytes);
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(sbase + C::kOffQ + pn * C::kPanelBytes, &p.tm_q, bar(kBarQ), pn * 64, it.qi * kBlockM, it.bh);
        ++q_loads;
        for (int q = 0; q < 2 * it.n && ok; ++q) {
          bool is_v;
          int jt;
          q1_ring_tile(it.n, q, is_v, jt);
          const int s = seq % NS;
          if (!(ok = mbar_wait(bar(bar_empty<NS>(s)), ((seq / NS) & 1) ^ 1, ab, kSiteQProd))) break;
          mbar_arrive_expect_tx(bar(bar_full(s)), C::kTileBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(sbase + C::kOffRing + s * C::kTileBytes + pn * C::kPanelBytes, is_v ? &p.tm_v : &p.tm_k,
                        bar(bar_full(s)), pn * 64, (it.j_start + jt) * kBlockN, it.kvh);
          ++seq;
        }
      }
      if (*abort_flag) {
        // another role gave up: let every copy this thread started land first
        volatile int never = 0;
        const Abort drain{&never, p.status};
        if (q_loads > 0) mbar_wait(bar(kBarQ), (q_loads - 1) & 1, drain, kSiteQDrain);
        for (int q = (seq > NS ? seq - NS : 0); q < seq; ++q)
          mbar_wait(bar(bar_full(q % NS)), (q / NS) & 1, drain, kSiteQDrain);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = sbase + C::kOffQ;
      auto ring = [&](int s) -> uint32_t { return sbase + C::kOffRing + s * C::kTileBytes; };
      int seq = 0;
      // next ring tile: wait until it has landed, return its slot
      auto take = [&](int& slot) -> bool {
        slot = seq % NS;
        const bool r = mbar_wait(bar(bar_full(slot)), (seq / NS) & 1, ab, kSiteQMmaFull);
        ++seq;
        return r;
      };
      // S(gg) = Q K^T into buffer gg % 2, once the softmax has read S(gg - 2) out of it
      auto issue_s = [&](int gg, bool last) -> bool {
        const int b = gg & 1;
        if (gg >= 2 && !mbar_wait(bar(bar_sfree(b)), ((gg - 2) >> 1) & 1, ab, kSiteQMmaSfree)) return false;
        int s;
        if (!take(s)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
          mma_f16_ss(tmem + C::kColS + 128 * b, smem_desc_sw128(q_addr + off, 16, 1024),
                     smem_desc_sw128(ring(s) + off, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(bar_s(b)));
        tc_commit(bar(bar_empty<NS>(s)));
        if (last) tc_commit(bar(kBarQFree));
        return true;
      };
      int g = 0;   // key tiles of this CTA's earlier items: the S / P / P V sequence
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int o = q1_my_item(k);
        if (o >= n_items) break;
        const Q1Item it = q1_item<CAUSAL>(p, n_q, o);
        const int n = it.n;
        if (!(ok = mbar_wait(bar(kBarQ), k & 1, ab, kSiteQMmaQ))) break;
        if (!(ok = issue_s(g, n == 1))) break;
        if (n > 1 && !(ok = issue_s(g + 1, n == 2))) break;
        for (int j = 0; j < n && ok; ++j) {
          const int gg = g + j;
          if (j + 2 < n && !(ok = issue_s(gg + 2, j + 3 == n))) break;
          // P V(j): P stored, and (first tile of an item) O read out of the previous item
          if (!(ok = mbar_wait(bar(kBarP), gg & 1, ab, kSiteQMmaP))) break;
          if (j == 0 && k > 0 && !(ok = mbar_wait(bar(kBarOFree), (k - 1) & 1, ab, kSiteQMmaO))) break;
          int s;
          if (!(ok = take(s))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk)   // V is MN-major; P packs 2 keys per column
            mma_f16_ts(tmem + C::kColO, tmem + C::kColP + 8 * kk,
                       smem_desc_sw128(ring(s) + kk * 16 * 128, C::kPanelBytes, 1024), kIdescO,
                       (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(kBarPV));
          tc_commit(bar(bar_empty<NS>(s)));
        }
        g += n;
      }
      // every MMA issued above must be finished before TMEM is released
      tc_commit(bar(kBarDrain));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(kBarDrain), 0, drain, kSiteQDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;                    // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tO = tmem + C::kColO + lane_off;
    const uint32_t tP = tmem + C::kColP + lane_off;
    int g = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int o = q1_my_item(k);
      if (o >= n_items) break;
      const Q1Item it = q1_item<CAUSAL>(p, n_q, o);
      const int row = it.qi * kBlockM + r;
      const float c = p.scale_log2;
      float m_use = -INFINITY;
      float l = 0.f;
      for (int j = 0; j < it.n; ++j) {
        const int gg = g + j;
        const int b = gg & 1;
        const int jb = it.j_start + j;
        if (!(ok = mbar_wait_warp(bar(bar_s(b)), (gg >> 1) & 1, ab, kSiteQSmS))) break;
        tc_fence_after();
        uint32_t u[128];
        tmem_ld128(tmem + C::kColS + 128 * b + lane_off, u);
        tc_fence_before();
        mbar_arrive(bar(bar_sfree(b)));             // the buffer may take S(gg + 2)
        const bool masked = (CAUSAL && (jb == it.qi || jb * kBlockN < it.qi * kBlockM + kBlockM - 1 - p.window)) ||
                            ((jb + 1) * kBlockN > p.N) || p.alibi != nullptr;
        if (masked) {
          // scaled scores, -inf where the key is hidden or past N: column i
          // is visible iff lo <= i < hi
          const int key0 = jb * kBlockN;
          const int hi = (CAUSAL ? min(row + 1, p.N) : p.N) - key0;
          const int lo = CAUSAL ? row - p.window - key0 : 0;
          if (p.alibi != nullptr) {   // + this query head's slope log2(e) * -|key - row|
            const float sl2 = p.alibi[it.bh % p.H] * 1.4426950408889634f;
            const float dk = static_cast<float>(key0 - row);
#pragma unroll
            for (int i = 0; i < 128; ++i) {
              const bool vis = i >= lo && i < hi;
              const float bias = -sl2 * fabsf(dk + static_cast<float>(i));
              u[i] = __float_as_uint(vis ? fmaf(__uint_as_float(u[i]), c, bias) : -INFINITY);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 128; ++i) {
              const bool vis = i >= lo && i < hi;
              u[i] = __float_as_uint(vis ? __uint_as_float(u[i]) * c : -INFINITY);
            }
          }
        }
        float mt;
        {
          float a[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) a[q] = fmaxf(__uint_as_float(u[q]), __uint_as_float(u[8 + q]));
#pragma unroll
          for (int i = 16; i < 128; i += 16) {
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] = max3f(a[q], __uint_as_float(u[i + q]), __uint_as_float(u[i + 8 + q]));
          }
          mt = max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
          if (!masked) mt *= c;
        }
        const float m_new = fmaxf(m_use, mt);
        const bool need = m_new > m_use + kRescaleTau;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_sfu(m_use - m_new);
          m_use = m_new;
        }
        // a row that has seen only hidden keys so far (sliding window) keeps
        // m = -inf; its p must be 0, not exp2(-inf + inf)
        const float neg_m = m_use == -INFINITY ? 0.f : -m_use;
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        if (masked) {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float p0 = ex2_sfu(__uint_as_float(u[2 * i]) + neg_m);
            const float p1 = ex2_sfu(__uint_as_float(u[2 * i + 1]) + neg_m);
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
            u[i] = pack_bf16x2(p0, p1);
          }
        } else {
          const uint64_t c2 = f2_pack(c, c);
          const uint64_t nm2 = f2_pack(neg_m, neg_m);
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])), c2, nm2);
            const uint64_t p2 = ((i & 7) < NPOLY) ? exp2_poly_f2<DEG>(x2) : exp2_sfu_f2(x2);
            acc[i & 3] = f2_add(acc[i & 3], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            u[i] = pack_bf16x2(p0, p1);
          }
        }
        // P's columns and O are free once the previous P V is done (the last
        // one of the previous item for the first tile of an item)
        if (gg > 0) {
          if (!(ok = mbar_wait_warp(bar(kBarPV), (gg - 1) & 1, ab, kSiteQSmPv))) break;
          tc_fence_after();
        }
        tmem_st64(tP, *reinterpret_cast<uint32_t(*)[64]>(&u[0]));
        if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t w[32];
            tmem_ld32(tO + ch * 32, w);
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
            tmem_st32(tO + ch * 32, w);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(kBarP));
        float sum4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float lo, hi;
          f2_unpack(acc[q], lo, hi);
          sum4[q] = lo + hi;
        }
        l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      }
      g += it.n;
      if (ok) ok = mbar_wait_warp(bar(kBarPV), (g - 1) & 1, ab, kSiteQEpi);
      // the four warps take the epilogue (and the next item) together or not at all
      ok = named_bar_and(1, 128, ok);
      if (!ok) break;
      tc_fence_after();
      // ------------------------------------------------------------ epilogue
      // O / l from TMEM straight to global memory (each thread its own row);
      // TMEM O is free again after the loads
      const float inv_l = 1.f / l;
      uint16_t* orow = p.o + (static_cast<size_t>(it.bh) * p.N + (row < p.N ? row : 0)) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t w[32];
        tmem_ld32(tO + ch * 32, w);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(w[2 * i]) * inv_l, __uint_as_float(w[2 * i + 1]) * inv_l);
        if (row < p.N) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint16_t* dst = orow + ch * 32 + 8 * q;
            asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(pk[4 * q]),
                         "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                         : "memory");
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kBarOFree));
      if (row < p.N) p.lse[static_cast<size_t>(it.bh) * p.N + row] = (m_use + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool CAUSAL, int NPOLY, int DEG>
cudaError_t launch_q1(const FwdParams& p, cudaStream_t stream) {
  using C = Q1Cfg<D>;
  auto kern = fwd_q1_kernel<D, CAUSAL, NPOLY, DEG>;
  cudaError_t e = set_smem_once<fwd_q1_kernel<D, CAUSAL, NPOLY, DEG>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>(p.n_kv) * p.BH;
  const unsigned grid = static_cast<unsigned>(items > p.sms ? p.sms : items);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

template <int D, bool CAUSAL>
cudaError_t launch_q1_np(const FwdParams& p, cudaStream_t stream) {
  const bool deg4 = p.poly_deg == 4;
  switch (p.poly_pairs) {
    case 0: return launch_q1<D, CAUSAL, 0, 3>(p, stream);
    case 4: return deg4 ? launch_q1<D, CAUSAL, 4, 4>(p, stream) : launch_q1<D, CAUSAL, 4, 3>(p, stream);
    default: return deg4 ? launch_q1<D, CAUSAL, 2, 4>(p, stream) : launch_q1<D, CAUSAL, 2, 3>(p, stream);
  }
}

}  // namespace

cudaError_t launch_fwd_q1_bf16(const FwdParams& p, int d, bool causal, cudaStream_t stream) {
  if (d == 64) return causal ? launch_q1_np<64, true>(p, stream) : launch_q1_np<64, false>(p, stream);
  return causal ? launch_q1_np<128, true>(p, stream) : launch_q1_np<128, false>(p, stream);
}

}  // namespace fa
