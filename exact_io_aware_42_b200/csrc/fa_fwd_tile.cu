// Fused exact attention forward for sm_100a, two 128-row query tiles per
// work item (bf16 or E4M3 in, fp32 accumulate): the kernel for d = 64 and
// 128, run with one CTA per work item or as a persistent grid (PERS).
//
// What it computes: O = softmax(scale * Q K^T [causal]) V and the per-row
// logsumexp L, exactly as the standard definition ("FlashAttention" concept
// note, "How it works"), reached by the online softmax of "FlashAttention
// v1/v2/v3/v4: the librarian who never clears the desk" (online softmax
// section, eq. 2): per K/V tile the running max m and sum l are updated, the
// running output is rescaled by 2^(m_old - m_new), and the division by l is
// deferred to the end (lineage page, "FA2 (2023)", refinement 2).
//
// Work unit: one CTA owns two 128-row query tiles of one (b, h) and streams
// every needed 128-key K/V tile once for both (each K/V tile is read from
// L2/HBM once per 256 query rows).  One CTA per work item: the hardware
// hands CTAs to SMs in index order as SMs free up, which with the items
// ordered longest first is a dynamic longest-first schedule, and O leaves
// through shared memory and a TMA store.  Persistent (PERS): min(items, SMs)
// CTAs walk the items (causal: a longest-processing-time-first deal made on
// the host; otherwise, or for tables too large, rounds in snake order); one
// item's last products overlap the
// next item's Q and K/V copies (Q_t is reloaded as soon as the item's last
// S_t product has read it) and its first S products, and O is written from
// registers.  Roles:
//   warps 0-3  softmax for query tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q tiles, then K_0, V_0, K_1, V_1, ... into a
//              ring of 128 x d shared-memory tiles (full/empty mbarriers)
//   warp  9    allocates TMEM; one thread issues every tcgen05.mma
// TMEM (512 columns x 128 lanes, fp32):
//   [0,128)    S_0 (tile 0 scores); after softmax the first 64 columns hold
//              P_0 as packed bf16 pairs, read back as the A operand of P V
//   [128,256)  S_1 / P_1
//   [256,256+d)        O_0 accumulator
//   [256+d,256+2d)     O_1 accumulator
// MMA order per key tile j:  PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), so each
// softmax warpgroup works on its tile while the tensor core runs the other
// tile's two products (the lineage page's "pingpong" idea, "FA3 (2024)",
// carried by two TMEM-resident tiles instead of two register warpgroups).
// With P over S, S_t(j+1) cannot start before P V_t(j) has read P_t(j), so
// each tile's softmax waits for its own two products every key tile.  At
// d = 64 the O accumulators leave 128 columns free, P_t gets
//   [384 + 64 t, 448 + 64 t)   P_t (d = 64)
// and S_t(j+1) is issued as soon as the softmax has read S_t(j) out (before
// its exponentials): S_0(j+1), S_1(j+1), PV_0(j), PV_1(j).
//
// Conditional rescaling (librarian page, "FA4", idea 2): a row keeps its
// stale max m until a new tile's max exceeds it by more than kRescaleTau
// (log2 units).  p = 2^(x - m) is then at most 2^tau, the same stale m is
// used for p, l, O and L, and the result is unchanged up to rounding.  The
// O rescale in TMEM runs only for warps where some row moved its max.
//
// Causal: key j visible to query i iff j <= i.  Tiles entirely above the
// diagonal are never loaded or multiplied; only the diagonal tile and the
// ragged key tail (keys >= N, zero-filled by TMA) are masked to -inf.
#include <algorithm>
#include <cstring>
#include <numeric>
#include <type_traits>
#include <vector>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

// Persistent causal grid: each CTA's work items, dealt by the host longest
// processing time first (every item to the CTA with the least work so far,
// items in order of decreasing cost), passed as a kernel parameter.  With
// more items or CTAs than the table holds (n = 0) the kernel deals in snake
// order instead.
constexpr int kSchedMaxItems = 8192;
constexpr int kSchedMaxCtas = 256;
struct FwdSched {
  int n;                                   // items in the table (0: none)
  uint16_t off[kSchedMaxCtas + 1];         // CTA c: item[off[c] .. off[c + 1])
  uint16_t item[kSchedMaxItems];
};
struct FwdSchedNone {};

template <int D, bool FP8 = false>
struct TileCfg {
  static constexpr int kElem = FP8 ? 1 : 2;            // bytes per Q/K/V element
  static constexpr int kPanels = D * kElem / 128;      // 128-byte swizzle panels per row
  static constexpr int kPanelElems = 128 / kElem;      // elements per panel row
  static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBlockM * D * kElem;   // one 128 x D tile
  static constexpr int kStages = FP8 ? 8 : ((D == 128) ? 5 : 8);
  static constexpr int kThreads = 320;
  static constexpr int kOffQ = 0;                      // two query tiles
  // bf16 O is staged in the Q tile it replaces; FP8 tiles are half as large,
  // so FP8 stages O in a buffer of its own (2 x 128 x D bf16).
  static constexpr int kOffO = FP8 ? 2 * kTileBytes : 0;
  static constexpr int kOBytes = kBlockM * D * 2;
  static constexpr int kOffRing = FP8 ? kOffO + 2 * kOBytes : 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + kStages * kTileBytes;
  static constexpr int kNumBars = 2 + 2 * kStages + 11;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 48 + 1024;   // + base alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;       // + 128 * t
  static constexpr uint32_t kColO = 256;     // + D * t
  // d = 64: P_t in a region of its own at kColP + 64 t (see the kernel notes);
  // d = 128 has no room for it and stores P over the consumed S_t
  static constexpr bool kSepP = (D == 64);
  static constexpr uint32_t kColP = 384;
  // P outside S: S_t(j+1) may start as soon as S_t(j) has been read out
  static constexpr bool kEarlyS = kSepP;
};
static_assert(TileCfg<128, true>::kSmemBytes <= 232448, "fp8 forward shared memory");
static_assert(TileCfg<128, false>::kSmemBytes <= 232448, "bf16 forward shared memory");

// barrier slots
__device__ __forceinline__ int bar_q(int t) { return t; }
template <int NS> __device__ __forceinline__ int bar_full(int s) { return 2 + s; }
template <int NS> __device__ __forceinline__ int bar_empty(int s) { return 2 + NS + s; }
template <int NS> __device__ __forceinline__ int bar_s(int t) { return 2 + 2 * NS + t; }
template <int NS> __device__ __forceinline__ int bar_p(int t) { return 4 + 2 * NS + t; }
template <int NS> __device__ __forceinline__ int bar_pv(int t) { return 6 + 2 * NS + t; }
template <int NS> __device__ __forceinline__ int bar_drain() { return 8 + 2 * NS; }
template <int NS> __device__ __forceinline__ int bar_sfree(int t) { return 9 + 2 * NS + t; }   // S_t read out
// persistent grid: the last S_t product of an item has read Q_t
template <int NS> __device__ __forceinline__ int bar_qfree(int t) { return 11 + 2 * NS + t; }

// wait-site codes reported in bits 8..15 of the status word
enum : unsigned int { kSiteProdEmpty = 1, kSiteMmaQ, kSiteMmaFull, kSiteMmaP, kSiteSmS, kSiteSmPv,
                      kSiteEpiPv, kSiteDrain, kSiteMmaSfree };

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// E4M3 byte pair <- (lo, hi), round to nearest even, saturating at +-448.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  unsigned short lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// NPOLY of every 8 column pairs take the polynomial exp2 (degree DEG), the
// rest the SFU.  FP8: Q, K, V are E4M3 with per-128-row block scales and both
// products run as kind::f8f6f4 (see the FP8 notes at the softmax).
// ALIBI: the bias of p.alibi (a separate build, so that the plain kernel
// carries none of its code).
// PERS: a persistent grid of at most one CTA per SM walks the work items
// (sch: the causal deal, see FwdSched), so that one item's end overlaps the
// next item's copies and first products; O is then written from registers
// (the Q buffer takes the next item's Q early).
template <int D, bool CAUSAL, int NPOLY, int DEG, bool FP8, bool ALIBI, bool PERS = false>
using SchedFor = std::conditional_t<PERS && CAUSAL, FwdSched, FwdSchedNone>;

template <int D, bool CAUSAL, int NPOLY, int DEG, bool FP8, bool ALIBI, bool PERS = false>
__global__ void __launch_bounds__(320, 1) fwd_tile_kernel(
    const __grid_constant__ FwdParams p, const __grid_constant__ SchedFor<D, CAUSAL, NPOLY, DEG, FP8, ALIBI, PERS> sch) {
  using C = TileCfg<D, FP8>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Causal: within each group of group_heads heads, the heaviest pairs first
  // (longest-first balances the uneven work; the hardware hands out CTAs in
  // index order as SMs free up, so group boundaries cost no balance, and a
  // group's K and V stay in L2 while its CTAs run).  Non-causal: head-major,
  // so the resident CTAs cover a few heads whose K and V stay in L2.
  struct Item {
    int bh, kvh, qt0, j_start, n0, n1;   // n_t: key blocks of query tile t
  };
  auto item_at = [&](int o) -> Item {
    Item it;
    int pair;
    if constexpr (CAUSAL) {
      const int per_group = p.group_heads * p.n_pairs;
      const int g = o / per_group;
      const int rr = o - g * per_group;
      const int gh = min(p.group_heads, p.BH - g * p.group_heads);   // the last group may be short
      it.bh = g * p.group_heads + rr % gh;
      pair = p.n_pairs - 1 - rr / gh;
    } else {
      it.bh = o / p.n_pairs;
      pair = o % p.n_pairs;
    }
    // Grouped K/V heads: query head h of batch b reads K/V head b * H_kv + h / G,
    // which in the flattened [B * H] index is bh / G.
    it.kvh = it.bh / p.kv_group;
    it.qt0 = 2 * pair;
    // Sliding window (causal only): key j is visible to query i iff
    // i - window <= j <= i.  Key blocks wholly left of tile 0's window are
    // never loaded; both tiles start at the same block (tile 1's first block
    // may then be fully masked for it, which the softmax handles).
    it.j_start = CAUSAL ? max(0, it.qt0 * kBlockM - p.window) / kBlockN : 0;
    it.n0 = (CAUSAL ? min(it.qt0 + 1, p.n_kv) : p.n_kv) - it.j_start;
    it.n1 = (CAUSAL ? min(it.qt0 + 2, p.n_kv) : p.n_kv) - it.j_start;
    return it;
  };
  // The k-th item of this CTA (n_items when there is none): one item per CTA,
  // or, persistent, rounds of gridDim.x items, every other round in reverse
  // CTA order, so that with longest-first items the CTAs' totals even out.
  const int n_items = p.n_pairs * p.BH;
  auto my_item = [&](int k) -> int {
    if constexpr (PERS) {
      const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
      if constexpr (CAUSAL) {
        if (sch.n > 0) {
          const int i = sch.off[c] + k;
          return i < sch.off[c + 1] ? static_cast<int>(sch.item[i]) : n_items;
        }
      }
      return k * G + ((k & 1) ? G - 1 - c : c);
    } else {
      return k == 0 ? static_cast<int>(blockIdx.x) : n_items;
    }
  };
  // the first item (its copies start before the CTA-wide sync); the
  // persistent bf16 build decodes every item afresh in the role loops, which
  // keeps fewer values live across them
  const Item it0 = item_at(my_item(0));

  // The producer thread initialises the barriers and starts the copies of
  // Q_0, K(0), Q_1 and the rest of the first ring round before the CTA-wide
  // sync, so that their latency overlaps the TMEM allocation and the sync
  // (no other thread touches a barrier before the sync).
  // ring copy number seq (over the CTA's items) is copy c of item it: K(c / 2) or V(c / 2)
  auto load_kv = [&](int seq, const Item& it, int c) {
    const int s = seq % NS;
    mbar_arrive_expect_tx(bar(bar_full<NS>(s)), C::kTileBytes);
    const CUtensorMap* m = (c & 1) ? &p.tm_v : &p.tm_k;
    for (int pn = 0; pn < C::kPanels; ++pn)
      tma_load_3d(sbase + C::kOffRing + s * C::kTileBytes + pn * C::kPanelBytes, m, bar(bar_full<NS>(s)),
                  pn * C::kPanelElems, (it.j_start + c / 2) * kBlockN, it.kvh);
  };
  auto load_q = [&](int t, const Item& it) {
    mbar_arrive_expect_tx(bar(bar_q(t)), C::kTileBytes);
    for (int pn = 0; pn < C::kPanels; ++pn)
      tma_load_3d(sbase + C::kOffQ + t * C::kTileBytes + pn * C::kPanelBytes, &p.tm_q, bar(bar_q(t)),
                  pn * C::kPanelElems, (it.qt0 + t) * kBlockM, it.bh);
  };
  // ring copies of the first item that need no free slot
  const int n_first = it0.bh < p.BH ? min(NS, 2 * it0.n1) : 0;
  if (warp == 8 && lane == 0) {
    mbar_init(bar(bar_q(0)), 1);
    mbar_init(bar(bar_q(1)), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(bar_full<NS>(s)), 1);
      mbar_init(bar(bar_empty<NS>(s)), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(bar_s<NS>(t)), 1);
      mbar_init(bar(bar_p<NS>(t)), 128);
      mbar_init(bar(bar_pv<NS>(t)), 1);
      mbar_init(bar(bar_sfree<NS>(t)), 128);
      mbar_init(bar(bar_qfree<NS>(t)), 1);
    }
    mbar_init(bar(bar_drain<NS>()), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    if (n_first > 0) {
      load_q(0, it0);
      load_kv(0, it0, 0);
      load_q(1, it0);
      for (int sq = 1; sq < n_first; ++sq) load_kv(sq, it0, sq);
    }
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
      int seq = n_first;   // the first ring round went out before the sync
      int nq[2] = {n_first > 0 ? 1 : 0, n_first > 0 ? 1 : 0};   // Q loads issued per tile
      bool ok = true;
      for (int k = 0; ok && (PERS || k == 0); ++k) {
        const int o = my_item(k);
        if (o >= n_items) break;
        const Item it = ((!PERS || FP8) && k == 0) ? it0 : item_at(o);
        const int seq0 = (k == 0) ? 0 : seq;   // this item's first ring copy
        // Q_t of this item once the previous item's last S_t has read the
        // buffer: Q_0, K(0), Q_1, then the rest of the item's K and V
        if (nq[0] == k) {
          if (k > 0 && !(ok = mbar_wait(bar(bar_qfree<NS>(0)), (k - 1) & 1, ab, kSiteProdEmpty))) break;
          load_q(0, it);
          ++nq[0];
        }
        for (; seq < seq0 + 2 * it.n1; ++seq) {
          if (!(ok = mbar_wait(bar(bar_empty<NS>(seq % NS)), ((seq / NS) & 1) ^ 1, ab, kSiteProdEmpty))) break;
          load_kv(seq, it, seq - seq0);
          if (nq[1] == k) {
            if (k > 0 && !(ok = mbar_wait(bar(bar_qfree<NS>(1)), (k - 1) & 1, ab, kSiteProdEmpty))) {
              ++seq;   // the copy above went out
              break;
            }
            load_q(1, it);
            ++nq[1];
          }
        }
      }
      if (*abort_flag) {
        // Another role gave up: let every copy this thread started land before
        // the CTA exits (bounded, ignoring the abort flag).
        volatile int never = 0;
        const Abort drain{&never, p.status};
        for (int t = 0; t < 2; ++t)
          if (nq[t] > 0) mbar_wait(bar(bar_q(t)), (nq[t] - 1) & 1, drain, kSiteDrain);
        const int first = seq > NS ? seq - NS : 0;
        for (int q = first; q < seq; ++q)
          mbar_wait(bar(bar_full<NS>(q % NS)), (q / NS) & 1, drain, kSiteDrain);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS =
          FP8 ? idesc_e4m3_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescO =
          FP8 ? idesc_e4m3_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
      constexpr int kK = FP8 ? 32 : 16;            // K elements per MMA (32 bytes)
      const uint32_t q_addr[2] = {sbase + C::kOffQ, sbase + C::kOffQ + C::kTileBytes};
      auto ring = [&](int s) -> uint32_t { return sbase + C::kOffRing + s * C::kTileBytes; };
      auto issue_s = [&](int t, uint32_t k_addr) {
#pragma unroll
        for (int kk = 0; kk < D / kK; ++kk) {
          const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
          const uint64_t a = smem_desc_sw128(q_addr[t] + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(k_addr + off, 16, 1024);
          if constexpr (FP8)
            mma_f8_ss(tmem + C::kColS + 128 * t, a, b, kIdescS, kk > 0 ? 1u : 0u);
          else
            mma_f16_ss(tmem + C::kColS + 128 * t, a, b, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(bar_s<NS>(t)));
      };
      auto issue_pv = [&](int t, uint32_t v_addr, bool acc) {
#pragma unroll
        for (int kk = 0; kk < kBlockN / kK; ++kk) {
          // V is MN-major (d contiguous); one K step is kK key rows of 128 bytes.
          // P in TMEM packs 32 bits per column: 2 bf16 or 4 E4M3 keys.
          const uint64_t b = smem_desc_sw128(v_addr + kk * kK * 128, C::kPanelBytes, 1024);
          if constexpr (FP8)
            mma_f8_ts(tmem + C::kColO + D * t, tmem + C::kColS + 128 * t + kk * 8, b, kIdescO,
                      (acc || kk > 0) ? 1u : 0u);
          else
            mma_f16_ts(tmem + C::kColO + D * t,
                       tmem + (C::kSepP ? C::kColP + 64 * t : C::kColS + 128 * t) + kk * 8, b, kIdescO,
                       (acc || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(bar_pv<NS>(t)));
      };
      // Phases: bar_s, bar_p, bar_sfree and bar_pv of tile t complete once per
      // key block of that tile, counted over the CTA's items (g[t] before
      // the current item); bar_q once per item.  With a persistent grid the
      // previous item's last P V products precede an item's first S products
      // on the tensor pipe, and the softmax has read S_t out before it
      // released the last P_t, so the S regions are free.
      int seq = 0;
      int g[2] = {0, 0};
      bool ok = true;
      for (int k = 0; ok && (PERS || k == 0); ++k) {
        const int o = my_item(k);
        if (o >= n_items) break;
        const Item it = ((!PERS || FP8) && k == 0) ? it0 : item_at(o);
        const int n_t[2] = {it.n0, it.n1};
        const int n_iter = it.n1;
        // S_0(0) as soon as Q_0 and K(0) are in, S_1(0) once Q_1 is
        int ks = seq % NS;
        if (!(ok = mbar_wait(bar(bar_q(0)), k & 1, ab, kSiteMmaQ) &&
                   mbar_wait(bar(bar_full<NS>(ks)), (seq / NS) & 1, ab, kSiteMmaFull)))
          break;
        ++seq;
        tc_fence_after();
        issue_s(0, ring(ks));
        if (PERS && n_t[0] == 1) tc_commit(bar(bar_qfree<NS>(0)));   // Q_0 may be replaced
        if (!(ok = mbar_wait(bar(bar_q(1)), k & 1, ab, kSiteMmaQ))) break;
        tc_fence_after();
        issue_s(1, ring(ks));
        if (PERS && n_t[1] == 1) tc_commit(bar(bar_qfree<NS>(1)));
        tc_commit(bar(bar_empty<NS>(ks)));
        for (int j = 0; j < n_iter && ok; ++j) {
          const int vs = seq % NS;
          if (!(ok = mbar_wait(bar(bar_full<NS>(vs)), (seq / NS) & 1, ab, kSiteMmaFull))) break;
          ++seq;
          const bool has_next = j + 1 < n_iter;
          if (has_next) {
            ks = seq % NS;
            if (!(ok = mbar_wait(bar(bar_full<NS>(ks)), (seq / NS) & 1, ab, kSiteMmaFull))) break;
            ++seq;
          }
          const int ph0 = (g[0] + j) & 1, ph1 = (g[1] + j) & 1;
          tc_fence_after();
          if constexpr (C::kEarlyS) {
            // S_t(j+1) as soon as the softmax has read S_t(j) out (P_t(j) is
            // elsewhere), then the P V products as P arrives
            if (has_next) {
              if (j + 1 < n_t[0]) {
                if (!(ok = mbar_wait(bar(bar_sfree<NS>(0)), ph0, ab, kSiteMmaSfree))) break;
                tc_fence_after();
                issue_s(0, ring(ks));
                if (PERS && j + 2 == n_t[0]) tc_commit(bar(bar_qfree<NS>(0)));
              }
              if (!(ok = mbar_wait(bar(bar_sfree<NS>(1)), ph1, ab, kSiteMmaSfree))) break;
              tc_fence_after();
              issue_s(1, ring(ks));
              if (PERS && j + 2 == n_t[1]) tc_commit(bar(bar_qfree<NS>(1)));
              tc_commit(bar(bar_empty<NS>(ks)));
            }
            if (j < n_t[0]) {
              if (!(ok = mbar_wait(bar(bar_p<NS>(0)), ph0, ab, kSiteMmaP))) break;
              tc_fence_after();
              issue_pv(0, ring(vs), j > 0);
            }
            if (!(ok = mbar_wait(bar(bar_p<NS>(1)), ph1, ab, kSiteMmaP))) break;
            tc_fence_after();
            issue_pv(1, ring(vs), j > 0);
            tc_commit(bar(bar_empty<NS>(vs)));
          } else {
            if (j < n_t[0]) {
              if (!(ok = mbar_wait(bar(bar_p<NS>(0)), ph0, ab, kSiteMmaP))) break;
              tc_fence_after();
              issue_pv(0, ring(vs), j > 0);
              if (j + 1 < n_t[0]) {
                issue_s(0, ring(ks));
                if (PERS && j + 2 == n_t[0]) tc_commit(bar(bar_qfree<NS>(0)));
              }
            }
            if (!(ok = mbar_wait(bar(bar_p<NS>(1)), ph1, ab, kSiteMmaP))) break;
            tc_fence_after();
            issue_pv(1, ring(vs), j > 0);
            tc_commit(bar(bar_empty<NS>(vs)));
            if (has_next) {
              issue_s(1, ring(ks));
              if (PERS && j + 2 == n_t[1]) tc_commit(bar(bar_qfree<NS>(1)));
              tc_commit(bar(bar_empty<NS>(ks)));
            }
          }
        }
        g[0] += n_t[0];
        g[1] += n_t[1];
      }
      // Every MMA issued above must be finished before TMEM is released,
      // also when a role gave up part-way.
      tc_commit(bar(bar_drain<NS>()));
      volatile int never = 0;
      const Abort drain{&never, p.status};
      mbar_wait(bar(bar_drain<NS>()), 0, drain, kSiteDrain);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;                 // query tile of this warpgroup
    const int r = threadIdx.x - 128 * t;     // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + C::kColS + 128 * t + lane_off;
    const uint32_t tO = tmem + C::kColO + D * t + lane_off;
    const uint32_t tP = tmem + C::kColP + 64 * t + lane_off;   // d = 64 only
    int gs = 0;   // key blocks of this tile in earlier items: the S and P V barriers' phase base
    bool ok = true;
    for (int k = 0; ok && (PERS || k == 0); ++k) {
      const int o = my_item(k);
      if (o >= n_items) break;
      const Item it = ((!PERS || FP8) && k == 0) ? it0 : item_at(o);
      const int bh = it.bh, kvh = it.kvh, j_start = it.j_start;
      const int qi = it.qt0 + t;
      const int row = qi * kBlockM + r;
      const int n = t ? it.n1 : it.n0;
      // FP8: scores are dequantised per tile pair with s_q(i) * s_k(j); P is
      // stored as E4M3 times 256 * s_v(j) / max_j s_v(j), which folds V's block
      // scale into P (p <= 2^0.75 because FP8 rescales once the max has grown by
      // more than kRescaleTauFp8, so P <= 430.5 < 448), and O is multiplied back
      // by max s_v / 256 at the end.
      const size_t sc_base = static_cast<size_t>(bh) * p.n_kv;      // Q's block scales
      const size_t kv_base = static_cast<size_t>(kvh) * p.n_kv;     // K's and V's
      float c_q = p.scale_log2;
      float v_max = 1.f;
      float sk_next = 1.f, sv_next = 1.f;
      if constexpr (FP8) {
        c_q *= (qi < p.n_kv) ? p.sq[sc_base + qi] : 1.f;
        // max over this head's V block scales: strided over the warpgroup's
        // 128 threads, then a shuffle and a shared-memory reduction
        float vm = 0.f;
        for (int jj = r; jj < p.n_kv; jj += 128) vm = fmaxf(vm, p.sv[kv_base + jj]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
        float* red = reinterpret_cast<float*>(smem + C::kOffMisc + 8) + 4 * t;   // 4 floats per tile
        if (lane == 0) red[warp & 3] = vm;
        named_bar_sync(1 + t, 128);
        v_max = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        sk_next = p.sk[kv_base + j_start];
        sv_next = p.sv[kv_base + j_start];
      }
      constexpr float kTau = FP8 ? kRescaleTauFp8 : kRescaleTau;
      float m_use = -INFINITY;
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int jb = j_start + j;      // key block; j counts this tile's iterations
        if (!(ok = mbar_wait_warp(bar(bar_s<NS>(t)), (gs + j) & 1, ab, kSiteSmS))) break;
        tc_fence_after();
        uint32_t u[128];
        tmem_ld128(tS, u);
        if constexpr (C::kEarlyS) {   // S_t may be overwritten by S_t(j+1) from here on
          tc_fence_before();
          mbar_arrive(bar(bar_sfree<NS>(t)));
        }
        const float c = c_q * sk_next;   // FP8: dequantise with s_q(i) s_k(j); bf16: sk_next = 1
        const float sv_j = sv_next;
        if constexpr (FP8) {             // next tile's scales, loaded while this one is processed
          if (j + 1 < n) {
            sk_next = p.sk[kv_base + jb + 1];
            sv_next = p.sv[kv_base + jb + 1];
          }
        }
        // ALiBi sends every block through this path: the bias is added to the
        // scaled scores before the row maximum is taken.
        // edge: the diagonal tile, the window's edge, the key tail (and with
        // ALiBi the diagonal tile, where keys lie on both sides of a row)
        const bool edge = (CAUSAL && (jb == qi || jb * kBlockN < qi * kBlockM + kBlockM - 1 - p.window)) ||
                          ((jb + 1) * kBlockN > p.N) || (ALIBI && jb == qi);
        // ALiBi off the diagonal tile: every key lies on the same side of every
        // row, so the bias -slope |key - row| is linear in the column
        const bool alibi_lin = ALIBI && !edge;
        const bool masked = edge || alibi_lin;   // u holds scaled (biased) scores
        if (alibi_lin) {
          const float sl2 = p.alibi[bh % p.H] * 1.4426950408889634f;
          const int key0 = jb * kBlockN;
          const float b0 = -sl2 * fabsf(static_cast<float>(key0 - row));
          const float bs = jb < qi ? sl2 : -sl2;
          const uint64_t c2 = f2_pack(c, c), bs2 = f2_pack(bs, bs), b02 = f2_pack(b0, b0);
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const uint64_t bias2 =
                f2_fma(bs2, f2_pack(static_cast<float>(2 * i), static_cast<float>(2 * i + 1)), b02);
            const uint64_t r2 = f2_fma(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])), c2, bias2);
            float r0, r1;
            f2_unpack(r2, r0, r1);
            u[2 * i] = __float_as_uint(r0);
            u[2 * i + 1] = __float_as_uint(r1);
          }
        }
        if (edge) {
          // scaled scores with -inf where the key is hidden or past N: column i
          // is visible iff lo <= i < hi
          const int key0 = jb * kBlockN;
          const int hi = (CAUSAL ? min(row + 1, p.N) : p.N) - key0;
          const int lo = CAUSAL ? row - p.window - key0 : 0;
          if constexpr (ALIBI) {   // + this query head's slope log2(e) * -|key - row|
            const float sl2 = p.alibi[bh % p.H] * 1.4426950408889634f;
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
          for (int k = 0; k < 8; ++k) a[k] = fmaxf(__uint_as_float(u[k]), __uint_as_float(u[8 + k]));
#pragma unroll
          for (int i = 16; i < 128; i += 16) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              a[k] = max3f(a[k], __uint_as_float(u[i + k]), __uint_as_float(u[i + 8 + k]));
          }
          mt = max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
          if (!masked) mt *= c;
        }
        const float m_new = fmaxf(m_use, mt);
        const bool need = m_new > m_use + kTau;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_sfu(m_use - m_new);
          m_use = m_new;
        }
        // a row that has seen only hidden keys so far (sliding window) keeps
        // m = -inf; its p must be 0, not exp2(-inf + inf)
        const float neg_m = m_use == -INFINITY ? 0.f : -m_use;
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        if constexpr (FP8) {
          const float f8 = 256.f * sv_j / v_max;
          const uint64_t c2 = f2_pack(c, c);
          const uint64_t nm2 = f2_pack(neg_m, neg_m);
          const uint64_t f82 = f2_pack(f8, f8);   // P is stored as E4M3 of p * f8 (packed products)
          float keep0 = 0.f, keep1 = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const uint64_t s2 = f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
            const uint64_t x2 = masked ? f2_add(s2, nm2) : f2_fma(s2, c2, nm2);
            const uint64_t p2 = ((i & 7) < NPOLY) ? exp2_poly_f2<DEG>(x2) : exp2_sfu_f2(x2);
            acc[i & 3] = f2_add(acc[i & 3], p2);
            float q0, q1;
            f2_unpack(f2_mul(p2, f82), q0, q1);
            if (i & 1)
              u[i / 2] = pack_e4m3x4(keep0, keep1, q0, q1);
            keep0 = q0;
            keep1 = q1;
          }
          tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        } else {
          if (ALIBI && masked) {   // scores already scaled: p = 2^(u - m)
            const uint64_t nm2 = f2_pack(neg_m, neg_m);
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const uint64_t p2 =
                  exp2_sfu_f2(f2_add(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])), nm2));
              acc[i & 3] = f2_add(acc[i & 3], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              u[i] = pack_bf16x2(p0, p1);       // P overwrites the consumed scores
            }
          } else if (masked) {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float p0 = ex2_sfu(__uint_as_float(u[2 * i]) + neg_m);
              const float p1 = ex2_sfu(__uint_as_float(u[2 * i + 1]) + neg_m);
              acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
              u[i] = pack_bf16x2(p0, p1);       // P overwrites the consumed scores
            }
          } else {
            const uint64_t c2 = f2_pack(c, c);
            const uint64_t nm2 = f2_pack(neg_m, neg_m);
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const uint64_t x2 =
                  f2_fma(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])), c2, nm2);
              const uint64_t p2 = ((i & 7) < NPOLY) ? exp2_poly_f2<DEG>(x2) : exp2_sfu_f2(x2);
              acc[i & 3] = f2_add(acc[i & 3], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              u[i] = pack_bf16x2(p0, p1);
            }
          }
          if constexpr (!C::kEarlyS) tmem_st64(tS, *reinterpret_cast<uint32_t(*)[64]>(&u[0]));
        }
        if constexpr (!C::kEarlyS) tmem_st_wait();
        float sum4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float lo, hi;
          f2_unpack(acc[k], lo, hi);
          sum4[k] = lo + hi;
        }
        l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
        if (j > 0) {
          // PV(j-1) must be done before O is touched or PV(j) is released (and,
          // with P outside S, before P_t is overwritten); waiting every tile
          // also keeps this waiter within one phase.
          if (!(ok = mbar_wait_warp(bar(bar_pv<NS>(t)), (gs + j - 1) & 1, ab, kSiteSmPv))) break;
          tc_fence_after();
        }
        // P outside S goes out first, so its registers are free for the O rescale
        if constexpr (C::kSepP) tmem_st64(tP, *reinterpret_cast<uint32_t(*)[64]>(&u[0]));
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
        if (C::kSepP || (j > 0 && __any_sync(0xffffffffu, need))) tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(bar_p<NS>(t)));
      }
      if (ok) ok = mbar_wait_warp(bar(bar_pv<NS>(t)), (gs + n - 1) & 1, ab, kSiteEpiPv);
      gs += n;
      // All 128 threads of the warpgroup reach this barrier (every wait above is
      // bounded) and take the epilogue together or not at all.
      ok = named_bar_and(1 + t, 128, ok);
      if (!ok) break;
      tc_fence_after();
      // ------------------------------------------------------------ epilogue
      const float inv_l = (FP8 ? v_max * (1.f / 256.f) : 1.f) / l;
      if constexpr (PERS) {
        // O / l straight from registers, each thread its own row (2 d
        // contiguous bytes): the Q buffer already holds the next item's Q
        uint16_t* orow = p.o + (static_cast<size_t>(bh) * p.N + (row < p.N ? row : 0)) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t u[32];
          tmem_ld32(tO + ch * 32, u);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
          if (row < p.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(orow + ch * 32 + 8 * q) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        // (O_t is overwritten only by this item's successor's first P V, which
        // the MMA issues after this warpgroup's next P; the loads above have
        // completed by then)
      } else {
        // bf16: stage O in Q_t, no longer read; FP8: in its own buffer
        const uint32_t o_stage = FP8 ? sbase + C::kOffO + t * C::kOBytes : sbase + C::kOffQ + t * C::kTileBytes;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t u[32];
          tmem_ld32(tO + ch * 32, u);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
          const int col0 = ch * 32;
          const uint32_t panel = o_stage + (col0 / 64) * C::kPanelBytes + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t chunk = ((col0 % 64) / 8 + q) ^ (r & 7);
            st_shared_v4(panel + (chunk << 4), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + t, 128);
        if (r == 0 && qi * kBlockM < p.N) {   // a tile wholly past N is padding
          for (int pn = 0; pn < D / 64; ++pn)
            tma_store_3d(&p.tm_o, o_stage + pn * C::kPanelBytes, pn * 64, qi * kBlockM, bh);   // bf16 O
          tma_store_commit();
          tma_store_wait_read_all();   // the stores complete after the CTA has exited
        }
      }
      if (row < p.N) p.lse[static_cast<size_t>(bh) * p.N + row] = (m_use + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// The longest-processing-time-first deal of the causal items over G CTAs:
// an item's cost is its number of key blocks per tile pair (2 n_1, the two
// tiles' blocks plus the last single-tile block) plus one for its start; the
// kernel's item order (item_at) and key-block counts are followed exactly.
// Cached per thread for the last shape.
const FwdSched* causal_schedule(const FwdParams& p, int G) {
  struct Key {
    int n_pairs, BH, group_heads, window, n_kv, G;
    bool operator==(const Key& o) const {
      return n_pairs == o.n_pairs && BH == o.BH && group_heads == o.group_heads && window == o.window &&
             n_kv == o.n_kv && G == o.G;
    }
  };
  thread_local Key key{-1, -1, -1, -1, -1, -1};
  thread_local FwdSched sched;
  const Key k{p.n_pairs, p.BH, p.group_heads, p.window, p.n_kv, G};
  if (k == key) return &sched;
  const long long items = static_cast<long long>(p.n_pairs) * p.BH;
  sched.n = 0;
  if (items <= kSchedMaxItems && G <= kSchedMaxCtas && G > 0) {
    std::vector<int> cost(items);
    for (int o = 0; o < items; ++o) {
      const int per_group = p.group_heads * p.n_pairs;
      const int g = o / per_group, rr = o - g * per_group;
      const int gh = std::min(p.group_heads, p.BH - g * p.group_heads);
      const int pair = p.n_pairs - 1 - rr / gh;
      const int qt0 = 2 * pair;
      const int j_start = std::max(0, qt0 * kBlockM - p.window) / kBlockN;
      const int n1 = std::min(qt0 + 2, p.n_kv) - j_start;
      cost[o] = 2 * n1 + 1;
    }
    // items in order of decreasing cost; with head groups (group_heads <
    // BH) group by group, each group's items longest first (item_at's order)
    std::vector<int> order(items);
    std::iota(order.begin(), order.end(), 0);
    if (p.group_heads >= p.BH)
      std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
    std::vector<long long> load(G, 0);
    std::vector<std::vector<int>> lists(G);
    for (const int o : order) {
      const int c = static_cast<int>(std::min_element(load.begin(), load.end()) - load.begin());
      load[c] += cost[o];
      lists[c].push_back(o);
    }
    int at = 0;
    for (int c = 0; c < G; ++c) {
      sched.off[c] = static_cast<uint16_t>(at);
      for (const int o : lists[c]) sched.item[at++] = static_cast<uint16_t>(o);
    }
    sched.off[G] = static_cast<uint16_t>(at);
    sched.n = at;
  }
  key = k;
  return &sched;
}

template <int D, bool CAUSAL, int NPOLY, int DEG, bool FP8, bool ALIBI = false, bool PERS = false>
cudaError_t launch_impl(const FwdParams& p, cudaStream_t stream) {
  using C = TileCfg<D, FP8>;
  auto kern = fwd_tile_kernel<D, CAUSAL, NPOLY, DEG, FP8, ALIBI, PERS>;
  cudaError_t e = set_smem_once<fwd_tile_kernel<D, CAUSAL, NPOLY, DEG, FP8, ALIBI, PERS>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>(p.n_pairs) * p.BH;
  const unsigned grid = static_cast<unsigned>((PERS && items > p.sms) ? p.sms : items);
  if constexpr (PERS && CAUSAL) {
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(p, *causal_schedule(p, static_cast<int>(grid)));
  } else {
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(p, FwdSchedNone{});
  }
  return cudaGetLastError();
}

// The exp2 split (pairs of 8 on the polynomial) and the polynomial's degree.
template <int D, bool CAUSAL, bool FP8>
cudaError_t launch_np(const FwdParams& p, cudaStream_t stream) {
  if (p.alibi != nullptr) return launch_impl<D, CAUSAL, 0, 3, FP8, true>(p, stream);   // SFU-only exp2
  if (p.persistent) return launch_impl<D, CAUSAL, 0, 3, FP8, false, true>(p, stream);   // SFU-only exp2
  const bool deg4 = p.poly_deg == 4;
  switch (p.poly_pairs) {
    case 0: return launch_impl<D, CAUSAL, 0, 3, FP8>(p, stream);
    case 4: return deg4 ? launch_impl<D, CAUSAL, 4, 4, FP8>(p, stream) : launch_impl<D, CAUSAL, 4, 3, FP8>(p, stream);
    default: return deg4 ? launch_impl<D, CAUSAL, 2, 4, FP8>(p, stream) : launch_impl<D, CAUSAL, 2, 3, FP8>(p, stream);
  }
}

}  // namespace

cudaError_t launch_fwd_tile_bf16(const FwdParams& p, int d, bool causal, cudaStream_t stream) {
  if (d == 64) return causal ? launch_np<64, true, false>(p, stream) : launch_np<64, false, false>(p, stream);
  return causal ? launch_np<128, true, false>(p, stream) : launch_np<128, false, false>(p, stream);
}

cudaError_t launch_fwd_tile_fp8(const FwdParams& p, bool causal, cudaStream_t stream) {
  return causal ? launch_np<128, true, true>(p, stream) : launch_np<128, false, true>(p, stream);
}

}  // namespace fa
