// Fused exact attention forward for sm_100a (bf16 in, fp32 accumulate).
//
// What it computes: O = softmax(scale * Q K^T [causal]) V and the per-row
// logsumexp L, exactly as the standard definition ("FlashAttention" concept
// note, "How it works"), reached by the online softmax of "FlashAttention
// v1/v2/v3/v4: the librarian who never clears the desk" (online softmax
// section, eq. 2): per K/V tile the running max m and sum l are updated, the
// running output is rescaled by 2^(m_old - m_new), and the division by l is
// deferred to the end (lineage page, "FA2 (2023)", refinement 2).
//
// Work unit: a pair of 128-row query tiles of one (b, h); every needed
// 128-key K/V tile is streamed once for both (each K/V tile is read from
// L2/HBM once per 256 query rows).  The grid is persistent: one CTA per SM
// walks its share of the work items (longest first when causal), and one
// item's epilogue overlaps the next item's Q load and first S products.
// Roles:
//   warps 0-3  softmax for query tile 0 (thread r owns row r = TMEM lane r),
//              and that tile's epilogue (O / l written from registers)
//   warps 4-7  softmax and epilogue for query tile 1
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
// Optionally (FA_TUNE_FWD_SPLIT_PV) each P V runs in two halves of 64 keys,
// the first released while the softmax still computes the second; measured
// slower at d <= 128, so off by default.
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
#include <type_traits>

#include "fa_exp2.cuh"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int kElem = FP8 ? 1 : 2;            // bytes per Q/K/V element
  static constexpr int kPanels = D * kElem / 128;      // 128-byte swizzle panels per row
  static constexpr int kPanelElems = 128 / kElem;      // elements per panel row
  static constexpr int kPanelBytes = 128 * 128;        // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBlockM * D * kElem;   // one 128 x D tile
  static constexpr int kStages = FP8 ? 8 : ((D == 128) ? 5 : 8);
  static constexpr int kThreads = 320;
  static constexpr int kOffQ = 0;                      // two query tiles
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + kStages * kTileBytes;
  static constexpr int kNumBars = 15 + 2 * kStages;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 48 + 1024;   // + base alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;       // + 128 * t
  static constexpr uint32_t kColO = 256;     // + D * t
};
static_assert(FwdCfg<128, true>::kSmemBytes <= 232448, "fp8 forward shared memory");
static_assert(FwdCfg<128, false>::kSmemBytes <= 232448, "bf16 forward shared memory");

// barrier slots
__device__ __forceinline__ int bar_q(int t) { return t; }                 // Q_t landed
__device__ __forceinline__ int bar_qfree(int t) { return 2 + t; }         // last S of Q_t done
template <int NS> __device__ __forceinline__ int bar_full(int s) { return 4 + s; }
template <int NS> __device__ __forceinline__ int bar_empty(int s) { return 4 + NS + s; }
template <int NS> __device__ __forceinline__ int bar_s(int t) { return 4 + 2 * NS + t; }
template <int NS> __device__ __forceinline__ int bar_p(int t) { return 6 + 2 * NS + t; }    // P keys 0..63
template <int NS> __device__ __forceinline__ int bar_ph(int t) { return 8 + 2 * NS + t; }   // P keys 64..127
template <int NS> __device__ __forceinline__ int bar_pv(int t) { return 10 + 2 * NS + t; }
template <int NS> __device__ __forceinline__ int bar_ofree(int t) { return 12 + 2 * NS + t; }  // O_t read out
template <int NS> __device__ __forceinline__ int bar_drain() { return 14 + 2 * NS; }

// wait-site codes reported in bits 8..15 of the status word
enum : unsigned int { kSiteProdEmpty = 1, kSiteMmaQ, kSiteMmaFull, kSiteMmaP, kSiteSmS, kSiteSmPv,
                      kSiteEpiPv, kSiteDrain, kSiteProdQ, kSiteMmaO };

__device__ __forceinline__ void st_global_v4(void* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// E4M3 byte pair <- (lo, hi), round to nearest even, saturating at +-448.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  unsigned short lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// One work item: a pair of 128-row query tiles (qt0, qt0 + 1) of one (b, h).
struct Item {
  int bh, kvh, qt0, j_start, n_t0, n_t1;
};

// Work item o of the launch.  Causal: the heaviest pairs of every head first
// (longest-first balances the uneven work); non-causal: head-major, so the
// CTAs working at any time cover a few heads whose K and V stay in L2.
template <bool CAUSAL>
__device__ __forceinline__ Item item_at(const FwdParams& p, int o) {
  Item it;
  it.bh = CAUSAL ? o % p.BH : o / p.n_pairs;
  const int pair = CAUSAL ? p.n_pairs - 1 - o / p.BH : o % p.n_pairs;
  // Grouped K/V heads: query head h of batch b reads K/V head b * H_kv + h / G,
  // which in the flattened [B * H] index is bh / G.
  it.kvh = it.bh / p.kv_group;
  it.qt0 = 2 * pair;
  // Sliding window (causal only): key j is visible to query i iff
  // i - window <= j <= i.  Key blocks wholly left of tile 0's window are
  // never loaded; both tiles start at the same block (tile 1's first block
  // may then be fully masked for it, which the softmax handles).
  it.j_start = CAUSAL ? max(0, it.qt0 * kBlockM - p.window) / kBlockN : 0;
  it.n_t0 = (CAUSAL ? min(it.qt0 + 1, p.n_kv) : p.n_kv) - it.j_start;
  it.n_t1 = (CAUSAL ? min(it.qt0 + 2, p.n_kv) : p.n_kv) - it.j_start;
  return it;
}

// The k-th item of this CTA: the grid walks the item list in rounds of
// gridDim.x, every other round in reverse CTA order ("snake"), so that with
// longest-first items each CTA's total work comes out nearly equal.
__device__ __forceinline__ int my_item(int k) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// Persistent forward: one CTA per SM walks its list of work items.  NPOLY of
// every 8 column pairs take the polynomial exp2 (degree DEG), the rest the
// SFU.  FP8: Q, K, V are E4M3 with per-128-row block scales and both products
// run as kind::f8f6f4 (see the FP8 notes at the softmax).
template <int D, bool CAUSAL, int NPOLY, int DEG, bool FP8>
__global__ void __launch_bounds__(320, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D, FP8>;
  constexpr int kWarpProd = 8;
  constexpr int kWarpMma = 9;
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
  const int n_items = p.n_pairs * p.BH;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(bar_q(t)), 1);
      mbar_init(bar(bar_qfree(t)), 1);
      mbar_init(bar(bar_s<NS>(t)), 1);
      mbar_init(bar(bar_p<NS>(t)), 128);
      mbar_init(bar(bar_ph<NS>(t)), 128);
      mbar_init(bar(bar_pv<NS>(t)), 1);
      mbar_init(bar(bar_ofree<NS>(t)), 128);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(bar_full<NS>(s)), 1);
      mbar_init(bar(bar_empty<NS>(s)), 1);
    }
    mbar_init(bar(bar_drain<NS>()), 1);
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
      int seq = 0;
      int q_loads[2] = {0, 0};   // Q tile loads issued per tile
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int o = my_item(k);
        if (o >= n_items) break;
        const Item it = item_at<CAUSAL>(p, o);
        for (int t = 0; t < 2 && ok; ++t) {
          // Q_t of the previous item is free once its last S product is done
          if (k > 0 && !(ok = mbar_wait(bar(bar_qfree(t)), (k - 1) & 1, ab, kSiteProdQ))) break;
          mbar_arrive_expect_tx(bar(bar_q(t)), C::kTileBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(sbase + C::kOffQ + t * C::kTileBytes + pn * C::kPanelBytes, &p.tm_q,
                        bar(bar_q(t)), pn * C::kPanelElems, (it.qt0 + t) * kBlockM, it.bh);
          ++q_loads[t];
        }
        for (int j = 0; j < it.n_t1 && ok; ++j) {
          for (int w = 0; w < 2; ++w) {
            const int s = seq % NS;
            const uint32_t ph = (seq / NS) & 1;
            if (!(ok = mbar_wait(bar(bar_empty<NS>(s)), ph ^ 1, ab, kSiteProdEmpty))) break;
            mbar_arrive_expect_tx(bar(bar_full<NS>(s)), C::kTileBytes);
            const CUtensorMap* m = (w == 0) ? &p.tm_k : &p.tm_v;
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d(sbase + C::kOffRing + s * C::kTileBytes + pn * C::kPanelBytes, m,
                          bar(bar_full<NS>(s)), pn * C::kPanelElems, (it.j_start + j) * kBlockN, it.kvh);
            ++seq;
          }
        }
      }
      if (*abort_flag) {
        // Another role gave up: let every copy this thread started land before
        // the CTA exits (bounded, ignoring the abort flag).
        volatile int never = 0;
        const Abort drain{&never, p.status};
        for (int t = 0; t < 2; ++t)
          if (q_loads[t] > 0) mbar_wait(bar(bar_q(t)), (q_loads[t] - 1) & 1, drain, kSiteDrain);
        const int first = seq > NS ? seq - NS : 0;
        for (int q = first; q < seq; ++q)
          mbar_wait(bar(bar_full<NS>(q % NS)), (q / NS) & 1, drain, kSiteDrain);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
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
      // P V in two halves: keys 0..63 as soon as the softmax has stored that
      // half of P (bar_p), keys 64..127 after the rest (bar_ph), so the
      // product's first half overlaps the softmax's second half.
      auto issue_pv_half = [&](int t, uint32_t v_addr, bool acc, int h) {
        constexpr int kHalf = kBlockN / kK / 2;
#pragma unroll
        for (int kq = 0; kq < kHalf; ++kq) {
          const int kk = h * kHalf + kq;
          // V is MN-major (d contiguous); one K step is kK key rows of 128 bytes.
          // P in TMEM packs 32 bits per column: 2 bf16 or 4 E4M3 keys.
          const uint32_t a_col = 8 * kk;
          const uint64_t b = smem_desc_sw128(v_addr + kk * kK * 128, C::kPanelBytes, 1024);
          if constexpr (FP8)
            mma_f8_ts(tmem + C::kColO + D * t, tmem + C::kColS + 128 * t + a_col, b, kIdescO,
                      (acc || kk > 0) ? 1u : 0u);
          else
            mma_f16_ts(tmem + C::kColO + D * t, tmem + C::kColS + 128 * t + a_col, b, kIdescO,
                       (acc || kk > 0) ? 1u : 0u);
        }
      };
      int g[2] = {0, 0};   // P V products issued per tile (all items): the P barriers' phase
      // returns false if a wait gave up
      auto issue_pv = [&](int t, uint32_t v_addr, bool acc) -> bool {
        // split: the first half as soon as it is in TMEM (bar_p), the second
        // after bar_ph; otherwise all of P behind the one release (bar_p)
        if (!mbar_wait(bar(bar_p<NS>(t)), g[t] & 1, ab, kSiteMmaP)) return false;
        tc_fence_after();
        issue_pv_half(t, v_addr, acc, 0);
        if (p.split_pv) {
          if (!mbar_wait(bar(bar_ph<NS>(t)), g[t] & 1, ab, kSiteMmaP)) return false;
          tc_fence_after();
        }
        issue_pv_half(t, v_addr, acc, 1);
        tc_commit(bar(bar_pv<NS>(t)));
        ++g[t];
        return true;
      };
      int seq = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int o = my_item(k);
        if (o >= n_items) break;
        const Item it = item_at<CAUSAL>(p, o);
        const int n_t[2] = {it.n_t0, it.n_t1};
        if (!(ok = mbar_wait(bar(bar_q(0)), k & 1, ab, kSiteMmaQ))) break;
        if (!(ok = mbar_wait(bar(bar_q(1)), k & 1, ab, kSiteMmaQ))) break;
        int ks = seq % NS;
        if (!(ok = mbar_wait(bar(bar_full<NS>(ks)), (seq / NS) & 1, ab, kSiteMmaFull))) break;
        ++seq;
        tc_fence_after();
        // The previous item's last P V products precede these S products on
        // the tensor pipe, so the S regions are free.
        issue_s(0, ring(ks));
        if (n_t[0] == 1) tc_commit(bar(bar_qfree(0)));
        issue_s(1, ring(ks));
        if (n_t[1] == 1) tc_commit(bar(bar_qfree(1)));
        tc_commit(bar(bar_empty<NS>(ks)));
        for (int j = 0; j < n_t[1] && ok; ++j) {
          const int vs = seq % NS;
          if (!(ok = mbar_wait(bar(bar_full<NS>(vs)), (seq / NS) & 1, ab, kSiteMmaFull))) break;
          ++seq;
          const bool has_next = j + 1 < n_t[1];
          if (has_next) {
            ks = seq % NS;
            if (!(ok = mbar_wait(bar(bar_full<NS>(ks)), (seq / NS) & 1, ab, kSiteMmaFull))) break;
            ++seq;
          }
          tc_fence_after();
          if (j < n_t[0]) {
            // O_0 of the previous item must have been read out before this
            // item's first P V overwrites it
            if (j == 0 && k > 0 && !(ok = mbar_wait(bar(bar_ofree<NS>(0)), (k - 1) & 1, ab, kSiteMmaO))) break;
            if (!(ok = issue_pv(0, ring(vs), j > 0))) break;
            if (j + 1 < n_t[0]) {
              issue_s(0, ring(ks));
              if (j + 2 == n_t[0]) tc_commit(bar(bar_qfree(0)));
            }
          }
          if (j == 0 && k > 0 && !(ok = mbar_wait(bar(bar_ofree<NS>(1)), (k - 1) & 1, ab, kSiteMmaO))) break;
          if (!(ok = issue_pv(1, ring(vs), j > 0))) break;
          tc_commit(bar(bar_empty<NS>(vs)));
          if (has_next) {
            issue_s(1, ring(ks));
            if (j + 2 == n_t[1]) tc_commit(bar(bar_qfree(1)));
            tc_commit(bar(bar_empty<NS>(ks)));
          }
        }
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
    constexpr float kTau = FP8 ? 0.f : kRescaleTau;
    int gs = 0;        // this tile's score tiles over all items: the S / P V barriers' phase
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int o = my_item(k);
      if (o >= n_items) break;
      const Item it = item_at<CAUSAL>(p, o);
      const int bh = it.bh;
      const int qi = it.qt0 + t;
      const int row = qi * kBlockM + r;
      const int n = t ? it.n_t1 : it.n_t0;
      // FP8: scores are dequantised per tile pair with s_q(i) * s_k(j); P is
      // stored as E4M3 times 256 * s_v(j) / max_j s_v(j), which folds V's block
      // scale into P (p <= 1 because FP8 rescales on every max increase), and O
      // is multiplied back by max s_v / 256 at the end.
      const size_t sc_base = static_cast<size_t>(bh) * p.n_kv;      // Q's block scales
      const size_t kv_base = static_cast<size_t>(it.kvh) * p.n_kv;  // K's and V's
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
        sk_next = p.sk[kv_base + it.j_start];
        sv_next = p.sv[kv_base + it.j_start];
      }
      float m_use = -INFINITY;
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int jb = it.j_start + j;      // key block; j counts this tile's iterations
        const int gj = gs + j;
        if (!(ok = mbar_wait_warp(bar(bar_s<NS>(t)), gj & 1, ab, kSiteSmS))) break;
        tc_fence_after();
        uint32_t u[128];
        tmem_ld128(tS, u);
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
        const bool masked = (CAUSAL && (jb == qi || jb * kBlockN < qi * kBlockM + kBlockM - 1 - p.window)) ||
                            ((jb + 1) * kBlockN > p.N) || p.alibi != nullptr;
        if (masked) {
          // scaled scores with -inf where the key is hidden or past N: column i
          // is visible iff lo <= i < hi
          const int key0 = jb * kBlockN;
          const int hi = (CAUSAL ? min(row + 1, p.N) : p.N) - key0;
          const int lo = CAUSAL ? row - p.window - key0 : 0;
          if (p.alibi != nullptr) {   // + this query head's slope log2(e) * -|key - row|
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
          for (int q = 0; q < 8; ++q) a[q] = fmaxf(__uint_as_float(u[q]), __uint_as_float(u[8 + q]));
#pragma unroll
          for (int i = 16; i < 128; i += 16) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              a[q] = max3f(a[q], __uint_as_float(u[i + q]), __uint_as_float(u[i + 8 + q]));
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
        const uint64_t c2 = f2_pack(c, c);
        const uint64_t nm2 = f2_pack(neg_m, neg_m);
        const float f8 = FP8 ? 256.f * sv_j / v_max : 1.f;
        // p for score pairs [32 h, 32 h + 32) (keys 64 h .. 64 h + 63), packed
        // over the scores already consumed: bf16 pairs into u[32 h ..], E4M3
        // quads into u[16 h ..].
        auto exp_half = [&](auto hc) {
          constexpr int h = decltype(hc)::value;
          if constexpr (FP8) {
            float keep0 = 0.f, keep1 = 0.f;
#pragma unroll
            for (int i = 32 * h; i < 32 * h + 32; ++i) {
              const uint64_t s2 = f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
              const uint64_t x2 = masked ? f2_add(s2, nm2) : f2_fma(s2, c2, nm2);
              const uint64_t p2 = ((i & 7) < NPOLY) ? exp2_poly_f2<DEG>(x2) : exp2_sfu_f2(x2);
              acc[i & 3] = f2_add(acc[i & 3], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              if (i & 1)
                u[i / 2] = pack_e4m3x4(keep0 * f8, keep1 * f8, p0 * f8, p1 * f8);
              keep0 = p0;
              keep1 = p1;
            }
          } else if (masked) {
#pragma unroll
            for (int i = 32 * h; i < 32 * h + 32; ++i) {
              const float p0 = ex2_sfu(__uint_as_float(u[2 * i]) + neg_m);
              const float p1 = ex2_sfu(__uint_as_float(u[2 * i + 1]) + neg_m);
              acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
              u[i] = pack_bf16x2(p0, p1);       // P overwrites the consumed scores
            }
          } else {
#pragma unroll
            for (int i = 32 * h; i < 32 * h + 32; ++i) {
              const uint64_t x2 =
                  f2_fma(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])), c2, nm2);
              const uint64_t p2 = ((i & 7) < NPOLY) ? exp2_poly_f2<DEG>(x2) : exp2_sfu_f2(x2);
              acc[i & 3] = f2_add(acc[i & 3], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              u[i] = pack_bf16x2(p0, p1);
            }
          }
        };
        // split: the first half of P, the O correction, release of that half
        // to the P V product, then the second half.  Otherwise all of P, the
        // correction, and one release (measured faster at d <= 128: the extra
        // wait for the first half's TMEM store lies on the softmax's path).
        auto correct_o = [&]() -> bool {
          if (j > 0) {
            // PV(j-1) must be done before O is touched or PV(j) is released;
            // waiting every tile also keeps this waiter within one phase.
            if (!mbar_wait_warp(bar(bar_pv<NS>(t)), (gj - 1) & 1, ab, kSiteSmPv)) return false;
            tc_fence_after();
            if (__any_sync(0xffffffffu, need)) {
#pragma unroll
              for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t w[32];
                tmem_ld32(tO + ch * 32, w);
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
                tmem_st32(tO + ch * 32, w);
              }
            }
          }
          return true;
        };
        if (p.split_pv) {
          exp_half(std::integral_constant<int, 0>{});
          if constexpr (FP8)
            tmem_st16(tS, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
          else
            tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          if (!(ok = correct_o())) break;
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(bar_p<NS>(t)));
          exp_half(std::integral_constant<int, 1>{});
          if constexpr (FP8)
            tmem_st16(tS + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
          else
            tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(bar_ph<NS>(t)));
        } else {
          exp_half(std::integral_constant<int, 0>{});
          exp_half(std::integral_constant<int, 1>{});
          if constexpr (FP8)
            tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          else
            tmem_st64(tS, *reinterpret_cast<uint32_t(*)[64]>(&u[0]));
          if (!(ok = correct_o())) break;
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(bar_p<NS>(t)));
        }
        float sum4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float lo, hi;
          f2_unpack(acc[q], lo, hi);
          sum4[q] = lo + hi;
        }
        l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      }
      gs += n;
      if (ok) ok = mbar_wait_warp(bar(bar_pv<NS>(t)), (gs - 1) & 1, ab, kSiteEpiPv);
      // All 128 threads of the warpgroup reach this barrier (every wait above
      // is bounded) and take the epilogue, and the next item, together or
      // not at all.
      ok = named_bar_and(1 + t, 128, ok);
      if (!ok) break;
      tc_fence_after();
      // ------------------------------------------------------------ epilogue
      // O / l straight from registers to global memory (each thread writes
      // its own row, 2 d contiguous bytes); TMEM O_t is free again after the
      // loads, and the next item's first P V may overwrite it.
      const float inv_l = (FP8 ? v_max * (1.f / 256.f) : 1.f) / l;
      uint16_t* orow = p.o + (static_cast<size_t>(bh) * p.N + (row < p.N ? row : 0)) * D;
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
          for (int q = 0; q < 4; ++q)
            st_global_v4(orow + ch * 32 + 8 * q, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(bar_ofree<NS>(t)));
      if (row < p.N) p.lse[static_cast<size_t>(bh) * p.N + row] = (m_use + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool CAUSAL, int NPOLY, int DEG, bool FP8>
cudaError_t launch_impl(const FwdParams& p, cudaStream_t stream) {
  using C = FwdCfg<D, FP8>;
  auto kern = fwd_kernel<D, CAUSAL, NPOLY, DEG, FP8>;
  cudaError_t e = set_smem_once<fwd_kernel<D, CAUSAL, NPOLY, DEG, FP8>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (at most one per work item); otherwise one
  // CTA per work item, scheduled by the hardware in item order
  const long long items = static_cast<long long>(p.n_pairs) * p.BH;
  const unsigned grid = static_cast<unsigned>(p.persistent && items > p.sms ? p.sms : items);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

// The exp2 split (pairs of 8 on the polynomial) and the polynomial's degree.
template <int D, bool CAUSAL>
cudaError_t launch_np(const FwdParams& p, cudaStream_t stream) {
  const bool deg4 = p.poly_deg == 4;
  switch (p.poly_pairs) {
    case 0: return launch_impl<D, CAUSAL, 0, 3, false>(p, stream);
    case 4: return deg4 ? launch_impl<D, CAUSAL, 4, 4, false>(p, stream) : launch_impl<D, CAUSAL, 4, 3, false>(p, stream);
    default: return deg4 ? launch_impl<D, CAUSAL, 2, 4, false>(p, stream) : launch_impl<D, CAUSAL, 2, 3, false>(p, stream);
  }
}

}  // namespace

cudaError_t launch_fwd_bf16(const FwdParams& p, int d, bool causal, cudaStream_t stream) {
  if (d == 64) return causal ? launch_np<64, true>(p, stream) : launch_np<64, false>(p, stream);
  return causal ? launch_np<128, true>(p, stream) : launch_np<128, false>(p, stream);
}

template <bool CAUSAL>
cudaError_t launch_fp8_np(const FwdParams& p, cudaStream_t stream) {
  const bool deg4 = p.poly_deg == 4;
  switch (p.poly_pairs) {
    case 0: return launch_impl<128, CAUSAL, 0, 3, true>(p, stream);
    case 4: return deg4 ? launch_impl<128, CAUSAL, 4, 4, true>(p, stream) : launch_impl<128, CAUSAL, 4, 3, true>(p, stream);
    default: return deg4 ? launch_impl<128, CAUSAL, 2, 4, true>(p, stream) : launch_impl<128, CAUSAL, 2, 3, true>(p, stream);
  }
}

cudaError_t launch_fwd_fp8(const FwdParams& p, bool causal, cudaStream_t stream) {
  return causal ? launch_fp8_np<true>(p, stream) : launch_fp8_np<false>(p, stream);
}

}  // namespace fa
