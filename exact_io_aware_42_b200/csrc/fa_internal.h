// Internal launch interface between the C-ABI layer (fa_api.cu) and the
// kernels.  Not installed; not part of the public header.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Raise a kernel's dynamic shared-memory limit once per device and kernel
// (the template parameter is the kernel itself, so every instantiation has
// its own flags).
template <auto Kernel>
cudaError_t set_smem_once(int bytes) {
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

constexpr int kBlockM = 128;      // query rows per tile (one TMEM lane per row)
constexpr int kBlockN = 128;      // keys per K/V tile
constexpr float kRescaleTau = 8.0f;   // log2 units; see the forward kernel
// FP8 forward: P is stored as E4M3 of p * f with f <= 256, so p may exceed 1
// by at most 2^0.75 (430.5 < 448, the largest E4M3 value); measured faster
// than rescaling on every increase of the max (B2 H16 N8192, two same-process
// A/B runs: 1126 and 1142 vs 1114 and 1106 TFLOPS)
constexpr float kRescaleTauFp8 = 0.75f;
constexpr int kNoWindow = 1 << 30;    // window value meaning "no sliding window" (> any N + 128)

struct FwdParams {
  CUtensorMap tm_q;     // [BH, N, d] bf16 or e4m3, box {64 or 128 elems, 128, 1}
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_o;     // bf16 output, box {64, 128, 1}: the one-CTA-per-item kernel's TMA store
  uint16_t* o;          // bf16 output [BH, N, d]
  float* lse;           // [BH, N]
  unsigned int* status;
  const float* sq;      // fp8 only: block scales [BH, n_qblk]
  const float* sk;
  const float* sv;
  int N;
  int BH;
  int n_pairs;          // ceil(ceil(N/128) / 2): CTAs per (b, h)
  int n_kv;             // ceil(N / 128)
  int kv_group;         // G = H / H_kv query heads per K/V head (1: no grouping)
  int window;           // causal sliding window: key j visible to query i iff i - window <= j <= i
                        // (no window: kNoWindow)
  const float* alibi;   // ALiBi slopes [H] (natural-log units) or nullptr
  int H;                // query heads per batch: head of flattened index bh is bh % H
  float scale_log2;     // scale * log2(e)
  float scale;
  int poly_pairs;       // of every 8 column pairs, how many use the FMA-pipe exp2
  int poly_deg;         // degree of that polynomial (3 or 4)
  int sms;              // multiprocessor count: persistent grid size
  int persistent;       // 1: persistent grid of min(items, SMs) CTAs; 0: one CTA per work item
  int group_heads;      // one-CTA-per-item kernel, causal: CTA order longest first within groups
                        // of this many heads (>= BH: one group over all heads)
};

// Default share of the softmax exp2 taken by the polynomial (of 8 column
// pairs), chosen by measurement on B200: at d = 128 the SFU-only softmax was
// fastest (the polynomial's extra FMA-pipe instructions cost more than the
// SFU time they free); at d = 64, where the softmax is the bound, half the
// pairs on the polynomial was fastest.
constexpr int kDefaultPolyPairsD128 = 0;
// d = 64: SFU-only measured fastest with the persistent kernel (642 vs 560-595 TFLOPS non-causal)
constexpr int kDefaultPolyPairsD64 = 0;
constexpr int kDefaultPolyPairsD256 = 0;
constexpr int kDefaultPolyDegree = 4;
// d <= 128: the two-tile forward's grid by default, chosen by measurement on
// B200 (same-process A/B, TFLOPS, one CTA per item vs persistent): bf16
// gains from the persistent grid non-causal (B4 H16 N4096 d128 1112 vs
// 1140, d64 677 vs 682) and, with its causal items dealt longest processing
// time first, causal (B4 H16 N4096 d128 942 vs 962, N2048 693 vs 722, d64
// 587 vs 603; N >= 8192 even); FP8 gains causal (B4 H16 N4096 850 vs 863)
// and loses non-causal (B2 H16 N8192 1104 vs 1066).
constexpr int kDefaultFwdPersistentCausal = 1;
constexpr int kDefaultFwdPersistentNonCausal = 1;
constexpr int kDefaultFwdPersistentFp8Causal = 1;
constexpr int kDefaultFwdPersistentFp8NonCausal = 0;
// Causal item order of the two-tile forward, measured (same-process A/B):
// with one CTA per work item, grouping heads helped only once K and V of all
// heads far exceed L2 (B8 H16 N4096 d128: 948 vs 910 TFLOPS) and cost about
// 1% at B4 H16 N4096 (926 vs 932) and B1 H16 N16384, so that grid orders
// globally by default; the persistent grid's host-made deal gains from the
// groups (B4 H16 N4096 d128 962 vs 969, B1 H16 N16384 1143 vs 1160, d64 601
// vs 606, FP8 857 vs 863), so it groups by default.
constexpr int kDefaultFwdCausalGroupOneCta = 0;
constexpr int kDefaultFwdCausalGroupPersistent = 1;
// bf16 forward at d <= 128: the one-tile kernel with two score buffers runs
// by default only where the two-tile kernel would have fewer work items
// (pairs of query tiles) than SMs; measured on B200: B2 H8 N1024 d64 causal
// 105 vs 87 TFLOPS, while with at least one pair per SM the two-tile kernel
// wins (B4 H16 N4096 d128 causal 926 vs 776).
// K and V bytes of one head group in that order
constexpr long long kCausalGroupBytes = 32ll << 20;
// FP8 forward: share of the exp2 on the polynomial (pairs of 8)
constexpr int kDefaultPolyPairsFp8 = 0;

// One 128-row query tile per work item, two score buffers, persistent grid (bf16, d = 64, 128).
cudaError_t launch_fwd_q1_bf16(const FwdParams& p, int d, bool causal, cudaStream_t stream);
// Two query tiles per work item (d = 64, 128; FP8 d = 128): one CTA per item
// (needs tm_o) or, with p.persistent (SFU-only exp2, no ALiBi), a persistent grid.
cudaError_t launch_fwd_tile_bf16(const FwdParams& p, int d, bool causal, cudaStream_t stream);
cudaError_t launch_fwd_tile_fp8(const FwdParams& p, bool causal, cudaStream_t stream);
// Head dim 256 (one query tile per work item, K/V streamed as 64-column panels).
cudaError_t launch_fwd_d256(const FwdParams& p, bool causal, cudaStream_t stream);
// One CTA waiting on an mbarrier nothing arrives on (failure-path self-test).
cudaError_t launch_selftest_wait(unsigned int* status, cudaStream_t stream);
// y[i] = 2^x[i] by the softmax's exp2 (degree 0: the SFU; 3, 4, 5: the polynomial).
cudaError_t launch_selftest_exp2(const float* x, float* y, long long n, int degree, cudaStream_t stream);
// Block quantisation of one bf16 tensor to E4M3 (signs == nullptr: no rotation).
struct QuantParams {
  CUtensorMap tm_x;     // bf16 [BH, N, 128], box {64, 128, 1}, 128-byte swizzle
  CUtensorMap tm_x8;    // e4m3 [BH, N, 128], box {128, 128, 1}, 128-byte swizzle
  float* scales;        // [BH, nblk]
  const float* signs;   // d values or nullptr
  unsigned int* status;
  int N;
  int nblk;
};
cudaError_t launch_quant_fp8(const uint16_t* x, uint8_t* x8, float* scales, const float* signs,
                             int BH, int N, int d, cudaStream_t stream);
// d = 128 variant staged through TMA (tensor maps in ``q``).
cudaError_t launch_quant_fp8_tma(const QuantParams& q, int BH, cudaStream_t stream);

struct BwdParams {
  CUtensorMap tm_q;     // bf16 [BH, N, d], box {64, 128, 1}
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_do;
  CUtensorMap tm_dqacc; // fp32 [BH, N, d] accumulator, box {32, 128, 1}, for TMA reduce-add
  CUtensorMap tm_q64;   // bf16 [BH, N, d], box {64, 64, 1}: 64-row blocks (CTA-pair and d = 256 kernels)
  CUtensorMap tm_do64;
  CUtensorMap tm_k64;   // K, V with 64-row boxes (d = 256 dQ kernel)
  CUtensorMap tm_v64;
  const float* lse;     // [BH, N], natural log
  const float* delta;   // [BH, N], D = rowsum(dO o O)
  float* dq_acc;        // [BH, N, d] fp32, zeroed by the preprocess kernel
  uint16_t* dk;         // bf16 [BH, N, d]
  uint16_t* dv;
  uint16_t* dq;         // bf16 [BH, N, d]: written directly by the deterministic dQ kernel
  unsigned int* status;
  int N;
  int BH;
  int n_kv;             // ceil(N / 128): key blocks = CTAs per (b, h)
  int n_q;              // ceil(N / 128): query blocks
  int kv_group;         // G = H / H_kv query heads per K/V head (1: no grouping)
  int window;           // as in FwdParams
  const float* alibi;   // as in FwdParams
  int H;
  int kv_split;         // S: CTAs sharing one (K/V head, key block); 1 = dK, dV stored directly
  int dq_poly;          // deterministic dQ kernel, d = 64: of every 8 column pairs, how many use the FMA-pipe exp2
  float* kv_part;       // S > 1: fp32 partials [S][dV, dK][B * H_kv, N, d]
  float scale_log2;     // scale * log2(e)
  float scale;
  int poly_groups;      // of every 4 groups of 4 columns, how many use the FMA-pipe exp2
  int group_kv;         // causal CTA order: longest first within groups of this many K/V heads
                        // (1: head by head)
};

constexpr int kDefaultBwdPolyGroups = 0;
// Causal backward CTA order: longest first within groups of K/V heads whose
// K, V, Q, dO and dQ accumulator take about this many bytes (1: head by head).
constexpr long long kBwdGroupBytes = 48ll << 20;
constexpr int kDefaultBwdCausalGroup = 1;
// dK, dV of the deterministic backward at d = 128 on CTA pairs (1) or single CTAs (0)
constexpr int kDefaultBwdPair = 0;
constexpr int kDefaultDqPolyPairsD64 = 0;   // measured: the polynomial share did not help (latency-bound)

// D = rowsum(dO o O) per row, and dq_acc <- 0 (dq_acc == nullptr: D only).
cudaError_t launch_bwd_preprocess(const uint16_t* o, const uint16_t* dout, float* delta,
                                  float* dq_acc, long long rows, int d, cudaStream_t stream);
// with_dq: also accumulate dQ into dq_acc (atomic order); without: dK, dV only.
cudaError_t launch_bwd_main(const BwdParams& p, int d, bool causal, bool with_dq, cudaStream_t stream);
// dK, dV on CTA pairs (cta_group::2, d = 128; no dQ: pair with launch_bwd_dq).
cudaError_t launch_bwd_pair(const BwdParams& p, bool causal, cudaStream_t stream);
// Head dim 256: dK, dV per (key block, head-dim half) and dQ per query block.
cudaError_t launch_bwd_kv256(const BwdParams& p, bool causal, cudaStream_t stream);
cudaError_t launch_bwd_dq256(const BwdParams& p, bool causal, cudaStream_t stream);
// Deterministic dQ: one CTA per query block, key blocks in ascending order.
cudaError_t launch_bwd_dq(const BwdParams& p, int d, bool causal, cudaStream_t stream);
// dv, dk <- bf16(sum over the S splits of the fp32 partials); n = elements of one of dv, dk
cudaError_t launch_bwd_kv_reduce(const float* part, uint16_t* dv, uint16_t* dk, long long n, int splits,
                                 cudaStream_t stream);
// dq <- bf16(scale * dq_acc)
cudaError_t launch_bwd_postprocess(const float* dq_acc, uint16_t* dq, long long n, float scale,
                                   cudaStream_t stream);

// Causal backward CTA order.  The hardware hands CTAs to SMs in index order
// as SMs free up, so ordering the CTAs by decreasing work gives a dynamic
// longest-first schedule; doing it within groups of group_kv K/V heads keeps
// each group's K, V, Q, dO and dQ accumulator in L2 while its CTAs run.
// Key-block CTAs (u over groups x key blocks j, small j first x the group's
// K/V heads x splits):
__device__ __forceinline__ void causal_kv_order(int u, int n_kv, int kv_split, int group_kv, int BHkv, int& kvh,
                                                int& split, int& j) {
  const int per_group = group_kv * kv_split * n_kv;
  const int g = u / per_group;
  const int rr = u - g * per_group;
  const int lanes = min(group_kv, BHkv - g * group_kv) * kv_split;
  j = rr / lanes;
  kvh = g * group_kv + (rr % lanes) / kv_split;
  split = (rr % lanes) % kv_split;
}
// Query-block CTAs (u over groups of gq query heads x query blocks i, large i
// first x the group's query heads):
__device__ __forceinline__ void causal_q_order(int u, int n_q, int gq, int BH, int& bh, int& i) {
  const int per_group = gq * n_q;
  const int g = u / per_group;
  const int rr = u - g * per_group;
  const int lanes = min(gq, BH - g * gq);
  i = n_q - 1 - rr / lanes;
  bh = g * gq + rr % lanes;
}

}  // namespace fa
