// C-ABI layer: argument validation, TMA tensor-map encoding, the device
// status word, and dispatch to the kernels.  See include/fa.h for the
// contract of each entry point.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace fa {

// First in-kernel failure since the last fa_clear_status (one word per device).
__device__ unsigned int g_status = 0;

namespace {

constexpr int kMaxN = 1 << 20;
constexpr int kMaxBH = 1 << 20;
constexpr int kMaxDevices = 64;
// Work items (query-tile pairs x heads) of one forward launch: kept within int range.
constexpr long long kMaxWorkItems = (1LL << 31) - 4096;

struct DeviceInfo {
  std::atomic<int> state{0};   // 0 not probed, 1 usable, 2 unusable (sm_100 absent)
  unsigned int* status = nullptr;
  int sms = 0;                 // multiprocessor count
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Current device, probed once (under the lock): sm_100 present, SM count,
// status-word address, driver entry point for tensor-map encoding.  Later
// calls read the probed state without taking the lock.
fa_status current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  DeviceInfo& di = g_dev[dev];
  int s = di.state.load(std::memory_order_acquire);
  if (s == 0) {
    std::lock_guard<std::mutex> lock(g_mu);
    s = di.state.load(std::memory_order_relaxed);
    if (s == 0) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;   // not marked probed: a later call may try again
      }
      if (major != 10 || minor != 0) {
        di.state.store(2, std::memory_order_release);
        return FA_ERR_UNSUPPORTED;
      }
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_NO_DEVICE;
      }
      if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr) {
          cudaGetLastError();
          return FA_ERR_NO_DEVICE;
        }
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
      }
      di.status = static_cast<unsigned int*>(addr);
      di.sms = sms;
      s = 1;
      di.state.store(1, std::memory_order_release);
    }
  }
  if (s != 1) return FA_ERR_UNSUPPORTED;
  *out = &di;
  return FA_OK;
}

// Measurement controls (fa_set_tuning), stored as value + 1 so that the
// zero-initialised 0 means "the built-in default".
std::atomic<int> g_tune[FA_TUNE_COUNT];

int tune_raw(int knob) { return g_tune[knob].load(std::memory_order_relaxed) - 1; }

// Share of the forward's exp2 work on the FMA pipe (pairs of 8) and the
// polynomial's degree.
int poly_pairs(int d) {
  const int v = tune_raw(FA_TUNE_FWD_POLY_PAIRS);
  if (v >= 0) return v;
  return d == 64 ? kDefaultPolyPairsD64 : d == 256 ? kDefaultPolyPairsD256 : kDefaultPolyPairsD128;
}

int fp8_poly_pairs() {
  const int v = tune_raw(FA_TUNE_FP8_POLY_PAIRS);
  return v >= 0 ? v : kDefaultPolyPairsFp8;
}

int poly_degree() {
  const int v = tune_raw(FA_TUNE_FWD_POLY_DEGREE);
  return v >= 0 ? v : kDefaultPolyDegree;
}

// Backward P-phase exp2 share on the FMA pipe (groups of 4 of 16 column quads).
int bwd_poly_groups() {
  const int v = tune_raw(FA_TUNE_BWD_POLY_GROUPS);
  return v >= 0 ? v : kDefaultBwdPolyGroups;
}

// The two-tile forward's grid; the persistent mode is built for the SFU-only
// exp2 without ALiBi (the exp2 split is a measurement control).
int fwd_persistent(bool fp8, bool causal, int poly, const float* alibi) {
  if (poly != 0 || alibi != nullptr) return 0;
  const int v = tune_raw(FA_TUNE_FWD_PERSISTENT);
  if (v >= 0) return v;
  if (fp8) return causal ? kDefaultFwdPersistentFp8Causal : kDefaultFwdPersistentFp8NonCausal;
  return causal ? kDefaultFwdPersistentCausal : kDefaultFwdPersistentNonCausal;
}

// The one-tile forward kernel: set explicitly, or (default) when the
// two-tile kernel would have fewer work items than SMs.
int fwd_q1(long long pair_items, int sms) {
  const int v = tune_raw(FA_TUNE_FWD_Q1);
  return v >= 0 ? v : (pair_items < sms ? 1 : 0);
}

int fwd_causal_group(bool persistent) {
  const int v = tune_raw(FA_TUNE_FWD_CAUSAL_GROUP);
  return v >= 0 ? v : persistent ? kDefaultFwdCausalGroupPersistent : kDefaultFwdCausalGroupOneCta;
}

// Heads per group of the causal item order (see FwdParams::group_heads):
// K and V of the group's K/V heads within kCausalGroupBytes.
int fwd_group_heads(int BH, int kv_group, int N, int d, int elem_bytes, bool persistent) {
  if (!fwd_causal_group(persistent)) return BH;
  const long long kv_bytes = 2ll * N * d * elem_bytes;   // K and V of one K/V head
  const long long g = kCausalGroupBytes / kv_bytes * kv_group;
  return static_cast<int>(g < 1 ? 1 : g > BH ? BH : g);
}

int bwd_causal_group() {
  const int v = tune_raw(FA_TUNE_BWD_CAUSAL_GROUP);
  return v >= 0 ? v : kDefaultBwdCausalGroup;
}

// K/V heads per group of the causal backward's CTA order.
int bwd_group_kv(int BHkv, int kv_group, int N, int d) {
  if (!bwd_causal_group()) return 1;
  const long long per_kv = static_cast<long long>(N) * d * (4 + 8ll * kv_group);   // K, V; Q, dO, dQ acc
  const long long g = kBwdGroupBytes / per_kv;
  return static_cast<int>(g < 1 ? 1 : g > BHkv ? BHkv : g);
}

int bwd_pair() {
  const int v = tune_raw(FA_TUNE_BWD_PAIR);
  return v >= 0 ? v : kDefaultBwdPair;
}

// Deterministic dQ kernel at d = 64: pairs of 8 on the polynomial.
int dq_poly_pairs() {
  const int v = tune_raw(FA_TUNE_DQ_POLY_PAIRS);
  return v >= 0 ? v : kDefaultDqPolyPairsD64;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D view [BH, N, d] of a contiguous [B, H, N, d] tensor, 128-byte swizzle,
// box {box_inner elements, box_rows, 1}; out-of-range elements read as zero
// and are skipped on store.
bool encode_3d_uncached(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int d,
                        int N, int BH, int box_inner, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize,
                           static_cast<cuuint64_t>(N) * d * esize};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A tensor map is a pure function of its arguments (address, type, extents,
// box), so encoded maps are kept in a small per-thread cache: a repeated call
// on the same buffers and shape copies 128 bytes instead of encoding again.
// Nothing can go stale -- a different buffer or shape is a different key.
struct MapKey {
  const void* base;
  int dt, d, N, BH, box_inner, box_rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && dt == o.dt && d == o.d && N == o.N && BH == o.BH &&
           box_inner == o.box_inner && box_rows == o.box_rows;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool valid;
};
constexpr int kMapCacheSlots = 64;
thread_local MapEntry t_maps[kMapCacheSlots];

bool encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int d, int N,
               int BH, int box_inner, int box_rows) {
  const MapKey key{base, static_cast<int>(dt), d, N, BH, box_inner, box_rows};
  uint64_t h = reinterpret_cast<uintptr_t>(base) >> 8;
  h = h * 0x9E3779B97F4A7C15ull ^ (static_cast<uint64_t>(N) << 20) ^ (static_cast<uint64_t>(BH) << 3) ^
      static_cast<uint64_t>(dt * 131 + d * 7 + box_inner + box_rows);
  h *= 0xBF58476D1CE4E5B9ull;
  MapEntry& e = t_maps[(h >> 58) & (kMapCacheSlots - 1)];
  if (e.valid && e.key == key) {
    *m = e.map;
    return true;
  }
  if (!encode_3d_uncached(m, base, dt, esize, d, N, BH, box_inner, box_rows)) return false;
  e.key = key;
  e.map = *m;
  e.valid = true;
  return true;
}

// allow256: the bf16 forward also serves head dim 256.
fa_status check_shape(int B, int H, int N, int d, float scale, bool allow256 = false) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && !(allow256 && d == 256)) return FA_ERR_UNSUPPORTED;
  if (N > kMaxN || static_cast<long long>(B) * H > kMaxBH) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Grouped K/V heads: 1 <= H_kv, H a multiple of H_kv.
fa_status check_kv_heads(int H, int H_kv) {
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// CTAs sharing one (K/V head, key block) in the backward: the smallest
// divisor S of G = H / H_kv that gives the grid about three CTAs per SM, so
// that few K/V heads (MQA) still fill the GPU; 1 when the grid is large
// enough already.  ``sms`` is the device's multiprocessor count.
int kv_split_for(int B, int H, int H_kv, int N, int sms) {
  const int G = H / H_kv;
  const long long ctas = static_cast<long long>(B) * H_kv * ((N + 127) / 128);
  int S = 1;
  while (S < G && ctas * S < 3LL * sms) {
    int next = S + 1;
    while (G % next) ++next;
    S = next;
  }
  return S;
}

// Multiprocessor count of the current device for sizing decisions made
// before any launch (the workspace size query): the probed value, or 148
// (B200) when no usable device is current.
int current_sms() {
  DeviceInfo* di = nullptr;
  if (current_device(&di) == FA_OK && di->sms > 0) return di->sms;
  return 148;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Sliding window: -1 (none) or >= 0 with causal; returns the kernels' value.
fa_status check_window(int window_left, int causal, int* window) {
  if (window_left < -1 || (window_left >= 0 && !causal)) return FA_ERR_INVALID_ARG;
  *window = window_left < 0 ? kNoWindow : window_left;
  return FA_OK;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int H_kv, int N, int d, float scale, int causal,
                               int window_left, const float* alibi_slopes, void* stream) {
  fa_status st = check_shape(B, H, N, d, scale, true);
  if (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) return FA_ERR_MISALIGNED;
  if (st != FA_OK) return st;
  if (H > 0 && (st = check_kv_heads(H, H_kv)) != FA_OK) return st;
  int window = kNoWindow;
  if ((st = check_window(window_left, causal, &window)) != FA_OK) return st;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != FA_OK) return st;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int BH = B * H;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int BHkv = B * H_kv;
  if (!encode_3d(&p.tm_q, q, bf, 2, d, N, BH, 64, kBlockM) ||
      !encode_3d(&p.tm_k, k, bf, 2, d, N, BHkv, 64, kBlockN) ||
      !encode_3d(&p.tm_v, v, bf, 2, d, N, BHkv, 64, kBlockN))
    return FA_ERR_INVALID_ARG;
  p.o = static_cast<uint16_t*>(o);
  p.sms = di->sms;
  p.persistent = d == 256 ? 1 : fwd_persistent(false, causal != 0, poly_pairs(d), alibi_slopes);
  p.group_heads = fwd_group_heads(B * H, H / H_kv, N, d, 2, p.persistent != 0);
  if (!p.persistent && !encode_3d(&p.tm_o, o, bf, 2, d, N, BH, 64, kBlockM)) return FA_ERR_INVALID_ARG;
  p.lse = lse;
  p.status = di->status;
  p.N = N;
  p.BH = BH;
  p.kv_group = H / H_kv;
  p.window = window;
  p.alibi = alibi_slopes;
  p.H = H;
  p.n_kv = (N + kBlockN - 1) / kBlockN;
  p.n_pairs = ((N + kBlockM - 1) / kBlockM + 1) / 2;
  if (static_cast<long long>(p.n_pairs) * BH > kMaxWorkItems) return FA_ERR_UNSUPPORTED;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.poly_pairs = poly_pairs(d);
  p.poly_deg = poly_degree();
  if (d == 256 && static_cast<long long>(p.n_kv) * BH > kMaxWorkItems) return FA_ERR_UNSUPPORTED;
  const bool q1 = d != 256 && fwd_q1(static_cast<long long>(p.n_pairs) * BH, p.sms);
  if (q1 && static_cast<long long>(p.n_kv) * BH > kMaxWorkItems) return FA_ERR_UNSUPPORTED;
  cudaError_t e = d == 256 ? launch_fwd_d256(p, causal != 0, static_cast<cudaStream_t>(stream))
                  : q1 ? launch_fwd_q1_bf16(p, d, causal != 0, static_cast<cudaStream_t>(stream))
                  : launch_fwd_tile_bf16(p, d, causal != 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

extern "C" fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int H, int N, int d, float scale, int causal, void* stream) {
  return fa_fwd_ex(q, k, v, o, lse, B, H, H, N, d, scale, causal, -1, nullptr, stream);
}

extern "C" size_t fa_bwd_deterministic_workspace_size(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128 && d != 256)) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  return (rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

// d = 256 has one backward (no dQ accumulator): the same workspace as the
// deterministic call.
extern "C" size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (d == 256) return fa_bwd_deterministic_workspace_size(B, H, N, d);
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128)) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return up(rows * d * sizeof(float)) + up(rows * sizeof(float));
}

extern "C" size_t fa_bwd_ex_workspace_size(int B, int H, int H_kv, int N, int d, int deterministic) {
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128 && d != 256) || H_kv < 1 || (H > 0 && H % H_kv)) return 0;
  const size_t base = deterministic ? fa_bwd_deterministic_workspace_size(B, H, N, d)
                                    : fa_bwd_workspace_size(B, H, N, d);
  const int S = H > 0 ? kv_split_for(B, H, H_kv, N, current_sms()) : 1;
  const size_t part = S > 1 ? static_cast<size_t>(S) * 2 * B * H_kv * N * d * sizeof(float) : 0;
  return base + round256(part);
}

namespace {

// Both backward variants: shared argument checks and tensor maps; the
// atomic one accumulates dQ in fp32 scratch by TMA reductions, the
// deterministic one runs the main kernel without dQ and the dQ kernel.
fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
                     int d, float scale, int causal, int window_left, const float* alibi_slopes,
                     void* workspace, size_t workspace_bytes, void* stream, bool deterministic) {
  fa_status st = check_shape(B, H, N, d, scale, true);
  if (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) return FA_ERR_MISALIGNED;
  if (st != FA_OK) return st;
  if (H > 0 && (st = check_kv_heads(H, H_kv)) != FA_OK) return st;
  int window = kNoWindow;
  if ((st = check_window(window_left, causal, &window)) != FA_OK) return st;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  // d = 256 has a single, reproducible backward (no dQ accumulator)
  if (d == 256) deterministic = true;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_bwd_ex_workspace_size(B, H, H_kv, N, d, deterministic ? 1 : 0);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != FA_OK) return st;

  const int BH = B * H;
  const long long rows = static_cast<long long>(BH) * N;
  float* dq_acc = deterministic ? nullptr : static_cast<float*>(workspace);
  float* delta = deterministic
                     ? static_cast<float*>(workspace)
                     : reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                ((static_cast<size_t>(rows) * d * 4 + 255) & ~static_cast<size_t>(255)));
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int BHkv = B * H_kv;
  if (!encode_3d(&p.tm_q, q, bf, 2, d, N, BH, 64, 128) || !encode_3d(&p.tm_k, k, bf, 2, d, N, BHkv, 64, 128) ||
      !encode_3d(&p.tm_v, v, bf, 2, d, N, BHkv, 64, 128) || !encode_3d(&p.tm_do, dout, bf, 2, d, N, BH, 64, 128))
    return FA_ERR_INVALID_ARG;
  if (!deterministic &&
      !encode_3d(&p.tm_dqacc, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, N, BH, 32, 128))
    return FA_ERR_INVALID_ARG;
  const bool pair = deterministic && d == 128 && bwd_pair() == 1;
  if ((pair || d == 256) && (!encode_3d(&p.tm_q64, q, bf, 2, d, N, BH, 64, 64) ||
                             !encode_3d(&p.tm_do64, dout, bf, 2, d, N, BH, 64, 64)))
    return FA_ERR_INVALID_ARG;
  if (d == 256 && (!encode_3d(&p.tm_k64, k, bf, 2, d, N, BHkv, 64, 64) ||
                   !encode_3d(&p.tm_v64, v, bf, 2, d, N, BHkv, 64, 64)))
    return FA_ERR_INVALID_ARG;
  p.lse = lse;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.dq = static_cast<uint16_t*>(dq);
  p.status = di->status;
  p.N = N;
  p.BH = BH;
  p.n_kv = (N + 127) / 128;
  p.n_q = (N + 127) / 128;
  p.kv_group = H / H_kv;
  p.window = window;
  p.alibi = alibi_slopes;
  p.H = H;
  p.kv_split = kv_split_for(B, H, H_kv, N, di->sms);
  p.kv_part = p.kv_split > 1
                  ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             (deterministic ? fa_bwd_deterministic_workspace_size(B, H, N, d)
                                                            : fa_bwd_workspace_size(B, H, N, d)))
                  : nullptr;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.poly_groups = bwd_poly_groups();
  p.dq_poly = dq_poly_pairs();
  p.group_kv = bwd_group_kv(BHkv, H / H_kv, N, d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_bwd_preprocess(static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout),
                                        delta, dq_acc, rows, d, s);
  if (e == cudaSuccess)
    e = d == 256 ? launch_bwd_kv256(p, causal != 0, s)
        : pair   ? launch_bwd_pair(p, causal != 0, s)
                 : launch_bwd_main(p, d, causal != 0, !deterministic, s);
  if (e == cudaSuccess && p.kv_split > 1)
    e = launch_bwd_kv_reduce(p.kv_part, p.dv, p.dk, static_cast<long long>(B) * H_kv * N * d, p.kv_split, s);
  if (e == cudaSuccess) {
    if (d == 256)
      e = launch_bwd_dq256(p, causal != 0, s);
    else if (deterministic)
      e = launch_bwd_dq(p, d, causal != 0, s);
    else
      e = launch_bwd_postprocess(dq_acc, static_cast<uint16_t*>(dq), rows * d, scale, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            int B, int H, int N, int d, float scale, int causal, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, H, H, N, d, scale, causal, -1, nullptr,
                    workspace, workspace_bytes, stream, false);
}

extern "C" fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                          const void* dout, const float* lse, void* dq, void* dk,
                                          void* dv, int B, int H, int N, int d, float scale,
                                          int causal, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, H, H, N, d, scale, causal, -1, nullptr,
                    workspace, workspace_bytes, stream, true);
}

extern "C" fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               int B, int H, int H_kv, int N, int d, float scale, int causal,
                               int window_left, const float* alibi_slopes, int deterministic,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, H, H_kv, N, d, scale, causal, window_left,
                    alibi_slopes, workspace, workspace_bytes, stream, deterministic != 0);
}

extern "C" fa_status fa_quant_fp8(const void* x, void* x8, float* scales, int B, int H, int N,
                                  int d, const float* signs, void* stream) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (N > kMaxN || static_cast<long long>(B) * H > kMaxBH) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!x || !x8 || !scales) return FA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || (reinterpret_cast<uintptr_t>(scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(signs) & 3u))
    return FA_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  cudaError_t e;
  if (d == 128) {
    QuantParams qp;
    std::memset(&qp, 0, sizeof(qp));
    if (!encode_3d(&qp.tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, B * H, 64, 128) ||
        !encode_3d(&qp.tm_x8, x8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, B * H, 128, 128))
      return FA_ERR_INVALID_ARG;
    qp.scales = scales;
    qp.signs = signs;
    qp.status = di->status;
    qp.N = N;
    qp.nblk = (N + 127) / 128;
    e = launch_quant_fp8_tma(qp, B * H, static_cast<cudaStream_t>(stream));
  } else {
    e = launch_quant_fp8(static_cast<const uint16_t*>(x), static_cast<uint8_t*>(x8), scales, signs,
                         B * H, N, d, static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

extern "C" fa_status fa_fwd_fp8_ex(const void* q8, const void* k8, const void* v8, const float* sq,
                                   const float* sk, const float* sv, void* o, float* lse, int B,
                                   int H, int H_kv, int N, int d, float scale, int causal,
                                   int window_left, const float* alibi_slopes, void* stream) {
  fa_status st = check_shape(B, H, N, d, scale);
  if (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) return FA_ERR_MISALIGNED;
  if (st != FA_OK) return st;
  if (H > 0 && (st = check_kv_heads(H, H_kv)) != FA_OK) return st;
  int window = kNoWindow;
  if ((st = check_window(window_left, causal, &window)) != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!q8 || !k8 || !v8 || !sq || !sk || !sv || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) ||
      ((reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(sq) |
        reinterpret_cast<uintptr_t>(sk) | reinterpret_cast<uintptr_t>(sv)) & 3u))
    return FA_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != FA_OK) return st;
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int BH = B * H;
  const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const int BHkv = B * H_kv;
  if (!encode_3d(&p.tm_q, q8, u8, 1, d, N, BH, 128, kBlockM) ||
      !encode_3d(&p.tm_k, k8, u8, 1, d, N, BHkv, 128, kBlockN) ||
      !encode_3d(&p.tm_v, v8, u8, 1, d, N, BHkv, 128, kBlockN))
    return FA_ERR_INVALID_ARG;
  p.o = static_cast<uint16_t*>(o);
  p.sms = di->sms;
  p.persistent = fwd_persistent(true, causal != 0, fp8_poly_pairs(), alibi_slopes);
  p.group_heads = fwd_group_heads(B * H, H / H_kv, N, d, 1, p.persistent != 0);
  if (!p.persistent &&
      !encode_3d(&p.tm_o, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, BH, 64, kBlockM))
    return FA_ERR_INVALID_ARG;
  p.lse = lse;
  p.status = di->status;
  p.sq = sq;
  p.sk = sk;
  p.sv = sv;
  p.N = N;
  p.BH = BH;
  p.kv_group = H / H_kv;
  p.window = window;
  p.alibi = alibi_slopes;
  p.H = H;
  p.n_kv = (N + kBlockN - 1) / kBlockN;
  p.n_pairs = ((N + kBlockM - 1) / kBlockM + 1) / 2;
  if (static_cast<long long>(p.n_pairs) * BH > kMaxWorkItems) return FA_ERR_UNSUPPORTED;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.poly_pairs = fp8_poly_pairs();
  p.poly_deg = poly_degree();
  cudaError_t e = launch_fwd_tile_fp8(p, causal != 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

extern "C" fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                                const float* sk, const float* sv, void* o, float* lse, int B, int H,
                                int N, int d, float scale, int causal, void* stream) {
  return fa_fwd_fp8_ex(q8, k8, v8, sq, sk, sv, o, lse, B, H, H, N, d, scale, causal, -1, nullptr,
                       stream);
}

namespace {

bool tuning_value_ok(int knob, int value) {
  if (value == -1) return true;
  switch (knob) {
    case FA_TUNE_FWD_POLY_PAIRS: return value == 0 || value == 2 || value == 4;
    case FA_TUNE_FWD_POLY_DEGREE: return value == 3 || value == 4;
    case FA_TUNE_BWD_POLY_GROUPS: return value == 0 || value == 1 || value == 2;
    case FA_TUNE_DQ_POLY_PAIRS: return value == 0 || value == 2 || value == 4;
    case FA_TUNE_FP8_POLY_PAIRS: return value == 0 || value == 2 || value == 4;
    case FA_TUNE_BWD_PAIR: return value == 0 || value == 1;
    case FA_TUNE_FWD_PERSISTENT: return value == 0 || value == 1;
    case FA_TUNE_FWD_CAUSAL_GROUP: return value == 0 || value == 1;
    case FA_TUNE_FWD_Q1: return value == 0 || value == 1;
    case FA_TUNE_BWD_CAUSAL_GROUP: return value == 0 || value == 1;
    default: return false;
  }
}

}  // namespace

extern "C" fa_status fa_set_tuning(int knob, int value) {
  if (knob <= 0 || knob >= FA_TUNE_COUNT || !tuning_value_ok(knob, value)) return FA_ERR_INVALID_ARG;
  g_tune[knob].store(value + 1, std::memory_order_relaxed);
  return FA_OK;
}

extern "C" int fa_get_tuning(int knob, int d) {
  switch (knob) {
    case FA_TUNE_FWD_POLY_PAIRS: return poly_pairs(d);
    case FA_TUNE_FWD_POLY_DEGREE: return poly_degree();
    case FA_TUNE_BWD_POLY_GROUPS: return bwd_poly_groups();
    case FA_TUNE_DQ_POLY_PAIRS: return d == 64 ? dq_poly_pairs() : 0;
    case FA_TUNE_FP8_POLY_PAIRS: return fp8_poly_pairs();
    case FA_TUNE_BWD_PAIR: return d == 128 ? bwd_pair() : 0;
    case FA_TUNE_FWD_PERSISTENT: return d == 256 ? 1 : tune_raw(FA_TUNE_FWD_PERSISTENT);   // -1: chosen per call
    case FA_TUNE_FWD_CAUSAL_GROUP: return tune_raw(FA_TUNE_FWD_CAUSAL_GROUP);   // -1: by the grid
    case FA_TUNE_FWD_Q1: return d == 256 ? 0 : tune_raw(FA_TUNE_FWD_Q1);   // -1: chosen per call
    case FA_TUNE_BWD_CAUSAL_GROUP: return bwd_causal_group();
    default: return -1;
  }
}

extern "C" fa_status fa_selftest_exp2(const float* x, float* y, long long n, int degree, void* stream) {
  if (n < 0 || (n & 1) || (degree != 0 && degree != 3 && degree != 4 && degree != 5))
    return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!x || !y) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 7u) return FA_ERR_MISALIGNED;
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  if (launch_selftest_exp2(x, y, n, degree, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

extern "C" fa_status fa_selftest_wait_timeout(void* stream) {
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  if (launch_selftest_wait(di->status, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

extern "C" unsigned int fa_get_status(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  return v;
}

extern "C" void fa_clear_status(void) {
  const unsigned int z = 0;
  if (cudaMemcpyToSymbol(fa::g_status, &z, sizeof(z)) != cudaSuccess) cudaGetLastError();
}

extern "C" const char* fa_status_string(int s) {
  switch (s & 0xFF) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH";
    case FA_ERR_PIPELINE_TIMEOUT: return "FA_ERR_PIPELINE_TIMEOUT";
    case FA_ERR_NO_DEVICE: return "FA_ERR_NO_DEVICE";
    case FA_ERR_SCRATCH_LIMIT: return "FA_ERR_SCRATCH_LIMIT";
    default: return "FA_ERR_UNKNOWN";
  }
}
