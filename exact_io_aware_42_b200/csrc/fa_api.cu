// C-ABI layer: argument validation, TMA tensor-map encoding, the device
// status word, and dispatch to the kernels.  See include/fa.h for the
// contract of each entry point.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
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

struct DeviceInfo {
  bool probed = false;
  bool ok = false;
  unsigned int* status = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Current device checked once: sm_100 present, status-word address, driver
// entry point for tensor-map encoding.
fa_status current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.probed) {
    di.probed = true;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_DEVICE;
    }
    if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_DEVICE;
    }
    di.status = static_cast<unsigned int*>(addr);
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
    di.ok = true;
  }
  if (!di.ok) return FA_ERR_UNSUPPORTED;
  *out = &di;
  return FA_OK;
}

// Share of the exp2 work on the FMA pipe (pairs of 8); FA_POLY_PAIRS in the
// environment overrides the per-d default for measurement (0, 2 or 4).
int poly_pairs(int d) {
  static int env = [] {
    const char* e = std::getenv("FA_POLY_PAIRS");
    if (!e) return -1;
    const int x = std::atoi(e);
    return (x == 0 || x == 2 || x == 4) ? x : -1;
  }();
  if (env >= 0) return env;
  return d == 64 ? kDefaultPolyPairsD64 : kDefaultPolyPairsD128;
}

// Backward P-phase exp2 share on the FMA pipe (groups of 4); FA_BWD_POLY
// overrides the default for measurement (0, 1 or 2).
int bwd_poly_groups() {
  static int v = [] {
    const char* e = std::getenv("FA_BWD_POLY");
    const int x = e ? std::atoi(e) : -1;
    return (x == 0 || x == 1 || x == 2) ? x : kDefaultBwdPolyGroups;
  }();
  return v;
}

// Deterministic dQ kernel at d = 64: FA_DQ_POLY in {0, 2, 4} overrides the default share.
int dq_poly_pairs() {
  const char* s = std::getenv("FA_DQ_POLY");
  if (s && *s) {
    const int x = std::atoi(s);
    if (x == 0 || x == 2 || x == 4) return x;
  }
  return kDefaultDqPolyPairsD64;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D view [BH, N, d] of a contiguous [B, H, N, d] tensor, 128-byte swizzle,
// box {box_inner elements, box_rows, 1}; out-of-range elements read as zero
// and are skipped on store.
bool encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int d, int N,
               int BH, int box_inner, int box_rows) {
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

fa_status check_shape(int B, int H, int N, int d, float scale) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (N > kMaxN || static_cast<long long>(B) * H > kMaxBH) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Grouped K/V heads: 1 <= H_kv, H a multiple of H_kv.
fa_status check_kv_heads(int H, int H_kv) {
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// CTAs sharing one (K/V head, key block) in the backward: the smallest
// divisor S of G = H / H_kv that gives the grid about three CTAs per SM of
// the B200 (148 SMs), so that few K/V heads (MQA) still fill the GPU; 1 when
// the grid is large enough already.
int kv_split_for(int B, int H, int H_kv, int N) {
  const int G = H / H_kv;
  const long long ctas = static_cast<long long>(B) * H_kv * ((N + 127) / 128);
  int S = 1;
  while (S < G && ctas * S < 3 * 148) {
    int next = S + 1;
    while (G % next) ++next;
    S = next;
  }
  return S;
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
  fa_status st = check_shape(B, H, N, d, scale);
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
      !encode_3d(&p.tm_v, v, bf, 2, d, N, BHkv, 64, kBlockN) ||
      !encode_3d(&p.tm_o, o, bf, 2, d, N, BH, 64, kBlockM))
    return FA_ERR_INVALID_ARG;
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
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.poly_pairs = poly_pairs(d);
  cudaError_t e = launch_fwd_bf16(p, d, causal != 0, static_cast<cudaStream_t>(stream));
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

extern "C" size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128)) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return up(rows * d * sizeof(float)) + up(rows * sizeof(float));
}

extern "C" size_t fa_bwd_deterministic_workspace_size(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128)) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  return (rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

extern "C" size_t fa_bwd_ex_workspace_size(int B, int H, int H_kv, int N, int d, int deterministic) {
  if (B < 0 || H < 0 || N < 0 || (d != 64 && d != 128) || H_kv < 1 || (H > 0 && H % H_kv)) return 0;
  const size_t base = deterministic ? fa_bwd_deterministic_workspace_size(B, H, N, d)
                                    : fa_bwd_workspace_size(B, H, N, d);
  const int S = H > 0 ? kv_split_for(B, H, H_kv, N) : 1;
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
  fa_status st = check_shape(B, H, N, d, scale);
  if (reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) return FA_ERR_MISALIGNED;
  if (st != FA_OK) return st;
  if (H > 0 && (st = check_kv_heads(H, H_kv)) != FA_OK) return st;
  int window = kNoWindow;
  if ((st = check_window(window_left, causal, &window)) != FA_OK) return st;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
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
  p.kv_split = kv_split_for(B, H, H_kv, N);
  p.kv_part = p.kv_split > 1
                  ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             (deterministic ? fa_bwd_deterministic_workspace_size(B, H, N, d)
                                                            : fa_bwd_workspace_size(B, H, N, d)))
                  : nullptr;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.poly_groups = bwd_poly_groups();
  p.dq_poly = dq_poly_pairs();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_bwd_preprocess(static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout),
                                        delta, dq_acc, rows, d, s);
  if (e == cudaSuccess) e = launch_bwd_main(p, d, causal != 0, !deterministic, s);
  if (e == cudaSuccess && p.kv_split > 1)
    e = launch_bwd_kv_reduce(p.kv_part, p.dv, p.dk, static_cast<long long>(B) * H_kv * N * d, p.kv_split, s);
  if (e == cudaSuccess) {
    if (deterministic)
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
      !encode_3d(&p.tm_v, v8, u8, 1, d, N, BHkv, 128, kBlockN) ||
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
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaError_t e = launch_fwd_fp8(p, causal != 0, static_cast<cudaStream_t>(stream));
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
