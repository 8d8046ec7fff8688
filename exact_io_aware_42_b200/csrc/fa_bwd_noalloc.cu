// fa_bwd_noalloc: the attention backward with its scratch memory built into
// the library, for callers that cannot allocate device memory themselves --
// for instance code running inside a host framework that owns every device
// allocation through its own memory pool and forbids extra raw allocations,
// or a latency-critical path where a cudaMalloc (which can synchronise the
// whole device) is not acceptable.
//
// The scratch (fp32 dQ accumulator and the per-row D of the backward) lives
// in one file-scope device array of FA_BWD_NOALLOC_SCRATCH_BYTES.  Every GPU
// that loads the library holds that array until the process exits.  Nothing
// here calls cudaMalloc, cudaFree or any allocating routine.
//
// Host code cannot pass the array's name to a kernel: on the host that name
// is only a stand-in object, not a device address.  The device address is
// therefore looked up once per device, with that device current, through
// cudaGetSymbolAddress, the first time this entry point runs on it; that
// first call should come before any stream capture.  The address is kept
// together with the unique id of the CUDA context it was found in: after a
// device reset the module is loaded again into a new context, possibly at
// another address, so a changed context id triggers a new lookup.
//
// All calls share the one array and it keeps the previous call's contents;
// the part that must start at zero (the dQ accumulator) is cleared by the
// backward's own preprocessing kernel on every call.  Calls whose work can
// overlap on the GPU (different streams, or different host threads without
// ordering between them) race on the array and give wrong gradients:
// serialise them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"

namespace {

constexpr int kMaxDevicesNoAlloc = 64;

static __device__ __align__(256) unsigned char g_bwd_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

struct ScratchSlot {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;
};

std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevicesNoAlloc];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context (driver entry points looked up once;
// 0 if unavailable, which then only disables the reset check).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(fn);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
      get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of g_bwd_scratch on the current device (looked up once per
// device and context).
fa_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesNoAlloc) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  // (Before the first runtime call on this device there may be no context
  // yet: cudaGetSymbolAddress creates it, and the id is read after it.)
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  unsigned long long id = current_context_id();
  if (slot.addr == nullptr || (id != 0 && id != slot.ctx_id)) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return FA_ERR_NO_DEVICE;
    }
    slot.addr = ptr;
    slot.ctx_id = current_context_id();
  }
  *out = slot.addr;
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                    const void* dout, const float* lse, void* dq, void* dk,
                                    void* dv, int B, int H, int N, int d, float scale, int causal,
                                    void* stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_SCRATCH_LIMIT;
  if (need == 0) {
    // unsupported d or negative sizes, or an empty problem: the regular entry
    // point reports which, without touching the scratch
    return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, nullptr, 0, stream);
  }
  void* scratch = nullptr;
  const fa_status st = scratch_address(&scratch);
  if (st != FA_OK) return st;
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, scratch,
                FA_BWD_NOALLOC_SCRATCH_BYTES, stream);
}
