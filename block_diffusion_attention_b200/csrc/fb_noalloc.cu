// fb_noalloc.cu -- the prefix pass for callers that cannot allocate device
// memory.
//
// Some callers are not allowed to call cudaMalloc at all: an embedding whose
// memory planner hands out one fixed device arena at start-up and forbids
// allocator calls once it is running, a plug-in host that gives its plug-ins
// no allocator of their own, or a latency-critical serving loop that cannot
// afford the device-wide synchronisation a cudaMalloc or cudaFree may cause.
// For them the split-key partials of the prefix pass live in a fixed scratch
// array that is part of this library's device image instead of a
// caller-owned workspace.
//
// The array (FB_NOALLOC_SCRATCH_BYTES, 16 MiB) exists on every GPU that loads
// the library, for as long as the process runs.  All calls share it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "fb_internal.h"

namespace {

constexpr size_t kScratchBytes = FB_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

DriverFns driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

// Unique id of the calling thread's current context (0 if there is none yet
// or the driver cannot say).  A device reset ends the context: the next one
// gets a new id, and the library's device image (with the array) is loaded
// into it again, possibly at another address.
unsigned long long current_context_id() {
  const DriverFns f = driver_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct ScratchEntry {
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[64];  // per device

// On the host, g_noalloc_scratch names a host-side stand-in, not device
// memory: the kernels need the array's device address, looked up with the
// device current, once per device and again whenever the device's context has
// changed (after a device reset).
fb_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FB_ERR_LAUNCH;
  if (dev < 0 || dev >= 64) return FB_ERR_UNSUPPORTED;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& e = g_scratch[dev];
  if (!e.addr || id == 0 || id != e.ctx_id) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // do not leave the error for the caller's next call
      return FB_ERR_LAUNCH;
    }
    e.addr = p;
    // the lookup above created the context if there was none
    e.ctx_id = current_context_id();
  }
  *out = e.addr;
  return FB_OK;
}

}  // namespace

extern "C" fb_status fb_prefix_partial_noalloc(const fb_desc* d, const void* Q, const void* Kcache,
                                               const void* Vcache, const int32_t* chunk_idx,
                                               float* O_pre, float* LSE_pre, int32_t* dev_status,
                                               fb_stream_t stream) {
  void* scratch = nullptr;
  const fb_status st = scratch_address(&scratch);
  if (st != FB_OK) return st;
  // The regular entry point checks the arguments and returns
  // FB_ERR_WORKSPACE, before launching anything, when this call's split
  // partials need more than the array holds.  Every split CTA writes all of
  // its rows, so nothing in the array has to start at zero.
  return fb_prefix_partial(d, Q, Kcache, Vcache, chunk_idx, O_pre, LSE_pre, scratch, kScratchBytes,
                           dev_status, stream);
}
