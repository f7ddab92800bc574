// fb_noalloc.cu -- the prefix pass for callers that cannot allocate device
// memory.
//
// Some callers are not allowed to call cudaMalloc at all: a host program that
// records its work into a CUDA graph (allocation is not a capturable
// operation), an embedding that owns a fixed device-memory arena and forbids
// allocator calls once it is running, or a serving loop that cannot afford
// the device-wide synchronisation an allocation may cause.  For them the
// split-key partials of the prefix pass live in a fixed scratch array that is
// part of this library's device image instead of a caller-owned workspace.
//
// The array (FB_NOALLOC_SCRATCH_BYTES, 16 MiB) exists on every GPU that loads
// the library, for as long as the process runs.  All calls share it.
#include <cuda_runtime.h>

#include <mutex>

#include "fb_internal.h"

namespace {

constexpr size_t kScratchBytes = FB_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};  // device address of the array, per device

// On the host, g_noalloc_scratch names a host-side shadow, not device memory;
// the kernels need the device address, looked up once per device with that
// device current.
fb_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FB_ERR_LAUNCH;
  if (dev < 0 || dev >= 64) return FB_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // do not leave the error for the caller's next call
      return FB_ERR_LAUNCH;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
