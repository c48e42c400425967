// decode_noalloc.cu -- gdla_decode for callers that cannot hand the library a
// workspace: the decode scratch (status word, absorbed queries, split
// partials) lives in a fixed device array that belongs to this library.
//
// Who needs this: code that must not allocate device memory at call time,
// e.g. a step replayed inside a captured CUDA graph whose allocator is frozen,
// a real-time serving loop where an allocation could synchronise the device or
// fail under memory pressure, or a host framework/plugin that only passes the
// input and output buffers it owns and has no allocator to offer.
#include <mutex>

#include "../../include/gdla.h"
#include "common.cuh"

namespace {

// The scratch every call shares. Every GPU that loads the library keeps these
// 32 MiB until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[GDLA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The host-side
// name g_decode_scratch is only a stand-in for the symbol, not a device
// pointer, so the address is looked up once per device (with that device
// current) and cached.
gdla_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return GDLA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return GDLA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GDLA_OK;
}

}  // namespace

extern "C" gdla_status gdla_decode_noalloc(const gdla_decode_args* args, void* stream) {
  if (!args) return GDLA_ERR_INVALID_ARG;
  const size_t need = gdla_decode_workspace_size(args);
  if (need == 0) return GDLA_ERR_INVALID_ARG;
  if (need > (size_t)GDLA_DECODE_NOALLOC_SCRATCH_BYTES) return GDLA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  gdla_status st = scratch_on_current_device(&scratch);
  if (st != GDLA_OK) return st;
  gdla_decode_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = GDLA_DECODE_NOALLOC_SCRATCH_BYTES;
  // gdla_decode clears the status word at the start of the scratch on `stream`;
  // everything else it reads is written earlier in the same call.
  return gdla_decode(&a, stream);
}
