// decode_noalloc.cu -- gdla_decode for callers that cannot hand the library a
// workspace: the decode scratch (status word, query images, split partials)
// lives in a fixed device array that belongs to this library.
//
// Who needs this: code that must not allocate device memory at call time, e.g.
// a latency-bound serving loop, where an allocation can block on the device or
// fail under memory pressure in the middle of a step, or a host framework or
// plugin that only passes the input and output buffers it owns and has no
// device allocator to offer.
#include <cuda.h>

#include <mutex>

#include "../../include/gdla.h"
#include "common.cuh"

namespace {

// The scratch every call shares. Every GPU that loads the library keeps these
// 32 MiB until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[GDLA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;

// cuCtxGetCurrent through the runtime's driver entry-point query (the library does
// not link libcuda directly); a null result means "context unknown"
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}
struct ScratchAddr {
  CUcontext ctx;  // the context the address belongs to
  void* ptr;
};
ScratchAddr g_scratch[kMaxDevices] = {};

// Device address of the scratch array in the current context. On the host the
// name g_decode_scratch is only a stand-in for the symbol, not a device
// pointer, so the address is looked up with the device current and cached per
// device together with its context: after a device reset the library's module
// is loaded again in a new context, and the address is looked up again.
gdla_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return GDLA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  // the runtime makes the device's primary context current when it looks the symbol up;
  // a first call on a thread may see no current context yet, and then looks up anew
  CUcontext ctx = current_context();
  if (!g_scratch[dev].ptr || !ctx || g_scratch[dev].ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return GDLA_ERR_CUDA;
    }
    g_scratch[dev] = ScratchAddr{current_context(), p};
  }
  *out = g_scratch[dev].ptr;
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
