// diag.cu -- a diagnostic kernel for the failure path of the bounded device
// waits: one thread waits on an mbarrier that nothing ever arrives on. The wait
// gives up after its limit (the one every kernel wait uses) and records
// GDLA_ERR_TIMEOUT plus a tag in the caller's status word, which the host then
// reads with gdla_workspace_status. No trap, no invalid access, no endless loop.
#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace {

constexpr int kDiagTag = 901;

__global__ void diag_wait_kernel(int* status) {
  using namespace sm100;
  __shared__ __align__(8) uint64_t never;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&never), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&never), 0, status, kDiagTag);
}

}  // namespace

cudaError_t launch_diag_wait(int* status, cudaStream_t s) {
  diag_wait_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

}  // namespace gdla
