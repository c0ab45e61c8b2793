// Diagnostic kernel for the failure path of the bounded waits: a wait that can
// only end by its time limit.  It exercises exactly the code the prefill
// kernels run when a barrier is never completed (mbar_wait / mbar_spin), so a
// test can check on the GPU that such a wait ends and that the host reads the
// timeout from the status word, with no fault and the context still usable.
#include "tcgen05.cuh"
#include "internal.h"

namespace kascade {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int spin, unsigned* status) {
  __shared__ __align__(8) uint64_t bar;  // no thread ever arrives on it
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Phase 0 of a fresh barrier stays incomplete: only the ~2 s limit ends the wait.
    if (spin) mbar_spin(smem_u32(&bar), 0, status);
    else mbar_wait(smem_u32(&bar), 0, status);
  }
}

}  // namespace

cudaError_t launch_wait_timeout(bool spin, unsigned* status, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(spin ? 1 : 0, status);
  return cudaGetLastError();
}

}  // namespace kascade
