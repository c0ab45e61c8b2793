// Prefill-phase Kascade kernels (tcgen05 / TMEM): not yet implemented.
#include "common.cuh"
#include "internal.h"

namespace kascade {

size_t prefill_anchor_workspace_bytes(int, int, int, int) { return 0; }
size_t prefill_reuse_workspace_bytes(int, int, int, int, int) { return 0; }
cudaError_t launch_prefill_anchor(const PrefillParams&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_prefill_reuse(const PrefillParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kascade
