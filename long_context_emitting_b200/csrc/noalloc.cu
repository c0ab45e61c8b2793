// kascade_decode_anchor_static_ws: the decode anchor with its scratch memory in
// a fixed array that the library itself owns, for callers that must not
// allocate device memory while they run (see include/kascade.h).
//
// The array lives in this file as a file-scope __device__ object.  Host code
// cannot use its name as a device address, so the address is looked up once
// per device with cudaGetSymbolAddress and handed to the regular launcher.
#include "../../include/kascade.h"
#include "internal.h"

#include <cuda_runtime.h>

#include <atomic>

namespace kascade {

static __device__ __align__(256) unsigned char g_static_scratch[KASCADE_STATIC_SCRATCH_BYTES];

}  // namespace kascade

namespace {

constexpr int kMaxDevices = 64;

// Device address of g_static_scratch on the current device, looked up on the
// first call per device (the lookup may load the module on that device, which
// is why the first call should not happen inside a stream capture).  Threads
// that race on a first call all store the same address.
void* static_scratch_address() {
  static std::atomic<void*> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = cache[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, kascade::g_static_scratch) != cudaSuccess) return nullptr;
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace

extern "C" int kascade_decode_anchor_static_ws(kascade_shape s, const uint16_t* q,
                                               const uint16_t* k, const uint16_t* v,
                                               const int64_t* kv_off, const int32_t* seq_len,
                                               int32_t max_T, float scale, uint16_t* out,
                                               float* lse, float* pooled, int64_t ld_pooled,
                                               void* stream) {
  // The regular entry point's argument checks come first, in its order, so a
  // bad argument gets the same code from both; only then the size limit.
  const int rc = kascade::decode_anchor_check_args(s, q, k, v, kv_off, seq_len, max_T, scale, out,
                                                   lse, pooled, ld_pooled);
  if (rc != KASCADE_OK || s.B == 0) return rc;
  const size_t need = kascade_decode_anchor_workspace_bytes(s, max_T);
  if (need > (size_t)KASCADE_STATIC_SCRATCH_BYTES) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  void* ws = static_scratch_address();
  if (!ws) return KASCADE_ERR_CUDA;
  // Nothing in the scratch needs to start at zero: every partial and logit the
  // combine step reads is written earlier in the same call.
  return kascade_decode_anchor(s, q, k, v, kv_off, seq_len, max_T, scale, out, lse, pooled,
                               ld_pooled, ws, (size_t)KASCADE_STATIC_SCRATCH_BYTES, stream);
}
