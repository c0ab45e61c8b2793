// C ABI of the Kascade hot path: argument checks, workspace sizing, the sticky
// device status word, and dispatch to the kernel launchers.  See
// include/kascade.h for the contract of every entry point.
#include "../../include/kascade.h"
#include "common.cuh"
#include "internal.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

namespace kascade {
__device__ unsigned int g_device_status = 0u;
}

using namespace kascade;

namespace {

constexpr int kMaxDevices = 64;

// Device address of the status word on the current device, looked up once per
// device; threads that race on a first call all store the same address.
unsigned* device_status_ptr() {
  static std::atomic<unsigned*> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned* p = cache[dev].load(std::memory_order_acquire);
  if (!p) {
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_device_status) != cudaSuccess) return nullptr;
    p = static_cast<unsigned*>(q);
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(const kascade_shape& s) {
  if (s.B < 0 || s.Hq <= 0 || s.Hkv <= 0) return KASCADE_ERR_INVALID_ARG;
  if (s.d != kHeadDim) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  if (s.Hq % s.Hkv) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  const int G = s.Hq / s.Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  return KASCADE_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? KASCADE_OK : KASCADE_ERR_CUDA; }

// The decode anchor's workspace holds B·Hq·max_T fp32 logits plus smaller
// partials.  Shapes past 2^46 logits (256 TiB) are refused, so no workspace
// size computation can wrap around.
bool decode_logits_too_large(const kascade_shape& s, int32_t max_T) {
  const uint64_t heads = (uint64_t)s.B * (uint64_t)s.Hq;  // < 2^62
  return heads != 0 && (uint64_t)max_T > (1ull << 46) / heads;
}

// Per-row lengths (max_T, k_max) above 2^30 are refused: the kernels index a
// row's tokens with 32-bit integers and round split sizes up, which must not
// overflow (a 2^30-token row is already 512 GiB of K/V per key head).
constexpr int32_t kMaxRowLen = 1 << 30;

}  // namespace

extern "C" {

int32_t kascade_k_for_len(int32_t n) {
  if (n <= 0) return 0;
  const int32_t tenth = (int32_t)(((int64_t)n + 5) / 10);
  const int32_t k = tenth > 128 ? tenth : 128;
  return k < n ? k : n;
}

const char* kascade_status_string(int status) {
  switch (status) {
    case KASCADE_OK: return "KASCADE_OK";
    case KASCADE_ERR_INVALID_ARG: return "KASCADE_ERR_INVALID_ARG";
    case KASCADE_ERR_UNSUPPORTED_SHAPE: return "KASCADE_ERR_UNSUPPORTED_SHAPE";
    case KASCADE_ERR_WORKSPACE_TOO_SMALL: return "KASCADE_ERR_WORKSPACE_TOO_SMALL";
    case KASCADE_ERR_CUDA: return "KASCADE_ERR_CUDA";
    case KASCADE_ERR_BAD_INDEX: return "KASCADE_ERR_BAD_INDEX";
    case KASCADE_ERR_NONFINITE: return "KASCADE_ERR_NONFINITE";
    case KASCADE_ERR_TIMEOUT: return "KASCADE_ERR_TIMEOUT";
    default: return "KASCADE_ERR_UNKNOWN";
  }
}

int kascade_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KASCADE_ERR_CUDA;
  unsigned v = 0u;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return KASCADE_ERR_CUDA;
  const unsigned zero = 0u;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return KASCADE_ERR_CUDA;
  if (v & kStatusTimeout) return KASCADE_ERR_TIMEOUT;
  if (v & kStatusBadIndex) return KASCADE_ERR_BAD_INDEX;
  if (v & kStatusNonFinite) return KASCADE_ERR_NONFINITE;
  return KASCADE_OK;
}

int kascade_selftest_wait_timeout(int32_t spin, void* stream) {
  unsigned* status = device_status_ptr();
  if (!status) return KASCADE_ERR_CUDA;
  return from_cuda(launch_wait_timeout(spin != 0, status, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ decode --
size_t kascade_decode_anchor_workspace_bytes(kascade_shape s, int32_t max_T) {
  if (check_shape(s) != KASCADE_OK || max_T < 0 || max_T > kMaxRowLen || decode_logits_too_large(s, max_T))
    return 0;
  return decode_workspace_bytes(s.B, s.Hkv, s.Hq / s.Hkv, max_T, true);
}

}  // extern "C"

// Every host check of the decode anchor except the workspace ones, in the
// order the entry points apply them (also used by the static-scratch entry).
int kascade::decode_anchor_check_args(kascade_shape s, const uint16_t* q, const uint16_t* k,
                                      const uint16_t* v, const int64_t* kv_off,
                                      const int32_t* seq_len, int32_t max_T, float scale,
                                      const uint16_t* out, const float* lse, const float* pooled,
                                      int64_t ld_pooled) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (max_T < 0 || ld_pooled < max_T || (ld_pooled & 3) || !std::isfinite(scale))
    return KASCADE_ERR_INVALID_ARG;
  if (max_T > kMaxRowLen || decode_logits_too_large(s, max_T)) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  if (s.B == 0) return KASCADE_OK;
  if (!q || !k || !v || !kv_off || !seq_len || !out || !pooled) return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(pooled) ||
      (lse && !aligned16(lse)) || ((uintptr_t)kv_off & 7) || ((uintptr_t)seq_len & 3))
    return KASCADE_ERR_INVALID_ARG;
  return KASCADE_OK;
}

extern "C" {

static int kascade_decode_anchor_impl(kascade_shape s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                          int32_t max_T, float scale, uint16_t* out, float* lse,
                          float* pooled, int64_t ld_pooled, void* ws, size_t ws_bytes,
                          void* stream, bool f16) {
  int rc = decode_anchor_check_args(s, q, k, v, kv_off, seq_len, max_T, scale, out, lse, pooled, ld_pooled);
  if (rc || s.B == 0) return rc;
  if (!ws || !aligned16(ws)) return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < kascade_decode_anchor_workspace_bytes(s, max_T)) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  DecodeParams p = {};
  p.f16 = f16;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv;
  p.q = q; p.k = k; p.v = v; p.kv_off = kv_off; p.seq_len = seq_len; p.max_T = max_T;
  p.scale = scale; p.out = out; p.lse = lse; p.pooled = pooled; p.ld_pooled = ld_pooled;
  p.ws = ws;
  p.status = device_status_ptr();
  if (!p.status) return KASCADE_ERR_CUDA;
  return from_cuda(launch_decode_anchor(p, static_cast<cudaStream_t>(stream)));
}

int kascade_decode_anchor(kascade_shape s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                          int32_t max_T, float scale, uint16_t* out, float* lse,
                          float* pooled, int64_t ld_pooled, void* ws, size_t ws_bytes,
                          void* stream) {
  return kascade_decode_anchor_impl(s, q, k, v, kv_off, seq_len, max_T, scale, out, lse, pooled, ld_pooled, ws, ws_bytes, stream, false);
}

int kascade_decode_anchor_f16(kascade_shape s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                          int32_t max_T, float scale, uint16_t* out, float* lse,
                          float* pooled, int64_t ld_pooled, void* ws, size_t ws_bytes,
                          void* stream) {
  return kascade_decode_anchor_impl(s, q, k, v, kv_off, seq_len, max_T, scale, out, lse, pooled, ld_pooled, ws, ws_bytes, stream, true);
}

size_t kascade_decode_reuse_workspace_bytes(kascade_shape s, int32_t k_max) {
  if (check_shape(s) != KASCADE_OK || k_max < 0 || k_max > kMaxRowLen) return 0;
  return decode_workspace_bytes(s.B, s.Hkv, s.Hq / s.Hkv, k_max, false);
}

static int kascade_decode_reuse_impl(kascade_shape s, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                         const int32_t* idx, const int32_t* idx_k, int32_t k_max,
                         const int32_t* head_map, float scale, uint16_t* out, float* lse,
                         void* ws, size_t ws_bytes, void* stream, bool f16) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (k_max < 0 || !std::isfinite(scale)) return KASCADE_ERR_INVALID_ARG;
  if (k_max > kMaxRowLen) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  if (s.B == 0) return KASCADE_OK;
  const size_t need = kascade_decode_reuse_workspace_bytes(s, k_max);
  if (!q || !k || !v || !kv_off || !seq_len || !idx || !idx_k || !head_map || !out || (need && !ws))
    return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (ws && !aligned16(ws)) ||
      (lse && !aligned16(lse)) || ((uintptr_t)kv_off & 7) || ((uintptr_t)seq_len & 3) ||
      ((uintptr_t)idx & 3) || ((uintptr_t)idx_k & 3) || ((uintptr_t)head_map & 3))
    return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < need) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  DecodeParams p = {};
  p.f16 = f16;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv;
  p.q = q; p.k = k; p.v = v; p.kv_off = kv_off; p.seq_len = seq_len;
  p.max_T = 0x7fffffff;  // index validity is checked against each seq_len
  p.idx = idx; p.idx_k = idx_k; p.head_map = head_map; p.k_max = k_max;
  p.scale = scale; p.out = out; p.lse = lse; p.ws = ws;
  p.status = device_status_ptr();
  if (!p.status) return KASCADE_ERR_CUDA;
  return from_cuda(launch_decode_reuse(p, static_cast<cudaStream_t>(stream)));
}

int kascade_decode_reuse(kascade_shape s, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                         const int32_t* idx, const int32_t* idx_k, int32_t k_max,
                         const int32_t* head_map, float scale, uint16_t* out, float* lse,
                         void* ws, size_t ws_bytes, void* stream) {
  return kascade_decode_reuse_impl(s, q, k, v, kv_off, seq_len, idx, idx_k, k_max, head_map, scale, out, lse, ws, ws_bytes, stream, false);
}

int kascade_decode_reuse_f16(kascade_shape s, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                         const int32_t* idx, const int32_t* idx_k, int32_t k_max,
                         const int32_t* head_map, float scale, uint16_t* out, float* lse,
                         void* ws, size_t ws_bytes, void* stream) {
  return kascade_decode_reuse_impl(s, q, k, v, kv_off, seq_len, idx, idx_k, k_max, head_map, scale, out, lse, ws, ws_bytes, stream, true);
}

// ------------------------------------------------------------ decode, paged --
static int check_pages(const uint16_t* k, const uint16_t* v, const int32_t* block_table,
                       int32_t num_pages, int32_t max_pages, int32_t page_size) {
  if (!k || !v || !block_table || num_pages < 1 || max_pages < 1 || page_size < 16 ||
      (page_size % 16))
    return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || ((uintptr_t)block_table & 3)) return KASCADE_ERR_INVALID_ARG;
  return KASCADE_OK;
}

static int kascade_decode_anchor_paged_impl(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                const uint16_t* v_pages, int32_t num_pages,
                                const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                const int32_t* seq_len, int32_t max_T, float scale, uint16_t* out,
                                float* lse, float* pooled, int64_t ld_pooled, void* ws,
                                size_t ws_bytes, void* stream, bool f16) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (max_T < 0 || ld_pooled < max_T || (ld_pooled & 3) || !std::isfinite(scale))
    return KASCADE_ERR_INVALID_ARG;
  if (max_T > kMaxRowLen || decode_logits_too_large(s, max_T)) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  if (s.B == 0) return KASCADE_OK;
  if ((rc = check_pages(k_pages, v_pages, block_table, num_pages, max_pages, page_size))) return rc;
  if ((int64_t)max_pages * page_size < max_T) return KASCADE_ERR_INVALID_ARG;
  if (!q || !seq_len || !out || !pooled || !ws) return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(pooled) || !aligned16(ws) ||
      (lse && !aligned16(lse)) || ((uintptr_t)seq_len & 3))
    return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < kascade_decode_anchor_workspace_bytes(s, max_T)) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  DecodeParams p = {};
  p.f16 = f16;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv;
  p.q = q; p.k = k_pages; p.v = v_pages; p.seq_len = seq_len; p.max_T = max_T;
  p.block_table = block_table; p.max_pages = max_pages; p.page_size = page_size;
  p.num_pages = num_pages;
  p.scale = scale; p.out = out; p.lse = lse; p.pooled = pooled; p.ld_pooled = ld_pooled;
  p.ws = ws;
  p.status = device_status_ptr();
  if (!p.status) return KASCADE_ERR_CUDA;
  return from_cuda(launch_decode_anchor(p, static_cast<cudaStream_t>(stream)));
}

int kascade_decode_anchor_paged(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                const uint16_t* v_pages, int32_t num_pages,
                                const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                const int32_t* seq_len, int32_t max_T, float scale, uint16_t* out,
                                float* lse, float* pooled, int64_t ld_pooled, void* ws,
                                size_t ws_bytes, void* stream) {
  return kascade_decode_anchor_paged_impl(s, q, k_pages, v_pages, num_pages, block_table, max_pages, page_size,
                                          seq_len, max_T, scale, out, lse, pooled, ld_pooled, ws, ws_bytes,
                                          stream, false);
}

int kascade_decode_anchor_paged_f16(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                    const uint16_t* v_pages, int32_t num_pages,
                                    const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                    const int32_t* seq_len, int32_t max_T, float scale, uint16_t* out,
                                    float* lse, float* pooled, int64_t ld_pooled, void* ws,
                                    size_t ws_bytes, void* stream) {
  return kascade_decode_anchor_paged_impl(s, q, k_pages, v_pages, num_pages, block_table, max_pages, page_size,
                                          seq_len, max_T, scale, out, lse, pooled, ld_pooled, ws, ws_bytes,
                                          stream, true);
}

static int kascade_decode_reuse_paged_impl(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                               const uint16_t* v_pages, int32_t num_pages,
                               const int32_t* block_table, int32_t max_pages, int32_t page_size,
                               const int32_t* seq_len, const int32_t* idx, const int32_t* idx_k,
                               int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                               float* lse, void* ws, size_t ws_bytes, void* stream, bool f16) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (k_max < 0 || !std::isfinite(scale)) return KASCADE_ERR_INVALID_ARG;
  if (k_max > kMaxRowLen) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  if (s.B == 0) return KASCADE_OK;
  if ((rc = check_pages(k_pages, v_pages, block_table, num_pages, max_pages, page_size))) return rc;
  const size_t need = kascade_decode_reuse_workspace_bytes(s, k_max);
  if (!q || !seq_len || !idx || !idx_k || !head_map || !out || (need && !ws))
    return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || (ws && !aligned16(ws)) || (lse && !aligned16(lse)) ||
      ((uintptr_t)seq_len & 3) || ((uintptr_t)idx & 3) || ((uintptr_t)idx_k & 3) ||
      ((uintptr_t)head_map & 3))
    return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < need) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  DecodeParams p = {};
  p.f16 = f16;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv;
  p.q = q; p.k = k_pages; p.v = v_pages; p.seq_len = seq_len;
  p.block_table = block_table; p.max_pages = max_pages; p.page_size = page_size;
  p.num_pages = num_pages;
  // a sequence longer than its block table's pages is flagged and skipped
  const int64_t cap = (int64_t)max_pages * page_size;
  p.max_T = cap > 0x7fffffff ? 0x7fffffff : (int)cap;
  p.idx = idx; p.idx_k = idx_k; p.head_map = head_map; p.k_max = k_max;
  p.scale = scale; p.out = out; p.lse = lse; p.ws = ws;
  p.status = device_status_ptr();
  if (!p.status) return KASCADE_ERR_CUDA;
  return from_cuda(launch_decode_reuse(p, static_cast<cudaStream_t>(stream)));
}

int kascade_decode_reuse_paged(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                               const uint16_t* v_pages, int32_t num_pages,
                               const int32_t* block_table, int32_t max_pages, int32_t page_size,
                               const int32_t* seq_len, const int32_t* idx, const int32_t* idx_k,
                               int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                               float* lse, void* ws, size_t ws_bytes, void* stream) {
  return kascade_decode_reuse_paged_impl(s, q, k_pages, v_pages, num_pages, block_table, max_pages, page_size,
                                         seq_len, idx, idx_k, k_max, head_map, scale, out, lse, ws, ws_bytes,
                                         stream, false);
}

int kascade_decode_reuse_paged_f16(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                   const uint16_t* v_pages, int32_t num_pages,
                                   const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                   const int32_t* seq_len, const int32_t* idx, const int32_t* idx_k,
                                   int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                                   float* lse, void* ws, size_t ws_bytes, void* stream) {
  return kascade_decode_reuse_paged_impl(s, q, k_pages, v_pages, num_pages, block_table, max_pages, page_size,
                                         seq_len, idx, idx_k, k_max, head_map, scale, out, lse, ws, ws_bytes,
                                         stream, true);
}

// -------------------------------------------------------------------- topk --
size_t kascade_topk_workspace_bytes(int32_t rows, int64_t ld) {
  (void)rows;
  (void)ld;
  return 0;
}

int kascade_topk(const float* scores, int32_t rows, int64_t ld, const int32_t* row_len,
                 const int32_t* row_k, int32_t k_max, int32_t* idx_out, void* ws,
                 size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (rows < 0 || ld < 0 || k_max < 0) return KASCADE_ERR_INVALID_ARG;
  if (rows == 0) return KASCADE_OK;
  if (!scores || !row_len || !row_k || (k_max > 0 && !idx_out)) return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(scores) || (ld & 3) || ((uintptr_t)row_len & 3) || ((uintptr_t)row_k & 3) ||
      ((uintptr_t)idx_out & 3))
    return KASCADE_ERR_INVALID_ARG;
  unsigned* st = device_status_ptr();
  if (!st) return KASCADE_ERR_CUDA;
  return from_cuda(launch_topk(scores, rows, ld, row_len, row_k, k_max, idx_out, st,
                               static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------- calibration --
int kascade_similarity_rows(const float* p_b, int32_t rows, int64_t ld, const int32_t* row_len,
                            const int32_t* row_k, const int32_t* idx_a, const int32_t* idx_b,
                            int32_t k_max, int32_t n_out, const int32_t* b_row,
                            const int32_t* a_row, double* ratio, void* stream) {
  if (rows < 0 || ld < 0 || k_max < 0 || n_out < 0) return KASCADE_ERR_INVALID_ARG;
  if (n_out == 0) return KASCADE_OK;
  if (rows == 0 || !p_b || !row_len || !row_k || !ratio || (k_max > 0 && (!idx_a || !idx_b)))
    return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(p_b) || (ld & 3) || ((uintptr_t)row_len & 3) || ((uintptr_t)row_k & 3) ||
      ((uintptr_t)idx_a & 3) || ((uintptr_t)idx_b & 3) || ((uintptr_t)b_row & 3) ||
      ((uintptr_t)a_row & 3) || ((uintptr_t)ratio & 7))
    return KASCADE_ERR_INVALID_ARG;
  unsigned* st = device_status_ptr();
  if (!st) return KASCADE_ERR_CUDA;
  SimArgs a;
  a.p_b = p_b; a.rows = rows; a.ld = ld; a.row_len = row_len; a.row_k = row_k;
  a.idx_a = idx_a; a.idx_b = idx_b; a.k_max = k_max; a.b_row = b_row; a.a_row = a_row;
  a.ratio = ratio; a.status = st;
  return from_cuda(launch_similarity_rows(a, n_out, static_cast<cudaStream_t>(stream)));
}

// Checks shared by the aggregating calibration calls: rows of p_b / row_len /
// row_k / idx_a / idx_b as in kascade_similarity_rows.
static int check_sim_rows(const float* p_b, int32_t rows, int64_t ld, const int32_t* row_len,
                          const int32_t* row_k, const int32_t* idx_a, const int32_t* idx_b,
                          int32_t k_max) {
  if (rows <= 0 || ld < 0 || k_max < 0) return KASCADE_ERR_INVALID_ARG;
  if (!p_b || !row_len || !row_k || (k_max > 0 && (!idx_a || !idx_b))) return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(p_b) || (ld & 3) || ((uintptr_t)row_len & 3) || ((uintptr_t)row_k & 3) ||
      ((uintptr_t)idx_a & 3) || ((uintptr_t)idx_b & 3))
    return KASCADE_ERR_INVALID_ARG;
  return KASCADE_OK;
}

size_t kascade_similarity_mean_workspace_bytes(int32_t rows) {
  return rows > 0 ? align_up((size_t)rows * sizeof(double), 256) : 0;
}

int kascade_similarity_mean(const float* p_b, int32_t rows, int64_t ld, const int32_t* row_len,
                            const int32_t* row_k, const int32_t* idx_a, const int32_t* idx_b,
                            int32_t k_max, double* mean, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_sim_rows(p_b, rows, ld, row_len, row_k, idx_a, idx_b, k_max);
  if (rc) return rc;
  if (!mean || ((uintptr_t)mean & 7) || !ws || ((uintptr_t)ws & 7)) return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < kascade_similarity_mean_workspace_bytes(rows)) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  unsigned* st = device_status_ptr();
  if (!st) return KASCADE_ERR_CUDA;
  SimArgs a;
  a.p_b = p_b; a.rows = rows; a.ld = ld; a.row_len = row_len; a.row_k = row_k;
  a.idx_a = idx_a; a.idx_b = idx_b; a.k_max = k_max; a.b_row = nullptr; a.a_row = nullptr;
  a.ratio = nullptr; a.status = st;
  return from_cuda(launch_similarity_mean(a, static_cast<double*>(ws), mean, static_cast<cudaStream_t>(stream)));
}

size_t kascade_head_remap_workspace_bytes(int32_t Hkv, int32_t Q) {
  if (Hkv <= 0 || Hkv > 1024 || Q <= 0) return 0;
  const size_t pairs = (size_t)Hkv * Hkv;
  return align_up(pairs * Q * sizeof(double), 256) + align_up(pairs * sizeof(double), 256);
}

int kascade_head_remap(const float* p_reuse, int32_t Hkv, int32_t Q, int64_t ld, const int32_t* row_len,
                       const int32_t* row_k, const int32_t* idx_anchor, const int32_t* idx_reuse,
                       int32_t k_max, double* sim, int32_t* head_map, void* ws, size_t ws_bytes,
                       void* stream) {
  if (Hkv <= 0 || Hkv > 1024 || Q <= 0 || (int64_t)Hkv * Q > 0x7fffffff ||
      (int64_t)Hkv * Hkv * Q > 0x7fffffff)
    return KASCADE_ERR_INVALID_ARG;
  int rc = check_sim_rows(p_reuse, Hkv * Q, ld, row_len, row_k, idx_anchor, idx_reuse, k_max);
  if (rc) return rc;
  if (!head_map || ((uintptr_t)head_map & 3) || (sim && ((uintptr_t)sim & 7)) || !ws || ((uintptr_t)ws & 7))
    return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < kascade_head_remap_workspace_bytes(Hkv, Q)) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  unsigned* st = device_status_ptr();
  if (!st) return KASCADE_ERR_CUDA;
  const size_t pairs = (size_t)Hkv * Hkv;
  double* ratio = static_cast<double*>(ws);
  double* means = sim ? sim : reinterpret_cast<double*>(static_cast<char*>(ws) +
                                                        align_up(pairs * Q * sizeof(double), 256));
  SimArgs a;
  a.p_b = p_reuse; a.rows = Hkv * Q; a.ld = ld; a.row_len = row_len; a.row_k = row_k;
  a.idx_a = idx_anchor; a.idx_b = idx_reuse; a.k_max = k_max; a.b_row = nullptr; a.a_row = nullptr;
  a.ratio = nullptr; a.status = st;
  return from_cuda(launch_head_remap(a, Hkv, Q, ratio, means, head_map, static_cast<cudaStream_t>(stream)));
}

int kascade_select_anchors(const double* S, int32_t L, int32_t M, int32_t* anchors, double* best) {
  if (!S || !anchors || !best || L < 1 || L > 4096 || M < 1 || M > L) return KASCADE_ERR_INVALID_ARG;
  for (int64_t i = 0; i < (int64_t)L * L; ++i)
    if (!std::isfinite(S[i])) return KASCADE_ERR_NONFINITE;
  select_anchors_dp(S, L, M, anchors, best);
  return KASCADE_OK;
}

// ----------------------------------------------------------------- prefill --
static int check_prefill(const kascade_shape& s, int32_t N) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (N < 0) return KASCADE_ERR_INVALID_ARG;
  if (N % 128) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  return KASCADE_OK;
}

size_t kascade_prefill_anchor_workspace_bytes(kascade_shape s, int32_t N) {
  if (check_prefill(s, N) != KASCADE_OK) return 0;
  return prefill_anchor_workspace_bytes(s.B, s.Hq, s.Hkv, N);
}

static int kascade_prefill_anchor_impl(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, float scale, uint16_t* out, float* lse,
                           float* pooled, void* ws, size_t ws_bytes, void* stream, bool f16) {
  int rc = check_prefill(s, N);
  if (rc) return rc;
  if (!std::isfinite(scale) || !(scale > 0.f)) return KASCADE_ERR_INVALID_ARG;
  if (s.B == 0 || N == 0) return KASCADE_OK;
  const size_t need = kascade_prefill_anchor_workspace_bytes(s, N);
  if (!q || !k || !v || !out || !lse || !pooled || (need && !ws)) return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(pooled) || (ws && !aligned16(ws)))
    return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < need) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  PrefillParams p = {};
  p.f16 = f16;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv; p.N = N;
  p.q = q; p.k = k; p.v = v; p.scale = scale; p.out = out; p.lse = lse; p.pooled = pooled;
  p.ws = ws;
  p.status = device_status_ptr();
  if (!p.status) return KASCADE_ERR_CUDA;
  cudaError_t e = launch_prefill_anchor(p, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(e);
}

int kascade_prefill_anchor(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, float scale, uint16_t* out, float* lse,
                           float* pooled, void* ws, size_t ws_bytes, void* stream) {
  return kascade_prefill_anchor_impl(s, N, q, k, v, scale, out, lse, pooled, ws, ws_bytes, stream, false);
}

int kascade_prefill_anchor_f16(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, float scale, uint16_t* out, float* lse,
                           float* pooled, void* ws, size_t ws_bytes, void* stream) {
  return kascade_prefill_anchor_impl(s, N, q, k, v, scale, out, lse, pooled, ws, ws_bytes, stream, true);
}

size_t kascade_prefill_reuse_workspace_bytes(kascade_shape s, int32_t N, int32_t k_max) {
  if (check_prefill(s, N) != KASCADE_OK || k_max < 0) return 0;
  return prefill_reuse_workspace_bytes(s.B, s.Hq, s.Hkv, N, k_max);
}

static int kascade_prefill_reuse_impl(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* idx, const int32_t* idx_k,
                          int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                          float* lse, void* ws, size_t ws_bytes, void* stream, bool f16) {
  int rc = check_prefill(s, N);
  if (rc) return rc;
  if (k_max < 0 || !std::isfinite(scale) || !(scale > 0.f)) return KASCADE_ERR_INVALID_ARG;
  if (s.B == 0 || N == 0) return KASCADE_OK;
  const size_t need = kascade_prefill_reuse_workspace_bytes(s, N, k_max);
  if (!q || !k || !v || !idx || !idx_k || !head_map || !out || (need && !ws))
    return KASCADE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse && !aligned16(lse)) || (ws && !aligned16(ws)) || ((uintptr_t)idx & 3) ||
      ((uintptr_t)idx_k & 3) || ((uintptr_t)head_map & 3))
    return KASCADE_ERR_INVALID_ARG;
  if (ws_bytes < need) return KASCADE_ERR_WORKSPACE_TOO_SMALL;
  PrefillParams p = {};
  p.f16 = f16;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv; p.N = N;
  p.q = q; p.k = k; p.v = v; p.idx = idx; p.idx_k = idx_k; p.head_map = head_map;
  p.k_max = k_max; p.scale = scale; p.out = out; p.lse = lse; p.ws = ws;
  p.status = device_status_ptr();
  if (!p.status) return KASCADE_ERR_CUDA;
  cudaError_t e = launch_prefill_reuse(p, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KASCADE_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(e);
}

int kascade_prefill_reuse(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* idx, const int32_t* idx_k,
                          int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                          float* lse, void* ws, size_t ws_bytes, void* stream) {
  return kascade_prefill_reuse_impl(s, N, q, k, v, idx, idx_k, k_max, head_map, scale, out, lse, ws, ws_bytes, stream, false);
}

int kascade_prefill_reuse_f16(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* idx, const int32_t* idx_k,
                          int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                          float* lse, void* ws, size_t ws_bytes, void* stream) {
  return kascade_prefill_reuse_impl(s, N, q, k, v, idx, idx_k, k_max, head_map, scale, out, lse, ws, ws_bytes, stream, true);
}

}  // extern "C"
