// Internal launch interface between the C-ABI layer (api.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kascade.h"

namespace kascade {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- decode ----
struct DecodeParams {
  int B, Hq, Hkv, G;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int64_t* kv_off;        // contiguous cache (NULL when paged)
  const int32_t* block_table;   // paged cache [B, max_pages] (NULL when contiguous)
  int max_pages = 0, page_size = 0, num_pages = 0;
  bool f16 = false;             // q, k, v, out are fp16 (else bf16)
  const int32_t* seq_len;
  int max_T;
  // gather (reuse) only
  const int32_t* idx;
  const int32_t* idx_k;
  const int32_t* head_map;
  int k_max;
  float scale;
  uint16_t* out;
  float* lse;
  float* pooled;  // anchor only
  int64_t ld_pooled;
  void* ws;
  unsigned* status;
};

// Split geometry: each warp walks `tok_per_warp` items, 4 warps per CTA.
struct DecodeSplit {
  int tok_per_warp;
  int nsplit;  // CTAs per (b, h)
};
DecodeSplit decode_split_for(int units, int n_items, bool gather);
size_t decode_workspace_bytes(int B, int Hkv, int G, int n_items, bool with_logits);

cudaError_t launch_decode_anchor(const DecodeParams& p, cudaStream_t st);
// Host checks of kascade_decode_anchor other than the workspace (api.cu).
int decode_anchor_check_args(kascade_shape s, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const int64_t* kv_off, const int32_t* seq_len, int32_t max_T, float scale,
                             const uint16_t* out, const float* lse, const float* pooled, int64_t ld_pooled);
cudaError_t launch_decode_reuse(const DecodeParams& p, cudaStream_t st);

// ------------------------------------------------------------------ topk ----
size_t topk_smem_bytes(int64_t ld);
cudaError_t launch_topk(const float* scores, int rows, int64_t ld, const int32_t* row_len,
                        const int32_t* row_k, int k_max, int32_t* idx_out, unsigned* status,
                        cudaStream_t st);

// --------------------------------------------------------------- prefill ----
struct PrefillParams {
  int B, Hq, Hkv, G, N;
  bool f16 = false;  // q, k, v, out are fp16 (else bf16)
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  const int32_t* idx_k;
  const int32_t* head_map;
  int k_max;
  float scale;
  uint16_t* out;
  float* lse;
  float* pooled;
  void* ws;
  unsigned* status;
};
size_t prefill_anchor_workspace_bytes(int B, int Hq, int Hkv, int N);
size_t prefill_reuse_workspace_bytes(int B, int Hq, int Hkv, int N, int k_max);
cudaError_t launch_prefill_anchor(const PrefillParams& p, cudaStream_t st);
cudaError_t launch_prefill_reuse(const PrefillParams& p, cudaStream_t st);

// ----------------------------------------------------------- calibration ----
struct SimArgs {
  const float* p_b;
  int rows;
  int64_t ld;
  const int32_t* row_len;
  const int32_t* row_k;
  const int32_t* idx_a;
  const int32_t* idx_b;
  int k_max;
  const int32_t* b_row;
  const int32_t* a_row;
  double* ratio;
  unsigned* status;
  int remap_H = 0, remap_Q = 0;  // > 0: head-remap row arithmetic instead of b_row / a_row
};
cudaError_t launch_similarity_rows(const SimArgs& a, int n_out, cudaStream_t st);
// Ratios of a.rows rows into ratio_ws, then their mean into *mean (device).
cudaError_t launch_similarity_mean(const SimArgs& a, double* ratio_ws, double* mean, cudaStream_t st);
// Ratios of every (reuse head, anchor head, query) into ratio_ws [Hkv*Hkv*Q],
// their means over queries into sim [Hkv, Hkv], and the argmax into head_map.
cudaError_t launch_head_remap(const SimArgs& a, int Hkv, int Q, double* ratio_ws, double* sim,
                              int32_t* head_map, cudaStream_t st);

// One CTA whose first thread waits on an mbarrier nothing arrives at, through
// the prefill kernels' bounded wait (spin: the non-suspending variant); the
// wait gives up after about 2 s and ORs the timeout bit into *status.
cudaError_t launch_wait_timeout(bool spin, unsigned* status, cudaStream_t st);
void select_anchors_dp(const double* S, int L, int M, int32_t* anchors, double* best);

}  // namespace kascade
