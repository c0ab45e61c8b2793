/*
 * kascade.h -- C ABI of the Kascade attention hot path on NVIDIA B200 (sm_100a).
 *
 * Kascade (arXiv 2512.16391) splits a model's layers into anchor layers, which
 * run dense attention and take the Top-k keys of the post-softmax
 * distribution, and reuse layers, which attend only to the keys an anchor
 * chose, per key head through a head-remap table.
 * Sources, cited by page and section:
 *   [explainer] "論文解説: Kascade — レイヤー間スパーシティ再利用による実用的長文脈LLM推論高速化"
 *               (0h-n0.github.io), sections under 技術的詳細 and 実装のポイント;
 *   [abstract]  the arXiv abstract (fugumt.com listing of 2512.16391v1).
 *
 * General rules (every entry point):
 *   - Every pointer argument is a DEVICE pointer owned by the caller (the host-side
 *     calibration DP kascade_select_anchors excepted); the library never allocates,
 *     frees or keeps a pointer after the call returns.  Scratch memory is passed in
 *     as `ws` of `ws_bytes` (query the size first).  The one exception is
 *     kascade_decode_anchor_static_ws, whose scratch is a fixed array owned by the
 *     library (see its comment block).
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   - Every base pointer must be 16-byte aligned; every row stride named below is
 *     in elements and must keep rows 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued
 *     asynchronously; the return value reports only what the host can check before
 *     launching (arguments, shapes, workspace size, launch errors).
 *   - Errors found by the kernels themselves (an index, head-map entry or length
 *     out of range, a NaN score) never fault: the offending element is skipped, and
 *     a sticky per-device status word is set; read it with kascade_get_device_status.
 *   - Supported shapes: head_dim d == 128, Hq % Hkv == 0, group size Hq/Hkv in {1,2,4,8},
 *     prefill query tile fixed at 128 tokens, prefill length a multiple of 128, decode
 *     max_T and k_max at most 2^30 (KASCADE_ERR_UNSUPPORTED_SHAPE otherwise).
 *   - `scale` must be finite; the prefill calls also require scale > 0.
 *   - Returned status codes are the kascade_status values below; no C++ exception
 *     crosses this boundary.
 */
#ifndef KASCADE_H_
#define KASCADE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KASCADE_OK = 0,
  KASCADE_ERR_INVALID_ARG = 1,        /* NULL/misaligned pointer, negative size, k > length ... */
  KASCADE_ERR_UNSUPPORTED_SHAPE = 2,  /* d != 128, group > 8, prefill N not a multiple of 128,
                                         decode anchor with B·Hq·max_T > 2^46 */
  KASCADE_ERR_WORKSPACE_TOO_SMALL = 3,
  KASCADE_ERR_CUDA = 4,               /* a launch or CUDA runtime call failed */
  KASCADE_ERR_BAD_INDEX = 5,          /* device side: index / head map / length out of range */
  KASCADE_ERR_NONFINITE = 6,          /* device side: NaN in a Top-k score row */
  KASCADE_ERR_TIMEOUT = 7             /* device side: a bounded wait inside a kernel gave up */
} kascade_status;

/* Attention shape shared by all calls.  B = batch, Hq = query heads,
 * Hkv = key/value heads (GQA group G = Hq / Hkv), d = head dim (128). */
typedef struct {
  int32_t B, Hq, Hkv, d;
} kascade_shape;

/* ------------------------------------------------------------------------- */
/* Top-k size rule.  [explainer] 技術的詳細 › Top-k設定, k equation:
 * k = min(max(0.1·n, 128), n) with 0.1·n rounded half up, i.e.
 * min(max((n + 5) / 10, 128), n) in integer arithmetic.  n < 0 returns 0. */
int32_t kascade_k_for_len(int32_t n);

/* ------------------------------------------------------------------------- */
/* Decode anchor layer.  [explainer] 技術的詳細 › アンカーレイヤーと再利用レイヤー (full attention
 * in anchor layers, Top-k from the post-softmax distribution) and › ヘッドリマッピング (one
 * index set per key head under GQA).
 *
 * For sequence b, KV head h and each query head g of group h (g in [G·h, G·h+G)):
 *   s_{g,t} = scale · q[b,g,:] · K[b,h,t,:]       for t < T_b = seq_len[b]
 *   out[b,g,:] = sum_t softmax_t(s_g)_t · V[b,h,t,:]
 *   lse[b,g]   = log sum_t exp(s_{g,t})           (natural log)
 *   pooled[b,h,t] = (1/G) · sum_g exp(s_{g,t} - lse[b,g])   (mean post-softmax probability)
 *
 *   q       bf16 [B, Hq, d]
 *   k, v    bf16 caches; sequence b is a contiguous [Hkv, T_b, d] block starting at
 *           element kv_off[b] of k (and of v)
 *   kv_off  int64 [B] element offsets (multiples of 8); seq_len int32 [B], 0 <= T_b <= max_T
 *   max_T   host-side upper bound of seq_len (sizes the grid and the workspace)
 *   out     bf16 [B, Hq, d]; lse fp32 [B, Hq] (may be NULL)
 *   pooled  fp32 [B, Hkv, ld_pooled], ld_pooled >= max_T, ld_pooled % 4 == 0; entries at
 *           t >= T_b are left untouched
 *   ws      scratch of at least kascade_decode_anchor_workspace_bytes(s, max_T) bytes
 * A sequence with T_b == 0 gets out = 0 and lse = -inf.  Shapes with B·Hq·max_T > 2^46 are
 * refused (KASCADE_ERR_UNSUPPORTED_SHAPE; the workspace query returns 0), so that no
 * workspace size can wrap around. */
size_t kascade_decode_anchor_workspace_bytes(kascade_shape s, int32_t max_T);
int kascade_decode_anchor(kascade_shape s, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                          int32_t max_T, float scale, uint16_t* out, float* lse,
                          float* pooled, int64_t ld_pooled, void* ws, size_t ws_bytes,
                          void* stream);

/* Size of the library-owned scratch array used by kascade_decode_anchor_static_ws. */
#define KASCADE_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* Decode anchor without caller-provided scratch.  The method has no counterpart of
 * this entry point; it exists for callers that cannot allocate device memory at
 * the point where they run the layer: an inference-runtime plugin whose enqueue
 * step may not allocate, or a serving engine that has handed nearly all device
 * memory to its KV-cache pool up front (and cudaMalloc / cudaFree would also
 * synchronise the device in the middle of a step).
 *
 * Same arguments, results and checks as kascade_decode_anchor, minus ws/ws_bytes; the
 * argument checks run first, in the same order, so a bad argument returns the same
 * code as from kascade_decode_anchor; the scratch-size limit below is checked after them.
 * The scratch is a file-scope device array of KASCADE_STATIC_SCRATCH_BYTES that
 * every GPU which loads the library holds until the process exits.  The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - Problems whose scratch, kascade_decode_anchor_workspace_bytes(s, max_T), is
 *     larger than KASCADE_STATIC_SCRATCH_BYTES are refused with
 *     KASCADE_ERR_WORKSPACE_TOO_SMALL before anything is launched.  With 32 query
 *     heads, 16 sequences of 4K tokens or one of 64K fit; one of 128K does not.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (this may load the library's kernels on that device);
 *     make that first call before any stream capture.
 *   - Every call, from any stream or thread, shares the one array per device, and
 *     the array keeps the previous call's contents.  Calls whose kernels overlap on
 *     the GPU race on it and corrupt each other's results: order them (one stream,
 *     or events).  No part of the array needs to start at zero, because each call
 *     writes every scratch element it later reads. */
int kascade_decode_anchor_static_ws(kascade_shape s, const uint16_t* q, const uint16_t* k,
                                    const uint16_t* v, const int64_t* kv_off,
                                    const int32_t* seq_len, int32_t max_T, float scale,
                                    uint16_t* out, float* lse, float* pooled,
                                    int64_t ld_pooled, void* stream);

/* ------------------------------------------------------------------------- */
/* Row-wise Top-k select.  [explainer] 技術的詳細 › アンカーレイヤーと再利用レイヤー (exact Top-k
 * indices in anchor layers) and › Top-k設定 (k).  Ties are broken toward the lower index;
 * -0.0 equals +0.0; the selected indices are written in ascending order.
 *
 *   scores   fp32 [rows, ld]; row r uses its first row_len[r] entries
 *   row_len  int32 [rows], 0 <= row_len[r] <= ld
 *   row_k    int32 [rows], 0 <= row_k[r] <= min(row_len[r], k_max)
 *   idx_out  int32 [rows, k_max]; entries past row_k[r] are set to -1
 *   ws       scratch of kascade_topk_workspace_bytes(rows, ld) bytes (may be 0 / NULL)
 * A NaN in a row sets KASCADE_ERR_NONFINITE on the device (that row's output is
 * unspecified); a bad row_len / row_k sets KASCADE_ERR_BAD_INDEX and writes -1s. */
size_t kascade_topk_workspace_bytes(int32_t rows, int64_t ld);
int kascade_topk(const float* scores, int32_t rows, int64_t ld, const int32_t* row_len,
                 const int32_t* row_k, int32_t k_max, int32_t* idx_out, void* ws,
                 size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Decode reuse layer.  [explainer] アンカーレイヤーと再利用レイヤー (reuse layers attend only to
 * the keys the preceding anchor selected) and ヘッドリマッピング (reuse key head h takes the
 * indices of anchor key head head_map[h]).  The softmax is renormalised over the set.
 *
 * For sequence b, reuse KV head h, a = head_map[h], J = idx[b, a, 0 : idx_k[b·Hkv + a]]:
 *   out[b,g,:] = sum_{j in J} softmax_J(scale · q[b,g,:]·K[b,h,j,:])_j · V[b,h,j,:]
 *
 *   q, k, v, kv_off, seq_len   as in kascade_decode_anchor
 *   idx      int32 [B, Hkv, k_max]   anchor indices, each in [0, T_b)
 *   idx_k    int32 [B·Hkv]           valid count per anchor row, <= k_max
 *   head_map int32 [Hkv]             values in [0, Hkv)
 *   out bf16 [B, Hq, d]; lse fp32 [B, Hq] (may be NULL)
 *   ws       scratch of kascade_decode_reuse_workspace_bytes(s, k_max) bytes (currently 0:
 *            the splits of a row merge on chip; NULL is accepted when the size is 0)
 * Out-of-range indices are skipped (status KASCADE_ERR_BAD_INDEX). */
size_t kascade_decode_reuse_workspace_bytes(kascade_shape s, int32_t k_max);
int kascade_decode_reuse(kascade_shape s, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                         const int32_t* idx, const int32_t* idx_k, int32_t k_max,
                         const int32_t* head_map, float scale, uint16_t* out, float* lse,
                         void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Prefill anchor layer.  [explainer] 主要な貢献 (tile-level post-softmax pooling in
 * prefill), 実装のポイント (128-query tiles in prefill), アンカーレイヤーと再利用レイヤー.
 *
 * Causal attention over N tokens: query i sees keys j <= i.  For query tile t
 * (queries [128t, 128t+128)) and KV head h:
 *   pooled[b,t,h,j] = 1/(128·G) · sum_{i in tile t} sum_{g in group h}
 *                      exp(s_{g,i,j} - lse[b,g,i])          for j < 128t
 *
 *   q bf16 [B, Hq, N, d]; k, v bf16 [B, Hkv, N, d]
 *   out bf16 [B, Hq, N, d]; lse fp32 [B, Hq, N] (required: it is the pooling normaliser)
 *   pooled fp32 [B, N/128, Hkv, N]; entries at j >= 128t are left untouched
 *   ws scratch of kascade_prefill_anchor_workspace_bytes(s, N) bytes */
size_t kascade_prefill_anchor_workspace_bytes(kascade_shape s, int32_t N);
int kascade_prefill_anchor(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, float scale, uint16_t* out, float* lse,
                           float* pooled, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Prefill reuse layer.  [explainer] アンカーレイヤーと再利用レイヤー, ヘッドリマッピング,
 * 実装のポイント (128-query tiles).  Query i of tile t in reuse KV head h attends to
 *   J_t = idx[b, t, head_map[h], 0 : idx_k[(b·n_tiles + t)·Hkv + head_map[h]]]   (all < 128t)
 * together with its own diagonal block, causally (keys 128t <= j <= i); softmax over
 * that set.
 *
 *   q, k, v as in kascade_prefill_anchor
 *   idx int32 [B, N/128, Hkv, k_max]; idx_k int32 [B·(N/128)·Hkv]; head_map int32 [Hkv]
 *   out bf16 [B, Hq, N, d]; lse fp32 [B, Hq, N] (may be NULL)
 *   ws scratch of kascade_prefill_reuse_workspace_bytes(s, N, k_max) bytes
 *
 * Device-side errors (KASCADE_ERR_BAD_INDEX in the status word): an index
 * outside [0, 128t) is skipped; a head_map entry outside [0, Hkv), or an idx_k
 * entry outside [0, min(k_max, 128t)], drops that row's whole index set, and
 * its queries attend to their diagonal block alone. */
size_t kascade_prefill_reuse_workspace_bytes(kascade_shape s, int32_t N, int32_t k_max);
int kascade_prefill_reuse(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* idx, const int32_t* idx_k,
                          int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                          float* lse, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* fp16 variants (the evaluation's precision): the same contracts as the four
 * calls above, with q, k, v and out holding IEEE half-precision values (the
 * same uint16_t bit containers) instead of bfloat16.  Accumulation, softmax,
 * LSE and pooled probabilities stay fp32; workspace sizes are those of the
 * bfloat16 calls. */
int kascade_decode_anchor_f16(kascade_shape s, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                              int32_t max_T, float scale, uint16_t* out, float* lse, float* pooled,
                              int64_t ld_pooled, void* ws, size_t ws_bytes, void* stream);
int kascade_decode_reuse_f16(kascade_shape s, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, const int64_t* kv_off, const int32_t* seq_len,
                             const int32_t* idx, const int32_t* idx_k, int32_t k_max,
                             const int32_t* head_map, float scale, uint16_t* out, float* lse,
                             void* ws, size_t ws_bytes, void* stream);
int kascade_prefill_anchor_f16(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, float scale, uint16_t* out, float* lse,
                               float* pooled, void* ws, size_t ws_bytes, void* stream);
int kascade_prefill_reuse_f16(kascade_shape s, int32_t N, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const int32_t* idx, const int32_t* idx_k,
                              int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                              float* lse, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Paged KV cache variants of the two decode calls (the explainer's serving
 * integration keeps the cache in fixed-size pages).  Same operation, outputs
 * and workspace (kascade_decode_{anchor,reuse}_workspace_bytes) as the
 * contiguous calls; only where a token's K/V row lives differs:
 *   k_pages, v_pages  device bf16 [num_pages, Hkv, page_size, 128], 16-byte aligned
 *   block_table       device int32 [B, max_pages]: page j of sequence b holds its
 *                     tokens j*page_size .. j*page_size + page_size - 1
 *   page_size         multiple of 16 (>= 16)
 * Host checks as for the contiguous calls, plus: num_pages >= 1, max_pages >= 1,
 * and (anchor) max_pages * page_size >= max_T.  A block-table entry outside
 * [0, num_pages) skips the tokens it holds and sets KASCADE_ERR_BAD_INDEX in the
 * device status; a sequence longer than max_pages * page_size is skipped the same
 * way.  Results are bit-identical to the contiguous calls on the same data.
 * The _f16 variants take fp16 q, k_pages, v_pages and out (same containers),
 * like the contiguous _f16 calls. */
int kascade_decode_anchor_paged(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                const uint16_t* v_pages, int32_t num_pages,
                                const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                const int32_t* seq_len, int32_t max_T, float scale, uint16_t* out,
                                float* lse, float* pooled, int64_t ld_pooled, void* ws,
                                size_t ws_bytes, void* stream);
int kascade_decode_reuse_paged(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                               const uint16_t* v_pages, int32_t num_pages,
                               const int32_t* block_table, int32_t max_pages, int32_t page_size,
                               const int32_t* seq_len, const int32_t* idx, const int32_t* idx_k,
                               int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                               float* lse, void* ws, size_t ws_bytes, void* stream);
int kascade_decode_anchor_paged_f16(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                    const uint16_t* v_pages, int32_t num_pages,
                                    const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                    const int32_t* seq_len, int32_t max_T, float scale, uint16_t* out,
                                    float* lse, float* pooled, int64_t ld_pooled, void* ws,
                                    size_t ws_bytes, void* stream);
int kascade_decode_reuse_paged_f16(kascade_shape s, const uint16_t* q, const uint16_t* k_pages,
                                   const uint16_t* v_pages, int32_t num_pages,
                                   const int32_t* block_table, int32_t max_pages, int32_t page_size,
                                   const int32_t* seq_len, const int32_t* idx, const int32_t* idx_k,
                                   int32_t k_max, const int32_t* head_map, float scale, uint16_t* out,
                                   float* lse, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Calibration (Kascade explainer, レイヤー間類似度とアンカーレイヤー選択 and
 * 動的計画法): which layers are anchors and which anchor KV head each reuse
 * head follows are chosen offline from post-softmax distributions.
 *
 * kascade_similarity_rows: the sim ratio of the explainer per row, the share of
 * layer b's Top-k probability mass that layer a's Top-k indices recover.  For
 * output row r, with rb = b_row[r] (r if b_row is NULL) and ra = a_row[r]
 * (r if a_row is NULL) and k = row_k[rb]:
 *     ratio[r] = sum_{i<k} p_b[rb][idx_a[ra][i]] / sum_{i<k} p_b[rb][idx_b[rb][i]]
 * (fp64 sums; 0 when the denominator is 0).  The row maps let one call compare
 * every (anchor head, reuse head) pair without copying rows.
 *   p_b       device fp32 [rows, ld], 16-byte aligned, ld % 4 == 0: layer b's rows
 *   row_len   device int32 [rows]: valid length of each row (<= ld)
 *   row_k     device int32 [rows]: k of each row (<= row_len, <= k_max)
 *   idx_a     device int32 [rows, k_max]: layer a's Top-k indices (kascade_topk output)
 *   idx_b     device int32 [rows, k_max]: layer b's Top-k indices
 *   b_row, a_row  device int32 [n_out] or NULL: source rows of each output row
 *   ratio     device fp64 [n_out]: output
 * Indices or rows out of range are skipped and set KASCADE_ERR_BAD_INDEX in the
 * device status.  Asynchronous on `stream`. */
int kascade_similarity_rows(const float* p_b, int32_t rows, int64_t ld, const int32_t* row_len,
                            const int32_t* row_k, const int32_t* idx_a, const int32_t* idx_b,
                            int32_t k_max, int32_t n_out, const int32_t* b_row,
                            const int32_t* a_row, double* ratio, void* stream);

/* kascade_similarity_mean: sim(a, b) of two layers, the mean over the rows of the
 * ratios kascade_similarity_rows defines (with identity row maps), summed in fp64
 * in a fixed order.  The pages do not say how per-query ratios combine; the mean
 * over queries (or pooled rows) is taken.
 *   p_b, row_len, row_k, idx_a, idx_b, k_max  as in kascade_similarity_rows
 *   mean      device fp64 [1]: output
 *   ws        device scratch of kascade_similarity_mean_workspace_bytes(rows) bytes
 * Errors as for kascade_similarity_rows; rows must be >= 1. */
size_t kascade_similarity_mean_workspace_bytes(int32_t rows);
int kascade_similarity_mean(const float* p_b, int32_t rows, int64_t ld, const int32_t* row_len,
                            const int32_t* row_k, const int32_t* idx_a, const int32_t* idx_b,
                            int32_t k_max, double* mean, void* ws, size_t ws_bytes, void* stream);

/* kascade_head_remap: [explainer] ヘッドリマッピング.  For each key head h of a
 * reuse layer, the anchor-layer key head whose Top-k indices recover the most of
 * h's Top-k probability mass:
 *     sim[h][a]   = mean over q < Q of ratio(p_reuse row h·Q+q; idx_anchor row a·Q+q,
 *                                            idx_reuse row h·Q+q)
 *     head_map[h] = argmax_a sim[h][a], the lowest a among equal maxima
 * with ratio as in kascade_similarity_rows (a = anchor head, b = reuse head).
 *   p_reuse     device fp32 [Hkv·Q, ld]: the reuse layer's distributions, row h·Q+q
 *   row_len, row_k  device int32 [Hkv·Q]
 *   idx_anchor  device int32 [Hkv·Q, k_max]: the anchor layer's Top-k rows
 *   idx_reuse   device int32 [Hkv·Q, k_max]: the reuse layer's Top-k rows
 *   sim         device fp64 [Hkv, Hkv]: output, or NULL
 *   head_map    device int32 [Hkv]: output, values in [0, Hkv)
 *   ws          device scratch of kascade_head_remap_workspace_bytes(Hkv, Q) bytes
 * Returns KASCADE_ERR_INVALID_ARG unless 1 <= Hkv <= 1024, Q >= 1 and Hkv·Hkv·Q < 2^31;
 * other errors as for kascade_similarity_rows.  Asynchronous on `stream`. */
size_t kascade_head_remap_workspace_bytes(int32_t Hkv, int32_t Q);
int kascade_head_remap(const float* p_reuse, int32_t Hkv, int32_t Q, int64_t ld, const int32_t* row_len,
                       const int32_t* row_k, const int32_t* idx_anchor, const int32_t* idx_reuse,
                       int32_t k_max, double* sim, int32_t* head_map, void* ws, size_t ws_bytes,
                       void* stream);

/* kascade_select_anchors: Algorithm 1 of the explainer on the HOST (no GPU
 * work).  S is host fp64 [L, L] row-major, the weighted similarity matrix
 * (S[i][l] = w_l * sim(i, l) for l >= i).  Chooses M anchor layers maximising
 * sum_l S[a(l)][l], a(l) the last anchor at or before l, by
 *     dp[m][j] = max_{i=m-1..j-1} dp[m-1][i] + sum_{l=i}^{j-1} S[i][l]
 * with dp[0][0] = 0, dp[0][j>0] = -inf (so layer 0 is always an anchor), the
 * smallest i kept among equal maxima; O(M L^2) time, O(M L + L^2) memory.
 *   anchors   host int32 [M]: output, ascending
 *   best      host fp64: output, dp[M][L]
 * Returns KASCADE_ERR_INVALID_ARG unless 1 <= M <= L <= 4096 and the pointers
 * are non-NULL; KASCADE_ERR_NONFINITE if S holds a NaN or an infinity. */
int kascade_select_anchors(const double* S, int32_t L, int32_t M, int32_t* anchors, double* best);

/* ------------------------------------------------------------------------- */
/* Waits for `stream`, then returns and clears the sticky device status of the
 * current device.  The result is KASCADE_OK or one recorded code, chosen in this
 * order: KASCADE_ERR_TIMEOUT, then KASCADE_ERR_BAD_INDEX, then
 * KASCADE_ERR_NONFINITE.  It is KASCADE_ERR_CUDA if the wait fails.
 * KASCADE_ERR_TIMEOUT means that a prefill kernel's bounded wait gave up after
 * about 2 s; that call's outputs are incomplete, and the context stays usable. */
int kascade_get_device_status(void* stream);

/* Diagnostic for the failure path above.  Launches one CTA on `stream`.  Its
 * first thread waits on an mbarrier that nothing ever arrives at, through the
 * same bounded wait the prefill kernels use:
 *   spin == 0  suspending try_wait polls (the softmax and summing warps' wait)
 *   spin != 0  non-suspending test_wait polls (the MMA thread's wait)
 * The wait gives up after about 2 s and records the timeout bit, so the next
 * kascade_get_device_status returns KASCADE_ERR_TIMEOUT.  Returns
 * KASCADE_ERR_CUDA if the launch fails.  No memory is read or written apart from
 * the status word. */
int kascade_selftest_wait_timeout(int32_t spin, void* stream);

/* Human-readable name of a status code (static string). */
const char* kascade_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KASCADE_H_ */
