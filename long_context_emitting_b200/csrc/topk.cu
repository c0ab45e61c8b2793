// Row-wise exact Top-k select (ties toward the lower index, output ascending).
//
// Method: Kascade explainer (0h-n0.github.io), 技術的詳細 › アンカーレイヤーと再利用レイヤー
// (exact Top-k of the post-softmax distribution in anchor layers, one set per
// key head per ヘッドリマッピング) with k from › Top-k設定.
//
// Rows longer than the shared-memory cache run on topk_cluster_kernel: one
// thread-block cluster of C CTAs per row (C a power of two up to 16), each CTA
// caching one slice of the row.  Every radix pass sums the CTAs' histograms
// through distributed shared memory (each CTA computes the same selection), and
// the compaction takes each CTA's output offsets from the counts of the
// lower-ranked CTAs, so the result is the single-CTA kernel's, bit for bit.
//
// One CTA of 1024 threads per row.  Scores are mapped to order-preserving
// unsigned keys (-0.0 folded onto +0.0), cached in shared memory when the row
// fits (otherwise re-read from global memory / L2 on every pass), and an
// 11/11/10-bit radix select finds the exact k-th largest key tau and how many
// keys equal to tau are still needed.  A warp-ordered compaction then writes,
// in index order, every key > tau plus the first `need` keys == tau, which
// yields ascending indices with the lower-index tie-break.
#include "common.cuh"
#include "internal.h"

#include <cooperative_groups.h>

namespace kascade {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarpsPerRow = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kCacheMaxKeys = 49152;  // 192 KB of cached keys per row

__device__ __forceinline__ uint32_t order_key(uint32_t f) {
  if (f == 0x80000000u) f = 0u;  // -0.0 -> +0.0
  return (f & 0x80000000u) ? ~f : (f | 0x80000000u);
}

__device__ __forceinline__ bool is_nan_bits(uint32_t f) { return (f & 0x7fffffffu) > 0x7f800000u; }

struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* row_len;
  const int32_t* row_k;
  int k_max;
  int32_t* idx_out;
  int cache_cap;
  unsigned* status;
};

// Inclusive scan of one value per thread over the whole block (thread order).
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;  // inclusive totals
  }
  __syncthreads();
  const uint32_t before = warp ? warp_tot[warp - 1] : 0u;
  __syncthreads();
  return v + before;
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const TopkArgs a) {
  extern __shared__ uint32_t smem[];
  uint32_t* hist = smem;                 // kBins
  uint32_t* scratch = smem + kBins;      // 64 words
  uint32_t* keys = smem + kBins + 64;    // cache_cap
  __shared__ int s_sel_bin, s_sel_above;
  __shared__ uint32_t s_wgt[kWarpsPerRow], s_weq[kWarpsPerRow];

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int len = a.row_len[row];
  const int k = a.row_k[row];
  int32_t* out = a.idx_out + (int64_t)row * a.k_max;
  const float* src = a.scores + (int64_t)row * a.ld;

  if (len < 0 || (int64_t)len > a.ld || k < 0 || k > len || k > a.k_max) {
    if (tid == 0) flag_status(a.status, kStatusBadIndex);
    for (int i = tid; i < a.k_max; i += kThreads) out[i] = -1;
    return;
  }
  for (int i = k + tid; i < a.k_max; i += kThreads) out[i] = -1;

  const bool cached = len <= a.cache_cap;
  __syncthreads();

  // load (and cache) the row; detect NaN
  {
    int nan_seen = 0;
    const uint32_t* bits = reinterpret_cast<const uint32_t*>(src);
    const int n4 = len >> 2;
    for (int i = tid; i < n4; i += kThreads) {
      const uint4 w = *reinterpret_cast<const uint4*>(bits + 4 * i);
      nan_seen |= is_nan_bits(w.x) | is_nan_bits(w.y) | is_nan_bits(w.z) | is_nan_bits(w.w);
      if (cached) {
        keys[4 * i + 0] = order_key(w.x);
        keys[4 * i + 1] = order_key(w.y);
        keys[4 * i + 2] = order_key(w.z);
        keys[4 * i + 3] = order_key(w.w);
      }
    }
    for (int i = 4 * n4 + tid; i < len; i += kThreads) {
      const uint32_t f = bits[i];
      nan_seen |= is_nan_bits(f);
      if (cached) keys[i] = order_key(f);
    }
    if (__syncthreads_or(nan_seen) && tid == 0) flag_status(a.status, kStatusNonFinite);
  }
  if (k == 0) return;
  if (k == len) {
    for (int i = tid; i < len; i += kThreads) out[i] = i;
    return;
  }

  const uint32_t* gbits = reinterpret_cast<const uint32_t*>(src);
  auto key_at = [&](int i) -> uint32_t { return cached ? keys[i] : order_key(__ldg(gbits + i)); };

  // ---- radix select: 11 / 11 / 10 bits, most significant first -------------
  uint32_t prefix = 0u, pmask = 0u;
  int k_rem = k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass < 2 ? 0x7ffu : 0x3ffu;
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < len; i += kThreads) {
      const uint32_t key = key_at(i);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // thread t owns bins hi = 2047-2t and lo = 2046-2t (descending bin order)
    const uint32_t c_hi = hist[kBins - 1 - 2 * tid];
    const uint32_t c_lo = hist[kBins - 2 - 2 * tid];
    const uint32_t incl = block_inclusive_scan(c_hi + c_lo, scratch);
    const uint32_t excl = incl - c_hi - c_lo;
    const uint32_t kr = (uint32_t)k_rem;
    if (excl < kr && kr <= excl + c_hi) {
      s_sel_bin = kBins - 1 - 2 * tid;
      s_sel_above = (int)excl;
    } else if (excl + c_hi < kr && kr <= incl) {
      s_sel_bin = kBins - 2 - 2 * tid;
      s_sel_above = (int)(excl + c_hi);
    }
    __syncthreads();
    k_rem -= s_sel_above;
    prefix |= (uint32_t)s_sel_bin << shift;
    pmask |= dmask << shift;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need_eq = k_rem;  // keys equal to tau still to take (>= 1)

  // ---- ordered compaction --------------------------------------------------
  const int lane = tid & 31, warp = tid >> 5;
  const int seg = (((len + kWarpsPerRow - 1) / kWarpsPerRow) + 31) & ~31;
  const int s_lo = min(warp * seg, len), s_hi = min(s_lo + seg, len);
  uint32_t n_gt = 0, n_eq = 0;
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s_hi ? key_at(i) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, i < s_hi && key > tau));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < s_hi && key == tau));
  }
  if (lane == 0) {
    s_wgt[warp] = n_gt;
    s_weq[warp] = n_eq;
  }
  __syncthreads();
  uint32_t gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += s_wgt[w];
    eq_before += s_weq[w];
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s_hi ? key_at(i) : 0u;
    const bool is_gt = i < s_hi && key > tau;
    const bool is_eq = i < s_hi && key == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt);
    const uint32_t me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t my_gt = gt_before + __popc(mg & lt_mask);
    const uint32_t my_eq = eq_before + __popc(me & lt_mask);
    if (is_gt || (is_eq && my_eq < (uint32_t)need_eq)) {
      const uint32_t pos = my_gt + min(my_eq, (uint32_t)need_eq);
      out[pos] = i;
    }
    gt_before += __popc(mg);
    eq_before += __popc(me);
  }
}

// ---------------------------------------------------------------------------
// Long rows: one cluster of C CTAs per row.  All control flow that reaches a
// cluster barrier depends only on the row (its length, k, status), which every
// CTA of the cluster reads alike, so the CTAs always meet at every barrier.
__global__ void __launch_bounds__(kThreads, 1) topk_cluster_kernel(const TopkArgs a, int C, int seg) {
  namespace cg = cooperative_groups;
  extern __shared__ uint32_t smem[];
  uint32_t* hist = smem;                 // kBins (this CTA's slice)
  uint32_t* scratch = smem + kBins;      // 64 words
  uint32_t* keys = smem + kBins + 64;    // seg keys
  __shared__ int s_sel_bin, s_sel_above;
  __shared__ uint32_t s_wgt[kWarpsPerRow], s_weq[kWarpsPerRow];
  __shared__ uint32_t s_cta_gt, s_cta_eq;

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x;
  const int len = a.row_len[row];
  const int k = a.row_k[row];
  int32_t* out = a.idx_out + (int64_t)row * a.k_max;
  const float* src = a.scores + (int64_t)row * a.ld;

  if (len < 0 || (int64_t)len > a.ld || k < 0 || k > len || k > a.k_max) {
    if (rank == 0) {
      if (tid == 0) flag_status(a.status, kStatusBadIndex);
      for (int i = tid; i < a.k_max; i += kThreads) out[i] = -1;
    }
    return;  // every CTA of the cluster takes this branch
  }
  if (rank == 0)
    for (int i = k + tid; i < a.k_max; i += kThreads) out[i] = -1;

  // this CTA's slice [lo, hi) of the row, cached as order-preserving keys
  const int lo = min(rank * seg, len), hi = min(lo + seg, len);
  const int n = hi - lo;
  {
    int nan_seen = 0;
    const uint32_t* bits = reinterpret_cast<const uint32_t*>(src) + lo;
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t f = __ldg(bits + i);
      nan_seen |= is_nan_bits(f);
      keys[i] = order_key(f);
    }
    if (__syncthreads_or(nan_seen) && tid == 0) flag_status(a.status, kStatusNonFinite);
  }
  if (k == 0) return;
  if (k == len) {
    for (int i = tid; i < n; i += kThreads) out[lo + i] = lo + i;
    return;
  }

  // ---- radix select over the whole row: 11 / 11 / 10 bits --------------------
  uint32_t prefix = 0u, pmask = 0u;
  int k_rem = k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass < 2 ? 0x7ffu : 0x3ffu;
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    cluster.sync();  // every CTA's histogram is complete
    // thread t owns bins hi = 2047-2t and lo = 2046-2t, summed over the cluster
    uint32_t c_hi = 0u, c_lo = 0u;
    for (int r = 0; r < C; ++r) {
      const uint32_t* h = cluster.map_shared_rank(hist, r);
      c_hi += h[kBins - 1 - 2 * tid];
      c_lo += h[kBins - 2 - 2 * tid];
    }
    const uint32_t incl = block_inclusive_scan(c_hi + c_lo, scratch);
    const uint32_t excl = incl - c_hi - c_lo;
    const uint32_t kr = (uint32_t)k_rem;
    if (excl < kr && kr <= excl + c_hi) {
      s_sel_bin = kBins - 1 - 2 * tid;
      s_sel_above = (int)excl;
    } else if (excl + c_hi < kr && kr <= incl) {
      s_sel_bin = kBins - 2 - 2 * tid;
      s_sel_above = (int)(excl + c_hi);
    }
    cluster.sync();  // every CTA has read every histogram before the next pass clears its own
    k_rem -= s_sel_above;
    prefix |= (uint32_t)s_sel_bin << shift;
    pmask |= dmask << shift;
  }
  const uint32_t tau = prefix;
  const int need_eq = k_rem;

  // ---- ordered compaction across the cluster ---------------------------------
  const int lane = tid & 31, warp = tid >> 5;
  const int wseg = (((n + kWarpsPerRow - 1) / kWarpsPerRow) + 31) & ~31;
  const int s_lo = min(warp * wseg, n), s_hi = min(s_lo + wseg, n);
  uint32_t n_gt = 0, n_eq = 0;
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s_hi ? keys[i] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, i < s_hi && key > tau));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < s_hi && key == tau));
  }
  if (lane == 0) {
    s_wgt[warp] = n_gt;
    s_weq[warp] = n_eq;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kWarpsPerRow; ++w) {
      g += s_wgt[w];
      e += s_weq[w];
    }
    s_cta_gt = g;
    s_cta_eq = e;
  }
  cluster.sync();  // every CTA's counts are published
  uint32_t gt_before = 0, eq_before = 0;
  for (int r = 0; r < rank; ++r) {
    gt_before += *cluster.map_shared_rank(&s_cta_gt, r);
    eq_before += *cluster.map_shared_rank(&s_cta_eq, r);
  }
  for (int w = 0; w < warp; ++w) {
    gt_before += s_wgt[w];
    eq_before += s_weq[w];
  }
  cluster.sync();  // the peers' counts have been read before any CTA exits
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < s_hi ? keys[i] : 0u;
    const bool is_gt = i < s_hi && key > tau;
    const bool is_eq = i < s_hi && key == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt);
    const uint32_t me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t my_gt = gt_before + __popc(mg & lt_mask);
    const uint32_t my_eq = eq_before + __popc(me & lt_mask);
    if (is_gt || (is_eq && my_eq < (uint32_t)need_eq)) {
      const uint32_t pos = my_gt + min(my_eq, (uint32_t)need_eq);
      out[pos] = lo + i;
    }
    gt_before += __popc(mg);
    eq_before += __popc(me);
  }
}

}  // namespace

size_t topk_smem_bytes(int64_t ld) {
  const int64_t cap = ld < kCacheMaxKeys ? ld : kCacheMaxKeys;
  return (size_t)(kBins + 64 + cap) * sizeof(uint32_t);
}

cudaError_t launch_topk(const float* scores, int rows, int64_t ld, const int32_t* row_len,
                        const int32_t* row_k, int k_max, int32_t* idx_out, unsigned* status,
                        cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.row_len = row_len;
  a.row_k = row_k;
  a.k_max = k_max;
  a.idx_out = idx_out;
  a.cache_cap = (int)(ld < kCacheMaxKeys ? ld : kCacheMaxKeys);
  a.status = status;
  if (ld > kCacheMaxKeys) {
    // one cluster of C CTAs per row, C the smallest power of two whose slices fit the cache
    int C = 2;
    while (C < 16 && (ld + C - 1) / C > kCacheMaxKeys) C *= 2;
    int seg = (int)((ld + C - 1) / C);
    seg = (seg + 31) & ~31;
    if (seg <= kCacheMaxKeys) {
      const size_t smem = (size_t)(kBins + 64 + seg) * sizeof(uint32_t);
      cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)topk_smem_bytes(kCacheMaxKeys));
      if (e != cudaSuccess) return e;
      if (C > 8) {
        e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(rows * C));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)C;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, a, C, seg);
      if (e != cudaSuccess) return e;
      return cudaGetLastError();
    }
  }
  const size_t smem = topk_smem_bytes(ld);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)topk_smem_bytes(kCacheMaxKeys));
  if (e != cudaSuccess) return e;
  topk_kernel<<<rows, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kascade
