// Calibration parts of Kascade: the cross-layer similarity ratio on the GPU
// and the anchor-selection dynamic program on the host.
//
// Method: Kascade explainer (0h-n0.github.io), レイヤー間類似度とアンカーレイヤー選択
// (the sim equation: the share of layer b's Top-k probability mass that layer
// a's Top-k indices recover) and 動的計画法 (Algorithm 1: choose M anchor layers
// maximising the covered weighted similarity, O(M L^2)).
//
// similarity_rows_kernel
//   One CTA per output row r (head remap: one per (reuse head, anchor head,
//   query row), the rows implied by the index arithmetic).  With rb = b_row[r] (or r) and ra = a_row[r] (or
//   r) it sums, in fp64, P_b[rb, idx_a[ra, i]] and P_b[rb, idx_b[rb, i]] over
//   i < k = row_k[rb], and writes their ratio.  The index lists are the Top-k
//   outputs of layers a and b; indices outside [0, row_len[rb]) are skipped and
//   flagged in the device status.
// group_mean_kernel / remap_argmax_kernel
//   The aggregation of the ratios: the mean over a layer's rows (sim(a, b)),
//   and for the head remap the mean over queries of every head pair followed by
//   the argmax over anchor heads, ties to the lower head (ヘッドリマッピング).
#include "common.cuh"
#include "internal.h"

#include <cmath>
#include <vector>

namespace kascade {

namespace {

constexpr int kSimThreads = 256;

__global__ void __launch_bounds__(kSimThreads) similarity_rows_kernel(const SimArgs a) {
  __shared__ double s_num[kSimThreads / 32], s_den[kSimThreads / 32];
  const int r = blockIdx.x;
  int rb, ra;
  if (a.remap_Q > 0) {
    // every (reuse head h, anchor head an, row q): r = (h * Hkv + an) * Q + q
    const int Q = a.remap_Q, HQ = a.remap_H * a.remap_Q;
    const int h = r / HQ, an = (r % HQ) / Q, q = r % Q;
    rb = h * Q + q;
    ra = an * Q + q;
  } else {
    rb = a.b_row ? a.b_row[r] : r;
    ra = a.a_row ? a.a_row[r] : r;
  }
  double num = 0.0, den = 0.0;
  bool bad = rb < 0 || rb >= a.rows || ra < 0 || ra >= a.rows;
  if (!bad) {
    const int len = a.row_len[rb];
    const int k = a.row_k[rb];
    if (len < 0 || (int64_t)len > a.ld || k < 0 || k > len || k > a.k_max) {
      bad = true;
    } else {
      const float* p = a.p_b + (int64_t)rb * a.ld;
      const int32_t* ia = a.idx_a + (int64_t)ra * a.k_max;
      const int32_t* ib = a.idx_b + (int64_t)rb * a.k_max;
      for (int i = threadIdx.x; i < k; i += kSimThreads) {
        const int ja = __ldg(ia + i), jb = __ldg(ib + i);
        if (ja >= 0 && ja < len) num += (double)__ldg(p + ja);
        else bad = true;
        if (jb >= 0 && jb < len) den += (double)__ldg(p + jb);
        else bad = true;
      }
    }
  }
  if (bad) flag_status(a.status, kStatusBadIndex);
  for (int o = 16; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_num[warp] = num;
    s_den[warp] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double n = 0.0, d = 0.0;
    for (int w = 0; w < kSimThreads / 32; ++w) {  // fixed order: deterministic
      n += s_num[w];
      d += s_den[w];
    }
    a.ratio[r] = d > 0.0 ? n / d : 0.0;
  }
}

// Mean of each group of `len` consecutive ratios, in fp64 with a fixed
// summation order (strided per-thread sums, then a fixed tree), one CTA per group.
__global__ void __launch_bounds__(kSimThreads) group_mean_kernel(const double* ratio, int len, double* mean) {
  __shared__ double s_sum[kSimThreads / 32];
  const double* g = ratio + (int64_t)blockIdx.x * len;
  double acc = 0.0;
  for (int i = threadIdx.x; i < len; i += kSimThreads) acc += g[i];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_sum[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kSimThreads / 32; ++w) t += s_sum[w];
    mean[blockIdx.x] = len > 0 ? t / (double)len : 0.0;
  }
}

// head_map[h] = argmax over anchor heads a of sim[h][a], the lowest a among
// equal maxima; one thread per reuse head.
__global__ void remap_argmax_kernel(const double* sim, int Hkv, int32_t* head_map) {
  const int h = threadIdx.x;
  if (h >= Hkv) return;
  int best = 0;
  double bv = sim[(int64_t)h * Hkv];
  for (int a = 1; a < Hkv; ++a) {
    const double v = sim[(int64_t)h * Hkv + a];
    if (v > bv) {
      bv = v;
      best = a;
    }
  }
  head_map[h] = best;
}

}  // namespace

cudaError_t launch_similarity_rows(const SimArgs& a, int n_out, cudaStream_t st) {
  if (n_out == 0) return cudaSuccess;
  similarity_rows_kernel<<<n_out, kSimThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_similarity_mean(const SimArgs& a, double* ratio_ws, double* mean, cudaStream_t st) {
  SimArgs r = a;
  r.ratio = ratio_ws;
  cudaError_t e = launch_similarity_rows(r, a.rows, st);
  if (e != cudaSuccess) return e;
  group_mean_kernel<<<1, kSimThreads, 0, st>>>(ratio_ws, a.rows, mean);
  return cudaGetLastError();
}

cudaError_t launch_head_remap(const SimArgs& a, int Hkv, int Q, double* ratio_ws, double* sim,
                              int32_t* head_map, cudaStream_t st) {
  SimArgs r = a;
  r.ratio = ratio_ws;
  r.remap_H = Hkv;
  r.remap_Q = Q;
  r.b_row = r.a_row = nullptr;
  cudaError_t e = launch_similarity_rows(r, Hkv * Hkv * Q, st);
  if (e != cudaSuccess) return e;
  group_mean_kernel<<<Hkv * Hkv, kSimThreads, 0, st>>>(ratio_ws, Q, sim);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  remap_argmax_kernel<<<1, 32 * ((Hkv + 31) / 32), 0, st>>>(sim, Hkv, head_map);
  return cudaGetLastError();
}

// Algorithm 1 with the readings of the DP bounds: layers 0..L-1, dp[0][0] = 0,
// dp[0][j > 0] = -inf, dp[m][j] = max over i = m-1 .. j-1 of
// dp[m-1][i] + sum_{l=i}^{j-1} S[i][l]; the answer is dp[M][L]; the smallest i
// is kept among equal maxima; the anchors come back by backtracking.
void select_anchors_dp(const double* S, int L, int M, int32_t* anchors, double* best) {
  std::vector<double> cover((size_t)(L + 1) * (L + 1), 0.0);  // cover[i][j]
  for (int i = 0; i < L; ++i) {
    double run = 0.0;
    for (int j = i + 1; j <= L; ++j) {
      run += S[(size_t)i * L + (j - 1)];
      cover[(size_t)i * (L + 1) + j] = run;
    }
  }
  const double neg = -INFINITY;
  std::vector<double> dp((size_t)(M + 1) * (L + 1), neg);
  std::vector<int> arg((size_t)(M + 1) * (L + 1), -1);
  auto at = [&](int m, int j) { return (size_t)m * (L + 1) + j; };
  dp[at(0, 0)] = 0.0;
  for (int m = 1; m <= M; ++m) {
    for (int j = m; j <= L; ++j) {
      double b = neg;
      int bi = -1;
      for (int i = m - 1; i < j; ++i) {
        const double prev = dp[at(m - 1, i)];
        if (prev == neg) continue;
        const double v = prev + cover[(size_t)i * (L + 1) + j];
        if (v > b) {
          b = v;
          bi = i;
        }
      }
      dp[at(m, j)] = b;
      arg[at(m, j)] = bi;
    }
  }
  int j = L;
  for (int m = M; m >= 1; --m) {
    const int i = arg[at(m, j)];
    anchors[m - 1] = i;  // backtracking visits the anchors from the last to the first
    j = i;
  }
  *best = dp[at(M, L)];
}

}  // namespace kascade
