// Decode-phase Kascade kernels: split-K anchor attention that also records the
// scaled logits for the pooled-probability epilogue, the gathered reuse
// attention, and the combine/pooling kernel that finishes both.
//
// Method: Kascade explainer (0h-n0.github.io), 技術的詳細 › アンカーレイヤーと再利用レイヤー
// (anchor = full attention + post-softmax Top-k; reuse = attention over the
// anchor's keys) and › ヘッドリマッピング (per key head, via a head map).
//
// Work decomposition (per sequence b, KV head h): the key range is cut into
// splits of 4 warps x `tok_per_warp` tokens.  A warp walks its tokens 16 at a
// time with no shared-memory staging:
//   * each lane loads 16-byte chunks of two key rows and two value rows
//     (lane (g, t) of the mma layout owns rows g and g+8, chunks t, t+4, t+8,
//     t+12 -- 64 contiguous bytes per row per load instruction);
//   * S^T[16 tokens x 8 heads] = K · Q^T runs on mma.sync m16n8k16 with the
//     group's G <= 8 query heads as the N dimension.  The head dimension is
//     consumed in a permuted order that matches the chunk ownership above; Q
//     is loaded in the same order, so the dot products are unchanged;
//   * online softmax in base 2 (scale·log2 e folded into the logits);
//   * O^T[128 dims x 8 heads] += V^T · P^T, with V and P transposed in
//     registers by movmatrix.
// The 4 warps' partial states are merged in shared memory and one (m, l, o)
// partial per split is written to the workspace; the combine kernel merges the
// splits, writes O and the log-sum-exp, and (anchor) turns the stored logits
// into pooled probabilities, mean over the group's query heads.
#include "common.cuh"
#include "internal.h"

#include <cmath>

namespace kascade {

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kCombineThreads = 256;
constexpr int kPoolChunk = 2048;  // tokens per combine block for the pooled pass
constexpr float kLn2 = 0.6931471805599453f;

struct SplitArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int64_t* kv_off;
  const int32_t* seq_len;
  const int32_t* idx;
  const int32_t* idx_k;
  const int32_t* head_map;
  int k_max;
  int Hq, Hkv, G, max_T;
  int tok_per_warp;
  int nsplit;
  float scale_log2;
  float* logits;   // anchor: [B, Hkv, max_T, G] base-2 scaled logits
  float* part_ml;  // [B*Hkv, nsplit, G, 2]  (running max, running sum)
  float* part_o;   // [B*Hkv, nsplit, G, 128] unnormalised output
  unsigned* status;
};

// Resolve the row list of (b, h).  Returns the number of items (tokens for the
// anchor, selected indices for reuse) and sets T / the index row.
template <bool GATHER>
__device__ __forceinline__ int resolve_rows(const SplitArgs& a, int b, int h, int& T,
                                            int64_t& off, const int32_t*& rows) {
  T = a.seq_len[b];
  off = a.kv_off[b];
  bool ok = (T >= 0) && (T <= a.max_T) && ((off & 7) == 0) && off >= 0;
  int n = T;
  rows = nullptr;
  if (GATHER && ok) {
    const int am = a.head_map[h];
    if (am < 0 || am >= a.Hkv) {
      ok = false;
    } else {
      rows = a.idx + ((int64_t)b * a.Hkv + am) * a.k_max;
      n = a.idx_k[b * a.Hkv + am];
      if (n < 0 || n > a.k_max) ok = false;
    }
  }
  if (GATHER && T == 0) n = 0;  // nothing to gather from an empty sequence
  if (!ok) {
    T = 0;
    n = 0;
  }
  return ok ? n : -1;
}

template <bool GATHER>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(const SplitArgs a) {
  __shared__ float sm_o[kWarps][8][kHeadDim];
  __shared__ float sm_m[kWarps][8];
  __shared__ float sm_l[kWarps][8];

  const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = a.G;

  int T;
  int64_t off;
  const int32_t* rows;
  int n_items = resolve_rows<GATHER>(a, b, h, T, off, rows);
  if (n_items < 0) {
    if (threadIdx.x == 0 && split == 0) flag_status(a.status, kStatusBadIndex);
    n_items = 0;
  }

  const uint16_t* Kb = a.k + off + (int64_t)h * T * kHeadDim;
  const uint16_t* Vb = a.v + off + (int64_t)h * T * kHeadDim;
  const int i_begin = (split * kWarps + warp) * a.tok_per_warp;
  const int i_end = min(i_begin + a.tok_per_warp, n_items);

  // Q^T fragments of head `gid` (zero rows for gid >= G), chunks tig + 4j.
  uint32_t qf[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // rows gid >= G are padding: load a valid row (gid clamped) and zero it
    const int gq = gid < G ? gid : G - 1;
    uint4 t = ldg16(a.q + ((int64_t)b * a.Hq + h * G + gq) * kHeadDim + 8 * (tig + 4 * j));
    if (gid >= G) t = make_uint4(0, 0, 0, 0);
    qf[j][0] = t.x; qf[j][1] = t.y; qf[j][2] = t.z; qf[j][3] = t.w;
  }

  float m_run0 = -INFINITY, m_run1 = -INFINITY;
  float l_run0 = 0.f, l_run1 = 0.f;
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  float* lrow = nullptr;
  if (!GATHER) lrow = a.logits + ((int64_t)b * a.Hkv + h) * a.max_T * G;

  for (int i0 = i_begin; i0 < i_end; i0 += 16) {
    const int ia = i0 + gid, ib = i0 + gid + 8;
    bool va = ia < i_end, vb = ib < i_end;
    int ra = ia, rb = ib;
    if (GATHER) {
      ra = va ? __ldg(rows + ia) : 0;
      rb = vb ? __ldg(rows + ib) : 0;
      if (va && (ra < 0 || ra >= T)) { flag_status(a.status, kStatusBadIndex); va = false; }
      if (vb && (rb < 0 || rb >= T)) { flag_status(a.status, kStatusBadIndex); vb = false; }
      // masked lanes address row 0 (T >= 1 here), so no address leaves the sequence
      if (!va) ra = 0;
      if (!vb) rb = 0;
    } else {
      // masked lanes address the block's first row, which is < i_end <= T
      if (!va) ra = i0;
      if (!vb) rb = i0;
    }
    const uint16_t* kpa = Kb + (int64_t)ra * kHeadDim + 8 * tig;
    const uint16_t* kpb = Kb + (int64_t)rb * kHeadDim + 8 * tig;
    const uint16_t* vpa = Vb + (int64_t)ra * kHeadDim + 8 * tig;
    const uint16_t* vpb = Vb + (int64_t)rb * kHeadDim + 8 * tig;
    uint4 ka[4], kb[4], va4[4], vb4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ka[j] = va ? ldg_stream16(kpa + 32 * j) : make_uint4(0, 0, 0, 0);
      kb[j] = vb ? ldg_stream16(kpb + 32 * j) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va4[j] = va ? ldg_stream16(vpa + 32 * j) : make_uint4(0, 0, 0, 0);
      vb4[j] = vb ? ldg_stream16(vpb + 32 * j) : make_uint4(0, 0, 0, 0);
    }

    // S^T = K · Q^T  (rows: tokens ia / ib; cols: heads 2tig, 2tig+1)
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int st = 0; st < 8; ++st) {
      const int j = st >> 1, hf = st & 1;
      mma_bf16_16816(s, word_of(ka[j], 2 * hf), word_of(kb[j], 2 * hf),
                     word_of(ka[j], 2 * hf + 1), word_of(kb[j], 2 * hf + 1),
                     qf[j][2 * hf], qf[j][2 * hf + 1]);
    }
    s[0] = va ? s[0] * a.scale_log2 : -INFINITY;
    s[1] = va ? s[1] * a.scale_log2 : -INFINITY;
    s[2] = vb ? s[2] * a.scale_log2 : -INFINITY;
    s[3] = vb ? s[3] * a.scale_log2 : -INFINITY;

    if (!GATHER) {
      if (2 * tig + 1 < G) {
        if (va) *reinterpret_cast<float2*>(lrow + (int64_t)ia * G + 2 * tig) = make_float2(s[0], s[1]);
        if (vb) *reinterpret_cast<float2*>(lrow + (int64_t)ib * G + 2 * tig) = make_float2(s[2], s[3]);
      } else if (2 * tig < G) {
        if (va) lrow[(int64_t)ia * G + 2 * tig] = s[0];
        if (vb) lrow[(int64_t)ib * G + 2 * tig] = s[2];
      }
    }

    // online softmax (base 2)
    const float mx0 = warp_max_xor_gid(fmaxf(s[0], s[2]));
    const float mx1 = warp_max_xor_gid(fmaxf(s[1], s[3]));
    const float mn0 = fmaxf(m_run0, mx0), mn1 = fmaxf(m_run1, mx1);
    const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = fast_exp2(m_run0 - base0), al1 = fast_exp2(m_run1 - base1);
    const float p0 = fast_exp2(s[0] - base0), p1 = fast_exp2(s[1] - base1);
    const float p2 = fast_exp2(s[2] - base0), p3 = fast_exp2(s[3] - base1);
    l_run0 = l_run0 * al0 + p0 + p2;
    l_run1 = l_run1 * al1 + p1 + p3;
    m_run0 = mn0;
    m_run1 = mn1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      o[mt][0] *= al0; o[mt][1] *= al1; o[mt][2] *= al0; o[mt][3] *= al1;
    }

    // O^T += V^T · P^T
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        const uint32_t a0 = movmatrix_trans(word_of(va4[j], 2 * pp));
        const uint32_t a1 = movmatrix_trans(word_of(va4[j], 2 * pp + 1));
        const uint32_t a2 = movmatrix_trans(word_of(vb4[j], 2 * pp));
        const uint32_t a3 = movmatrix_trans(word_of(vb4[j], 2 * pp + 1));
        mma_bf16_16816(o[2 * j + pp], a0, a1, a2, a3, pb0, pb1);
      }
    }
  }

  // ---- merge the 4 warps of the CTA --------------------------------------
  const float lsum0 = warp_sum_xor_gid(l_run0);
  const float lsum1 = warp_sum_xor_gid(l_run1);
  if (gid == 0) {
    sm_m[warp][2 * tig] = m_run0;
    sm_m[warp][2 * tig + 1] = m_run1;
    sm_l[warp][2 * tig] = lsum0;
    sm_l[warp][2 * tig + 1] = lsum1;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
      const int d0 = 8 * ((gid >> 1) + 4 * j) + 4 * pp + (gid & 1);
      sm_o[warp][2 * tig][d0] = o[2 * j + pp][0];
      sm_o[warp][2 * tig + 1][d0] = o[2 * j + pp][1];
      sm_o[warp][2 * tig][d0 + 2] = o[2 * j + pp][2];
      sm_o[warp][2 * tig + 1][d0 + 2] = o[2 * j + pp][3];
    }
  }
  __syncthreads();

  const int64_t bh = (int64_t)b * a.Hkv + h;
  const int d = threadIdx.x;  // kThreads == kHeadDim
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][g]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = fast_exp2(sm_m[w][g] - M);
        acc += f * sm_o[w][g][d];
        lsum += f * sm_l[w][g];
      }
    }
    const int64_t slot = (bh * a.nsplit + split) * G + g;
    a.part_o[slot * kHeadDim + d] = acc;
    if (d == 0) {
      a.part_ml[slot * 2 + 0] = M;
      a.part_ml[slot * 2 + 1] = lsum;
    }
  }
}

struct CombineArgs {
  const int64_t* kv_off;
  const int32_t* seq_len;
  int Hq, Hkv, G, max_T, nsplit;
  const float* part_ml;
  const float* part_o;
  const float* logits;  // NULL: no pooled output
  float* pooled;
  int64_t ld_pooled;
  uint16_t* out;
  float* lse;
};

__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(const CombineArgs a) {
  __shared__ float s_M[8], s_L[8], s_lse2[8];
  const int b = blockIdx.z, h = blockIdx.y, chunk = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.G;
  const int64_t bh = (int64_t)b * a.Hkv + h;

  if (warp < G) {
    const float* ml = a.part_ml + bh * a.nsplit * G * 2;
    float M = -INFINITY;
    for (int s = lane; s < a.nsplit; s += 32) M = fmaxf(M, ml[(s * G + warp) * 2]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    if (M != -INFINITY)
      for (int s = lane; s < a.nsplit; s += 32)
        L += fast_exp2(ml[(s * G + warp) * 2] - M) * ml[(s * G + warp) * 2 + 1];
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      s_M[warp] = M;
      s_L[warp] = L;
      s_lse2[warp] = (L > 0.f) ? M + __log2f(L) : -INFINITY;
    }
  }
  __syncthreads();

  if (chunk == 0) {
    for (int e = threadIdx.x; e < G * kHeadDim; e += kCombineThreads) {
      const int g = e / kHeadDim, d = e % kHeadDim;
      const float M = s_M[g], L = s_L[g];
      float acc = 0.f;
      if (L > 0.f) {
        const float* ml = a.part_ml + bh * a.nsplit * G * 2;
        const float* po = a.part_o + bh * a.nsplit * G * kHeadDim;
        for (int s = 0; s < a.nsplit; ++s)
          acc += fast_exp2(ml[(s * G + g) * 2] - M) * po[((int64_t)s * G + g) * kHeadDim + d];
        acc /= L;
      }
      a.out[((int64_t)b * a.Hq + h * G + g) * kHeadDim + d] = to_bf16_bits(acc);
    }
    if (a.lse && threadIdx.x < G) {
      const float l2 = s_lse2[threadIdx.x];
      a.lse[(int64_t)b * a.Hq + h * G + threadIdx.x] = (l2 == -INFINITY) ? -INFINITY : l2 * kLn2;
    }
  }

  if (a.logits) {
    int T = a.seq_len[b];
    const int64_t off = a.kv_off[b];
    if (T < 0 || T > a.max_T || (off & 7) || off < 0) T = 0;
    const int t_lo = chunk * kPoolChunk;
    const int t_hi = min(t_lo + kPoolChunk, T);
    const float* lrow = a.logits + bh * a.max_T * G;
    float* prow = a.pooled + bh * a.ld_pooled;
    const float invG = 1.f / (float)G;
    if (G == 4) {
      const float l0 = s_lse2[0], l1 = s_lse2[1], l2 = s_lse2[2], l3 = s_lse2[3];
      for (int t = t_lo + threadIdx.x; t < t_hi; t += kCombineThreads) {
        const float4 s = *reinterpret_cast<const float4*>(lrow + (int64_t)t * 4);
        prow[t] = (fast_exp2(s.x - l0) + fast_exp2(s.y - l1) + fast_exp2(s.z - l2) +
                   fast_exp2(s.w - l3)) * invG;
      }
    } else {
      for (int t = t_lo + threadIdx.x; t < t_hi; t += kCombineThreads) {
        float acc = 0.f;
        for (int g = 0; g < G; ++g) acc += fast_exp2(lrow[(int64_t)t * G + g] - s_lse2[g]);
        prow[t] = acc * invG;
      }
    }
  }
}

struct WsLayout {
  size_t logits, part_ml, part_o, total;
};

WsLayout ws_layout(int B, int Hkv, int G, int max_T, int nsplit, bool with_logits) {
  WsLayout w;
  size_t off = 0;
  w.logits = off;
  if (with_logits) off = align_up(off + (size_t)B * Hkv * max_T * G * sizeof(float), 256);
  w.part_ml = off;
  off = align_up(off + (size_t)B * Hkv * nsplit * G * 2 * sizeof(float), 256);
  w.part_o = off;
  off = align_up(off + (size_t)B * Hkv * nsplit * G * kHeadDim * sizeof(float), 256);
  w.total = off;
  return w;
}

}  // namespace

DecodeSplit decode_split_for(int units, int n_items) {
  // Largest per-warp run (<= 256 items) that still gives >= 4 CTAs per SM.
  constexpr int kTargetCtas = 4 * 148;
  int tpw = 256;
  while (tpw > 16) {
    const int per_cta = kWarps * tpw;
    const long long ctas = (long long)units * ((n_items + per_cta - 1) / per_cta);
    if (ctas >= kTargetCtas) break;
    tpw /= 2;
  }
  DecodeSplit s;
  s.tok_per_warp = tpw;
  s.nsplit = n_items > 0 ? (n_items + kWarps * tpw - 1) / (kWarps * tpw) : 1;
  return s;
}

size_t decode_workspace_bytes(int B, int Hkv, int G, int n_items, bool with_logits) {
  const DecodeSplit sp = decode_split_for(B * Hkv, n_items);
  return ws_layout(B, Hkv, G, n_items, sp.nsplit, with_logits).total;
}

static cudaError_t launch_decode(const DecodeParams& p, bool gather, cudaStream_t st) {
  const int n_items = gather ? p.k_max : p.max_T;
  const DecodeSplit sp = decode_split_for(p.B * p.Hkv, n_items);
  const WsLayout w = ws_layout(p.B, p.Hkv, p.G, n_items, sp.nsplit, !gather);
  char* ws = static_cast<char*>(p.ws);

  SplitArgs a;
  a.q = p.q; a.k = p.k; a.v = p.v; a.kv_off = p.kv_off; a.seq_len = p.seq_len;
  a.idx = p.idx; a.idx_k = p.idx_k; a.head_map = p.head_map; a.k_max = p.k_max;
  a.Hq = p.Hq; a.Hkv = p.Hkv; a.G = p.G; a.max_T = p.max_T;
  a.tok_per_warp = sp.tok_per_warp;
  a.nsplit = sp.nsplit;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.logits = gather ? nullptr : reinterpret_cast<float*>(ws + w.logits);
  a.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
  a.part_o = reinterpret_cast<float*>(ws + w.part_o);
  a.status = p.status;

  dim3 grid(sp.nsplit, p.Hkv, p.B);
  if (gather)
    decode_split_kernel<true><<<grid, kThreads, 0, st>>>(a);
  else
    decode_split_kernel<false><<<grid, kThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  CombineArgs c;
  c.kv_off = p.kv_off; c.seq_len = p.seq_len;
  c.Hq = p.Hq; c.Hkv = p.Hkv; c.G = p.G; c.max_T = p.max_T; c.nsplit = sp.nsplit;
  c.part_ml = a.part_ml; c.part_o = a.part_o;
  c.logits = a.logits;
  c.pooled = p.pooled; c.ld_pooled = p.ld_pooled;
  c.out = p.out; c.lse = p.lse;
  const int nchunk = gather ? 1 : max(1, (p.max_T + kPoolChunk - 1) / kPoolChunk);
  dim3 cgrid(nchunk, p.Hkv, p.B);
  decode_combine_kernel<<<cgrid, kCombineThreads, 0, st>>>(c);
  return cudaGetLastError();
}

cudaError_t launch_decode_anchor(const DecodeParams& p, cudaStream_t st) {
  return launch_decode(p, false, st);
}

cudaError_t launch_decode_reuse(const DecodeParams& p, cudaStream_t st) {
  return launch_decode(p, true, st);
}

}  // namespace kascade
