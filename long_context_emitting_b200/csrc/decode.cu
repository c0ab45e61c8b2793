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
#include "tcgen05.cuh"

#include <cooperative_groups.h>

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
  const int64_t* kv_off;      // contiguous cache: sequence offsets (NULL when paged)
  const int32_t* block_table; // paged cache: [B, max_pages] page of each page_size tokens
  int max_pages, page_size, num_pages;
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
  uint16_t* out;      // reuse: written by rank 0 of each (b, h) cluster
  float* lse;
  unsigned* status;
};

// Resolve the row list of (b, h).  Returns the number of items (tokens for the
// anchor, selected indices for reuse) and sets T / the index row.
template <bool GATHER>
__device__ __forceinline__ int resolve_rows(const SplitArgs& a, int b, int h, int& T,
                                            int64_t& off, const int32_t*& rows) {
  T = a.seq_len[b];
  off = a.block_table ? 0 : a.kv_off[b];
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

// One block of 16 items (tokens or gathered indices) held in registers.
struct Blk {
  uint4 ka[4], kb[4], va[4], vb[4];
  int ia, ib;        // item positions (for the logits store)
  bool oka, okb;     // rows present
};

// Paged cache: element offset of token t of KV head h of sequence b in a
// [num_pages, Hkv, page_size, 128] page store, or -1 when its page entry is out
// of range.
__device__ __forceinline__ int64_t paged_row(const SplitArgs& a, int b, int h, int t) {
  const int pi = t / a.page_size;
  const int page = __ldg(a.block_table + (int64_t)b * a.max_pages + pi);
  if (page < 0 || page >= a.num_pages) return -1;
  return (((int64_t)page * a.Hkv + h) * a.page_size + (t - pi * a.page_size)) * kHeadDim;
}

// Loads one 16-row block of the anchor's contiguous K/V stream into registers.
__device__ __forceinline__ void load_blk(Blk& x, int i0, int i_end, const uint16_t* Kb, const uint16_t* Vb,
                                         int gid, int tig) {
  x.ia = i0 + gid;
  x.ib = i0 + gid + 8;
  x.oka = x.ia < i_end;
  x.okb = x.ib < i_end;
  // masked lanes address the block's first row, which is < i_end <= T
  const int ra = x.oka ? x.ia : i0, rb = x.okb ? x.ib : i0;
  const uint16_t* kpa = Kb + (int64_t)ra * kHeadDim + 8 * tig;
  const uint16_t* kpb = Kb + (int64_t)rb * kHeadDim + 8 * tig;
  const uint16_t* vpa = Vb + (int64_t)ra * kHeadDim + 8 * tig;
  const uint16_t* vpb = Vb + (int64_t)rb * kHeadDim + 8 * tig;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x.ka[j] = ldg_stream16(kpa + 32 * j);
    x.kb[j] = ldg_stream16(kpb + 32 * j);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x.va[j] = ldg_stream16(vpa + 32 * j);
    x.vb[j] = ldg_stream16(vpb + 32 * j);
  }
}

struct WarpState {
  float m0, m1, l0, l1;
  float o[8][4];
};

template <bool GATHER, bool F16>
__device__ __forceinline__ void compute_blk(const Blk& x, WarpState& w, const uint32_t (&qf)[4][4],
                                            float scale_log2, float* lrow, int G, int tig) {
  // S^T = K · Q^T  (rows: items ia / ib; cols: heads 2tig, 2tig+1)
  float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};  // two independent chains
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    mma_16816<F16>(s, word_of(x.ka[j], 0), word_of(x.kb[j], 0), word_of(x.ka[j], 1),
                   word_of(x.kb[j], 1), qf[j][0], qf[j][1]);
    mma_16816<F16>(s2, word_of(x.ka[j], 2), word_of(x.kb[j], 2), word_of(x.ka[j], 3),
                   word_of(x.kb[j], 3), qf[j][2], qf[j][3]);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) s[e] += s2[e];
  s[0] = x.oka ? s[0] * scale_log2 : -INFINITY;
  s[1] = x.oka ? s[1] * scale_log2 : -INFINITY;
  s[2] = x.okb ? s[2] * scale_log2 : -INFINITY;
  s[3] = x.okb ? s[3] * scale_log2 : -INFINITY;

  if (!GATHER) {
    if (2 * tig + 1 < G) {
      if (x.oka) *reinterpret_cast<float2*>(lrow + (int64_t)x.ia * G + 2 * tig) = make_float2(s[0], s[1]);
      if (x.okb) *reinterpret_cast<float2*>(lrow + (int64_t)x.ib * G + 2 * tig) = make_float2(s[2], s[3]);
    } else if (2 * tig < G) {
      if (x.oka) lrow[(int64_t)x.ia * G + 2 * tig] = s[0];
      if (x.okb) lrow[(int64_t)x.ib * G + 2 * tig] = s[2];
    }
  }

  // online softmax (base 2)
  const float mx0 = warp_max_xor_gid(fmaxf(s[0], s[2]));
  const float mx1 = warp_max_xor_gid(fmaxf(s[1], s[3]));
  const float mn0 = fmaxf(w.m0, mx0), mn1 = fmaxf(w.m1, mx1);
  const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
  const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
  const float al0 = fast_exp2(w.m0 - base0), al1 = fast_exp2(w.m1 - base1);
  const float p0 = fast_exp2(s[0] - base0), p1 = fast_exp2(s[1] - base1);
  const float p2 = fast_exp2(s[2] - base0), p3 = fast_exp2(s[3] - base1);
  w.l0 = w.l0 * al0 + p0 + p2;
  w.l1 = w.l1 * al1 + p1 + p3;
  w.m0 = mn0;
  w.m1 = mn1;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    w.o[mt][0] *= al0; w.o[mt][1] *= al1; w.o[mt][2] *= al0; w.o[mt][3] *= al1;
  }

  // O^T += V^T · P^T
  const uint32_t pb0 = movmatrix_trans(pack_x2<F16>(p0, p1));
  const uint32_t pb1 = movmatrix_trans(pack_x2<F16>(p2, p3));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
      const uint32_t a0 = movmatrix_trans(word_of(x.va[j], 2 * pp));
      const uint32_t a1 = movmatrix_trans(word_of(x.va[j], 2 * pp + 1));
      const uint32_t a2 = movmatrix_trans(word_of(x.vb[j], 2 * pp));
      const uint32_t a3 = movmatrix_trans(word_of(x.vb[j], 2 * pp + 1));
      mma_16816<F16>(w.o[2 * j + pp], a0, a1, a2, a3, pb0, pb1);
    }
  }
}

// Decode anchor over the K/V stream: two register buffers (the next block's
// loads in flight during the current block's math), 2 CTAs per SM.  PAGED: a
// warp's 16-token blocks start at multiples of 16 and the page size is a
// multiple of 16, so each block lies in one page, looked up once per block.
template <bool PAGED, bool F16>
__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(const SplitArgs a) {
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
  int n_items = resolve_rows<false>(a, b, h, T, off, rows);
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

  WarpState ws;
  ws.m0 = ws.m1 = -INFINITY;
  ws.l0 = ws.l1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ws.o[i][0] = ws.o[i][1] = ws.o[i][2] = ws.o[i][3] = 0.f;

  float* lrow = a.logits + ((int64_t)b * a.Hkv + h) * a.max_T * G;

  // the block of tokens i0 .. i0+15: contiguous, or through the block table
  // (a bad page entry masks the whole block, read from page 0)
  auto load = [&](Blk& x, int i0) {
    if constexpr (PAGED) {
      int64_t o = paged_row(a, b, h, i0);
      int end = i_end;
      if (o < 0) {
        flag_status(a.status, kStatusBadIndex);
        o = 0;
        end = i0;
      }
      load_blk(x, 0, end - i0, a.k + o, a.v + o, gid, tig);
      x.ia += i0;
      x.ib += i0;
    } else {
      load_blk(x, i0, i_end, Kb, Vb, gid, tig);
    }
  };
  Blk x0, x1;
  if (i_begin < i_end) load(x0, i_begin);
  for (int i0 = i_begin; i0 < i_end; i0 += 32) {
    const bool has1 = i0 + 16 < i_end;
    if (has1) load(x1, i0 + 16);
    compute_blk<false, F16>(x0, ws, qf, a.scale_log2, lrow, G, tig);
    if (!has1) break;
    if (i0 + 32 < i_end) load(x0, i0 + 32);
    compute_blk<false, F16>(x1, ws, qf, a.scale_log2, lrow, G, tig);
  }

  // ---- merge the 4 warps of the CTA --------------------------------------
  const float lsum0 = warp_sum_xor_gid(ws.l0);
  const float lsum1 = warp_sum_xor_gid(ws.l1);
  if (gid == 0) {
    sm_m[warp][2 * tig] = ws.m0;
    sm_m[warp][2 * tig + 1] = ws.m1;
    sm_l[warp][2 * tig] = lsum0;
    sm_l[warp][2 * tig + 1] = lsum1;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
      const int d0 = 8 * ((gid >> 1) + 4 * j) + 4 * pp + (gid & 1);
      sm_o[warp][2 * tig][d0] = ws.o[2 * j + pp][0];
      sm_o[warp][2 * tig + 1][d0] = ws.o[2 * j + pp][1];
      sm_o[warp][2 * tig][d0 + 2] = ws.o[2 * j + pp][2];
      sm_o[warp][2 * tig + 1][d0 + 2] = ws.o[2 * j + pp][3];
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

// Reuse (gathered rows): each warp keeps kGStages blocks of 16 rows in its own
// shared-memory ring, filled with 16-byte cp.async copies (each warp
// instruction moves two whole 256-byte rows) and consumed by the same warp, so
// the next blocks' loads are in flight while a block is computed without
// holding them in registers.  Chunk c of row r is stored at c ^ 4(r & 1) so the
// fragment reads (rows r, r+1 in one 8-lane phase) hit different banks.
// Masked rows (past the count, or an index out of range) are zero-filled and
// excluded from the softmax.
#ifndef KASCADE_GATHER_STAGES
#define KASCADE_GATHER_STAGES 2
#endif
constexpr int kGStages = KASCADE_GATHER_STAGES;
constexpr uint32_t kGStageBytes = 16u * 512u;  // 16 K rows, then 16 V rows
constexpr uint32_t kGSmem = kWarps * kGStages * kGStageBytes + 128;

__device__ __forceinline__ uint32_t gswz(int r, int c) {
  return (uint32_t)r * 256u + ((uint32_t)(c ^ ((r & 1) << 2)) << 4);
}

template <bool PAGED, bool F16>
__global__ void __launch_bounds__(kThreads, 3) decode_gather_kernel(const SplitArgs a) {
  grid_dependency_wait();
  extern __shared__ uint8_t gsm_raw[];
  uint8_t* gsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsm_raw) + 127) & ~uintptr_t(127));
  __shared__ uint32_t smask[kWarps][kGStages];
  __shared__ float sm_m[kWarps][8];
  __shared__ float sm_l[kWarps][8];
  __shared__ float sm_po[8][kHeadDim];  // this CTA's partial: unnormalised O, max, sum
  __shared__ float sm_pm[8], sm_pl[8];

  const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = a.G;

  int T;
  int64_t off;
  const int32_t* rows;
  int n_items = resolve_rows<true>(a, b, h, T, off, rows);
  if (n_items < 0) {
    if (threadIdx.x == 0 && split == 0) flag_status(a.status, kStatusBadIndex);
    n_items = 0;
  }
  const uint16_t* Kb = a.k + off + (int64_t)h * T * kHeadDim;
  const uint16_t* Vb = a.v + off + (int64_t)h * T * kHeadDim;
  const int i_begin = (split * kWarps + warp) * a.tok_per_warp;
  const int i_end = min(i_begin + a.tok_per_warp, n_items);
  const int nblk = i_end > i_begin ? (i_end - i_begin + 15) / 16 : 0;
  const uint32_t ring = smem_u32(gsm) + (uint32_t)warp * kGStages * kGStageBytes;

  uint32_t qf[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int gq = gid < G ? gid : G - 1;
    uint4 t = ldg16(a.q + ((int64_t)b * a.Hq + h * G + gq) * kHeadDim + 8 * (tig + 4 * j));
    if (gid >= G) t = make_uint4(0, 0, 0, 0);
    qf[j][0] = t.x; qf[j][1] = t.y; qf[j][2] = t.z; qf[j][3] = t.w;
  }

  // lane -> (row parity, 16-byte chunk): rows 2i + (lane >> 4), chunk lane & 15
  const int c16 = lane & 15, rpar = lane >> 4;
  auto issue = [&](int bi) {
    const int st = bi % kGStages;
    const uint32_t dst = ring + (uint32_t)st * kGStageBytes;
    // validity of the block's 16 rows (lanes 0..15), kept for the softmax mask
    const int itv = i_begin + 16 * bi + (lane & 15);
    bool okv = false;
    int64_t rowv = 0;  // paged: element offset of row lane & 15 in the page store
    if (itv < i_end) {
      const int key = __ldg(rows + itv);
      okv = key >= 0 && key < T;
      if constexpr (PAGED) {
        if (okv) {
          rowv = paged_row(a, b, h, key);
          okv = rowv >= 0;
          if (!okv) rowv = 0;
        }
      }
      if (!okv && lane < 16) flag_status(a.status, kStatusBadIndex);
    }
    const unsigned m = __ballot_sync(0xffffffffu, okv) & 0xffffu;
    if (lane == 0) smask[warp][st] = m;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 2 * i + rpar;
      const bool ok = (m >> r) & 1u;
      const uint32_t o = gswz(r, c16);
      if constexpr (PAGED) {
        int64_t ro = __shfl_sync(0xffffffffu, rowv, r);  // offset computed by lane r
        if (!ok) ro = 0;  // zero-filled from a valid address (page 0)
        cp_async16(dst + o, a.k + ro + c16 * 8, ok ? 16u : 0u);
        cp_async16(dst + 4096u + o, a.v + ro + c16 * 8, ok ? 16u : 0u);
      } else {
        const int it = i_begin + 16 * bi + r;
        int key = it < i_end ? __ldg(rows + it) : 0;
        if (!ok) key = 0;  // zero-filled from a valid address (T >= 1 whenever there are items)
        cp_async16(dst + o, Kb + (int64_t)key * kHeadDim + c16 * 8, ok ? 16u : 0u);
        cp_async16(dst + 4096u + o, Vb + (int64_t)key * kHeadDim + c16 * 8, ok ? 16u : 0u);
      }
    }
  };

  WarpState ws;
  ws.m0 = ws.m1 = -INFINITY;
  ws.l0 = ws.l1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ws.o[i][0] = ws.o[i][1] = ws.o[i][2] = ws.o[i][3] = 0.f;

  for (int bi = 0; bi < kGStages - 1; ++bi) {
    if (bi < nblk) issue(bi);
    cp_async_commit();
  }
  for (int bi = 0; bi < nblk; ++bi) {
    if (bi + kGStages - 1 < nblk) issue(bi + kGStages - 1);
    cp_async_commit();                  // one group per block (possibly empty)
    cp_async_wait<kGStages - 1>();      // this lane's copies of block bi landed
    __syncwarp();                       // ... and every other lane's
    const int st = bi % kGStages;
    const uint32_t src = ring + (uint32_t)st * kGStageBytes;
    const uint32_t m = smask[warp][st];
    Blk x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tig + 4 * j;
      x.ka[j] = lds128(src + gswz(gid, c));
      x.kb[j] = lds128(src + gswz(gid + 8, c));
      x.va[j] = lds128(src + 4096u + gswz(gid, c));
      x.vb[j] = lds128(src + 4096u + gswz(gid + 8, c));
    }
    x.oka = (m >> gid) & 1u;
    x.okb = (m >> (gid + 8)) & 1u;
    x.ia = x.ib = 0;
    __syncwarp();                       // stage fully read before it is refilled
    compute_blk<true, F16>(x, ws, qf, a.scale_log2, nullptr, G, tig);
  }
  cp_async_wait<0>();
  allow_dependents_launch();

  // ---- merge the 4 warps (the rings are free now) ---------------------------
  const float lsum0 = warp_sum_xor_gid(ws.l0);
  const float lsum1 = warp_sum_xor_gid(ws.l1);
  __syncthreads();
  float (*sm_o)[8][kHeadDim] = reinterpret_cast<float (*)[8][kHeadDim]>(gsm);  // 16 KB of the rings
  if (gid == 0) {
    sm_m[warp][2 * tig] = ws.m0;
    sm_m[warp][2 * tig + 1] = ws.m1;
    sm_l[warp][2 * tig] = lsum0;
    sm_l[warp][2 * tig + 1] = lsum1;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
      const int d0 = 8 * ((gid >> 1) + 4 * j) + 4 * pp + (gid & 1);
      sm_o[warp][2 * tig][d0] = ws.o[2 * j + pp][0];
      sm_o[warp][2 * tig + 1][d0] = ws.o[2 * j + pp][1];
      sm_o[warp][2 * tig][d0 + 2] = ws.o[2 * j + pp][2];
      sm_o[warp][2 * tig + 1][d0 + 2] = ws.o[2 * j + pp][3];
    }
  }
  __syncthreads();

  // CTA partial of each head, kept in shared memory for the cluster merge
  const int d = threadIdx.x;
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
    sm_po[g][d] = acc;
    if (d == 0) {
      sm_pm[g] = M;
      sm_pl[g] = lsum;
    }
  }

  // The splits of (b, h) form one thread-block cluster: rank 0 merges the
  // others' partials through distributed shared memory.
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  if (cluster.block_rank() == 0) {
    const int ns = (int)cluster.num_blocks();
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
      for (int r = 0; r < ns; ++r) M = fmaxf(M, *cluster.map_shared_rank(&sm_pm[g], r));
      float L = 0.f, acc = 0.f;
      if (M != -INFINITY) {
        for (int r = 0; r < ns; ++r) {
          const float f = fast_exp2(*cluster.map_shared_rank(&sm_pm[g], r) - M);
          L += f * *cluster.map_shared_rank(&sm_pl[g], r);
          acc += f * *cluster.map_shared_rank(&sm_po[g][d], r);
        }
      }
      a.out[((int64_t)b * a.Hq + h * G + g) * kHeadDim + d] = to_bits<F16>(L > 0.f ? acc / L : 0.f);
      if (a.lse && d == 0) a.lse[(int64_t)b * a.Hq + h * G + g] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    }
  }
  cluster.sync();  // peers keep their shared memory until rank 0 has read it
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

template <bool F16>
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
      a.out[((int64_t)b * a.Hq + h * G + g) * kHeadDim + d] = to_bits<F16>(acc);
    }
    if (a.lse && threadIdx.x < G) {
      const float l2 = s_lse2[threadIdx.x];
      a.lse[(int64_t)b * a.Hq + h * G + threadIdx.x] = (l2 == -INFINITY) ? -INFINITY : l2 * kLn2;
    }
  }

  if (a.logits) {
    int T = a.seq_len[b];
    const int64_t off = a.kv_off ? a.kv_off[b] : 0;  // NULL for a paged cache
    if (T < 0 || T > a.max_T || (off & 7) || off < 0) T = 0;
    const int t_lo = chunk * kPoolChunk;
    const int t_hi = min(t_lo + kPoolChunk, T);
    const float* lrow = a.logits + bh * a.max_T * G;
    float* prow = a.pooled + bh * a.ld_pooled;
    const float invG = 1.f / (float)G;
    if (G == 4) {
      const float l0 = s_lse2[0], l1 = s_lse2[1], l2 = s_lse2[2], l3 = s_lse2[3];
      constexpr int kU = kPoolChunk / kCombineThreads;  // tokens per thread, loads issued together
      float4 sv[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = t_lo + threadIdx.x + u * kCombineThreads;
        sv[u] = t < t_hi ? __ldcs(reinterpret_cast<const float4*>(lrow + (int64_t)t * 4))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = t_lo + threadIdx.x + u * kCombineThreads;
        if (t < t_hi)
          prow[t] = (fast_exp2(sv[u].x - l0) + fast_exp2(sv[u].y - l1) + fast_exp2(sv[u].z - l2) +
                     fast_exp2(sv[u].w - l3)) * invG;
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

// Anchor workspace: logits, then the split partials.  Reuse needs none: its
// splits merge on chip.
WsLayout ws_layout(int B, int Hkv, int G, int max_T, int nsplit, bool anchor) {
  WsLayout w = {0, 0, 0, 0};
  if (!anchor) return w;
  size_t off = 0;
  w.logits = off;
  off = align_up(off + (size_t)B * Hkv * max_T * G * sizeof(float), 256);
  w.part_ml = off;
  off = align_up(off + (size_t)B * Hkv * nsplit * G * 2 * sizeof(float), 256);
  w.part_o = off;
  off = align_up(off + (size_t)B * Hkv * nsplit * G * kHeadDim * sizeof(float), 256);
  w.total = off;
  return w;
}

}  // namespace

// The split policy assumes B200's 148 SMs (here and in kSlots below) rather
// than querying the device: the workspace query has no device argument, and
// its size must equal what the launch uses.  On a part with another SM count
// the results are the same, only the occupancy differs.
#ifndef KASCADE_DECODE_TARGET_CTAS
#define KASCADE_DECODE_TARGET_CTAS (4 * 148)
#endif
#ifndef KASCADE_DECODE_MAX_TPW
#define KASCADE_DECODE_MAX_TPW 256
#endif

DecodeSplit decode_split_for(int units, int n_items, bool gather) {
  DecodeSplit s;
  if (gather) {
    // One wave of the gather kernel (3 resident CTAs per SM): split each row
    // into floor(444 / rows) CTAs (between 1 and 16), 4 warps each, 16-row
    // blocks.  The splits of a row form one thread-block cluster: up to 8 is the
    // portable size, 16 needs the non-portable attribute set at launch.
    constexpr int kSlots = 3 * 148;
    int nsplit = units >= kSlots ? 1 : kSlots / units;
    if (nsplit > 16) nsplit = 16;
    // 64-bit intermediates: n_items may be near the 2^30 row-length limit
    int64_t tpw = ((int64_t)n_items + 4 * nsplit - 1) / (4 * nsplit);
    tpw = ((tpw + 15) / 16) * 16;
    s.tok_per_warp = (int)(tpw > 16 ? tpw : 16);
    const int64_t per_cta = 4 * (int64_t)s.tok_per_warp;
    s.nsplit = n_items > 0 ? (int)(((int64_t)n_items + per_cta - 1) / per_cta) : 1;
    return s;
  }
  // Largest per-warp run (<= KASCADE_DECODE_MAX_TPW items) that still gives at
  // least KASCADE_DECODE_TARGET_CTAS CTAs.  Runs stay multiples of 16 (halving
  // from a power of two >= 16), which the paged path relies on: a 16-token block
  // never crosses a page.
  static_assert(KASCADE_DECODE_MAX_TPW >= 16 && (KASCADE_DECODE_MAX_TPW & (KASCADE_DECODE_MAX_TPW - 1)) == 0,
                "per-warp runs must stay multiples of 16");
  constexpr int kTargetCtas = KASCADE_DECODE_TARGET_CTAS;
  int tpw = KASCADE_DECODE_MAX_TPW;
  while (tpw > 16) {
    const int64_t per_cta = (int64_t)kWarps * tpw;
    const int64_t ctas = (int64_t)units * (((int64_t)n_items + per_cta - 1) / per_cta);
    if (ctas >= kTargetCtas) break;
    tpw /= 2;
  }
  s.tok_per_warp = tpw;
  const int64_t per_cta = (int64_t)kWarps * tpw;
  s.nsplit = n_items > 0 ? (int)(((int64_t)n_items + per_cta - 1) / per_cta) : 1;
  return s;
}

size_t decode_workspace_bytes(int B, int Hkv, int G, int n_items, bool with_logits) {
  const DecodeSplit sp = decode_split_for(B * Hkv, n_items, !with_logits);
  return ws_layout(B, Hkv, G, n_items, sp.nsplit, with_logits).total;
}

static cudaError_t launch_decode(const DecodeParams& p, bool gather, cudaStream_t st) {
  const int n_items = gather ? p.k_max : p.max_T;
  const DecodeSplit sp = decode_split_for(p.B * p.Hkv, n_items, gather);
  const WsLayout w = ws_layout(p.B, p.Hkv, p.G, n_items, sp.nsplit, !gather);
  char* ws = static_cast<char*>(p.ws);

  SplitArgs a;
  a.q = p.q; a.k = p.k; a.v = p.v; a.kv_off = p.kv_off; a.seq_len = p.seq_len;
  a.block_table = p.block_table; a.max_pages = p.max_pages; a.page_size = p.page_size;
  a.num_pages = p.num_pages;
  const bool paged = p.block_table != nullptr;
  a.idx = p.idx; a.idx_k = p.idx_k; a.head_map = p.head_map; a.k_max = p.k_max;
  a.Hq = p.Hq; a.Hkv = p.Hkv; a.G = p.G; a.max_T = p.max_T;
  a.tok_per_warp = sp.tok_per_warp;
  a.nsplit = sp.nsplit;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.logits = gather ? nullptr : reinterpret_cast<float*>(ws + w.logits);
  a.part_ml = gather ? nullptr : reinterpret_cast<float*>(ws + w.part_ml);
  a.part_o = gather ? nullptr : reinterpret_cast<float*>(ws + w.part_o);
  a.out = p.out;
  a.lse = p.lse;
  a.status = p.status;

  dim3 grid(sp.nsplit, p.Hkv, p.B);
  if (gather) {
    // reuse: the nsplit CTAs of each (b, h) are one cluster and merge on chip
    auto kern = paged ? (p.f16 ? decode_gather_kernel<true, true> : decode_gather_kernel<true, false>)
                      : (p.f16 ? decode_gather_kernel<false, true> : decode_gather_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem);
    if (e != cudaSuccess) return e;
    if (sp.nsplit > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kGSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = sp.nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attribute();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  auto split = paged ? (p.f16 ? decode_split_kernel<true, true> : decode_split_kernel<true, false>)
                     : (p.f16 ? decode_split_kernel<false, true> : decode_split_kernel<false, false>);
  split<<<grid, kThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  CombineArgs c;
  c.kv_off = p.kv_off; c.seq_len = p.seq_len;
  c.Hq = p.Hq; c.Hkv = p.Hkv; c.G = p.G; c.max_T = p.max_T; c.nsplit = sp.nsplit;
  c.part_ml = a.part_ml; c.part_o = a.part_o;
  c.logits = a.logits;
  c.pooled = p.pooled; c.ld_pooled = p.ld_pooled;
  c.out = p.out; c.lse = p.lse;
  const int nchunk = max(1, (p.max_T + kPoolChunk - 1) / kPoolChunk);
  dim3 cgrid(nchunk, p.Hkv, p.B);
  if (p.f16) decode_combine_kernel<true><<<cgrid, kCombineThreads, 0, st>>>(c);
  else decode_combine_kernel<false><<<cgrid, kCombineThreads, 0, st>>>(c);
  return cudaGetLastError();
}

cudaError_t launch_decode_anchor(const DecodeParams& p, cudaStream_t st) {
  return launch_decode(p, false, st);
}

cudaError_t launch_decode_reuse(const DecodeParams& p, cudaStream_t st) {
  return launch_decode(p, true, st);
}

}  // namespace kascade
