// Prefill-phase Kascade kernels on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands in 128-byte-swizzled
// shared memory filled by TMA or cp.async).
//
// Method: Kascade explainer (0h-n0.github.io), 主要な貢献 (tile-level
// post-softmax pooling in prefill), 実装のポイント (128-query tiles),
// 技術的詳細 › アンカーレイヤーと再利用レイヤー and › ヘッドリマッピング.
//
// prefill_attn_kernel<GATHER>: one CTA (128 threads, thread r <-> query row r
//   <-> TMEM lane r) per (query tile t, query head g, sequence b).
//   * anchor (GATHER = false): key blocks 0..t of the causal row, loaded by TMA;
//     block t is the diagonal block and is masked causally.
//   * reuse (GATHER = true): the anchor's indices of row (t, head_map[h]) in
//     blocks of 128 gathered rows (cp.async into the same swizzled layout),
//     then the diagonal block.
//   Per block: S = Q K^T into TMEM (8 MMAs of K = 16), each thread reads its
//   row, online softmax in base 2 (the running maximum is only raised when a
//   block exceeds it by more than 2^8, so the O accumulator in TMEM is rarely
//   rescaled), P (bf16) goes to shared memory, O += P V into TMEM.
//   Epilogue: O / l to bf16 and the natural-log LSE.
// prefill_pool_kernel: one CTA per (tile t >= 1, KV head h, sequence b).  For
//   each key block before the tile it computes S^T = K Q_g^T for the group's
//   query heads (keys on TMEM lanes, queries on columns), so each thread owns
//   one key and sums exp2(s - lse2) over the 128 queries x G heads in
//   registers; pooled = sum / (128 G).
#include "tcgen05.cuh"
#include "internal.h"

#include <cudaTypedefs.h>

#include <cmath>

namespace kascade {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 128;
constexpr uint32_t kHalfBytes = 128u * 128u;     // 64 bf16 columns x 128 rows (one TMA box)
constexpr uint32_t kTileBytes = 2u * kHalfBytes;  // 128 x 128 bf16
constexpr float kRescaleLog2 = 8.f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

// shared-memory map of the attention kernel (offsets from a 1024-aligned base)
constexpr uint32_t kAttnQ = 0;
constexpr uint32_t kAttnK = kTileBytes;                 // 2 stages
constexpr uint32_t kAttnV = kAttnK + 2 * kTileBytes;    // 2 stages
constexpr uint32_t kAttnP = kAttnV + 2 * kTileBytes;
constexpr uint32_t kAttnMisc = kAttnP + kTileBytes;
constexpr uint32_t kAttnSmem = kAttnMisc + 2048 + 1024;  // misc + alignment slack

// shared-memory map of the pooling kernel
constexpr int kPoolHeads = 4;                           // query heads resident at once
constexpr uint32_t kPoolQ = 0;                          // kPoolHeads tiles
constexpr uint32_t kPoolK = kPoolHeads * kTileBytes;    // 2 stages
constexpr uint32_t kPoolMisc = kPoolK + 2 * kTileBytes;
constexpr uint32_t kPoolSmem = kPoolMisc + kPoolHeads * kTile * 4 + 1024 + 1024;

struct AttnArgs {
  int B, Hq, Hkv, G, N, n_tiles;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  const int32_t* idx_k;
  const int32_t* head_map;
  int k_max;
  float scale_log2;
  uint16_t* out;
  float* lse;
  unsigned* status;
};

struct PoolArgs {
  int B, Hq, Hkv, G, N, n_tiles;
  float scale_log2;
  const float* lse;
  float* pooled;
  unsigned* status;
};

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk16) {
  // byte offset of 16-byte chunk `chunk16` (0..15) of row `row` in a 128 x 128 bf16 tile
  return (chunk16 >> 3) * kHalfBytes + row * 128u + (((chunk16 & 7u) ^ (row & 7u)) << 4);
}

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sw128_desc(tile + (uint32_t)(ks >> 2) * kHalfBytes + (uint32_t)(ks & 3) * 32u, 16u, 1024u);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int ks) {
  return sw128_desc(tile + (uint32_t)ks * 2048u, kHalfBytes, 1024u);
}

template <bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAttnMisc);   // q, kv0, kv1, s, o
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kAttnMisc + 64);
  int* s_abort = reinterpret_cast<int*>(smem + kAttnMisc + 68);
  uint8_t* valid = smem + kAttnMisc + 128;                          // [2][128] (gather)

  const int tid = threadIdx.x, warp = tid >> 5;
  const int t = a.n_tiles - 1 - (int)blockIdx.x;  // longest rows first
  const int g = blockIdx.y, b = blockIdx.z;
  const int h = g / a.G;
  const uint32_t bar_q = smem_u32(&bars[0]);
  const uint32_t bar_s = smem_u32(&bars[3]);
  const uint32_t bar_o = smem_u32(&bars[4]);

  // ---- which key blocks ------------------------------------------------------
  int n_gather = 0, kt = 0;
  const int32_t* irow = nullptr;
  if (GATHER) {
    const int am = a.head_map[h];
    bool ok = am >= 0 && am < a.Hkv;
    if (ok) {
      const int64_t row = ((int64_t)b * a.n_tiles + t) * a.Hkv + am;
      kt = a.idx_k[row];
      irow = a.idx + row * a.k_max;
      ok = kt >= 0 && kt <= a.k_max && kt <= kTile * t;
    }
    if (!ok) {
      if (tid == 0) flag_status(a.status, kStatusBadIndex);
      kt = 0;
    }
    n_gather = (kt + kTile - 1) / kTile;
  }
  const int nblk = GATHER ? n_gather + 1 : t + 1;
  const int64_t q_row0 = ((int64_t)b * a.Hq + g) * a.N + (int64_t)kTile * t;
  const int64_t kv_row0 = ((int64_t)b * a.Hkv + h) * a.N;

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(smem_u32(&bars[i]), 1);
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  auto load_block = [&](int jb, int stage) {
    const uint32_t ks = sbase + kAttnK + stage * kTileBytes;
    const uint32_t vs = sbase + kAttnV + stage * kTileBytes;
    if (!GATHER) {
      if (tid == 0) {
        const uint32_t bar = smem_u32(&bars[1 + stage]);
        mbar_expect_tx(bar, 2 * kTileBytes);
        const int y = (int)(kv_row0 + (int64_t)kTile * jb);
        tma_load_2d(ks, &tm_k, 0, y, bar);
        tma_load_2d(ks + kHalfBytes, &tm_k, 64, y, bar);
        tma_load_2d(vs, &tm_v, 0, y, bar);
        tma_load_2d(vs + kHalfBytes, &tm_v, 64, y, bar);
      }
    } else {
      const bool diag = jb == n_gather;
      for (int e = tid; e < kTile * 16; e += kThreads) {
        const int row = e >> 4, c16 = e & 15;
        int key;
        bool ok;
        if (diag) {
          key = kTile * t + row;
          ok = true;
        } else {
          const int pos = kTile * jb + row;
          key = pos < kt ? __ldg(irow + pos) : -1;
          ok = key >= 0 && key < kTile * t;
          if (pos < kt && !ok && c16 == 0) flag_status(a.status, kStatusBadIndex);
        }
        const int64_t src_row = kv_row0 + (ok ? key : 0);
        const uint32_t off = swz(row, c16);
        cp_async16(ks + off, a.k + src_row * kHeadDim + c16 * 8, ok ? 16u : 0u);
        cp_async16(vs + off, a.v + src_row * kHeadDim + c16 * 8, ok ? 16u : 0u);
        if (c16 == 0) valid[stage * kTile + row] = ok ? 1 : 0;
      }
      cp_async_commit();
    }
  };

  if (tid == 0) {
    mbar_expect_tx(bar_q, kTileBytes);
    tma_load_2d(sbase + kAttnQ, &tm_q, 0, (int)q_row0, bar_q);
    tma_load_2d(sbase + kAttnQ + kHalfBytes, &tm_q, 64, (int)q_row0, bar_q);
  }
  load_block(0, 0);

  const uint32_t idesc_s = idesc_bf16(128, 128, false, false);
  const uint32_t idesc_o = idesc_bf16(128, 128, false, true);
  const int r = tid;
  float m_used = -INFINITY, l_sum = 0.f;
  bool failed = false;

  for (int it = 0; it < nblk; ++it) {
    const int stage = it & 1;
    if (it + 1 < nblk) load_block(it + 1, stage ^ 1);
    if (GATHER) {
      if (it + 1 < nblk) cp_async_wait<1>(); else cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncthreads();
    }
    // ---- S = Q K^T --------------------------------------------------------
    if (tid == 0) {
      bool ok = true;
      if (it == 0) ok = mbar_wait(bar_q, 0, a.status);
      if (!GATHER && ok) ok = mbar_wait(smem_u32(&bars[1 + stage]), (it >> 1) & 1, a.status);
      if (ok) {
        tc_fence_after();
        const uint32_t qs = sbase + kAttnQ, ksm = sbase + kAttnK + stage * kTileBytes;
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          umma_ss(tS, kmajor_desc(qs, k16), kmajor_desc(ksm, k16), idesc_s, k16 > 0 ? 1u : 0u);
        umma_commit(bar_s);
      } else {
        *s_abort = 1;
      }
    }
    __syncthreads();
    if (*s_abort) { failed = true; break; }
    if (!mbar_wait(bar_s, it & 1, a.status)) { *s_abort = 1; }
    tc_fence_after();

    // ---- softmax on row r ---------------------------------------------------
    uint32_t sr[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_base + 32 * c, sr[c]);
    tmem_wait_ld();
    const bool is_diag = GATHER ? (it == n_gather) : (it == t);
    const uint8_t* vflags = valid + stage * kTile;
    float mloc = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int col = 32 * c + e;
        bool ok = is_diag ? (col <= r) : (!GATHER || vflags[col]);
        float x = ok ? __uint_as_float(sr[c][e]) * a.scale_log2 : -INFINITY;
        sr[c][e] = __float_as_uint(x);
        mloc = fmaxf(mloc, x);
      }
    }
    float alpha = 1.f;
    bool rescale = false;
    if (m_used == -INFINITY) {
      m_used = mloc;
    } else if (mloc > m_used + kRescaleLog2) {
      alpha = fast_exp2(m_used - mloc);
      m_used = mloc;
      rescale = true;
    }
    const float base = (m_used == -INFINITY) ? 0.f : m_used;
    l_sum *= alpha;
    uint8_t* prow = smem + kAttnP;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {  // 8 keys -> one 16-byte chunk
        uint32_t w[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float p0 = fast_exp2(__uint_as_float(sr[c][8 * q8 + 2 * e2]) - base);
          const float p1 = fast_exp2(__uint_as_float(sr[c][8 * q8 + 2 * e2 + 1]) - base);
          l_sum += p0 + p1;
          w[e2] = pack_bf16x2(p0, p1);
        }
        const uint32_t chunk = (uint32_t)(4 * c + q8);  // keys 8*chunk .. 8*chunk+7
        *reinterpret_cast<uint4*>(prow + swz((uint32_t)r, chunk)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    if (__any_sync(0xffffffffu, rescale) && it > 0) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + lane_base + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(tO + lane_base + 32 * c, o);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- O += P V ---------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ps = sbase + kAttnP, vsm = sbase + kAttnV + stage * kTileBytes;
#pragma unroll
      for (int k16 = 0; k16 < 8; ++k16)
        umma_ss(tO, kmajor_desc(ps, k16), mnmajor_desc(vsm, k16), idesc_o,
                (it > 0 || k16 > 0) ? 1u : 0u);
      umma_commit(bar_o);
    }
    if (!mbar_wait(bar_o, it & 1, a.status)) { *s_abort = 1; }
    tc_fence_after();
    __syncthreads();
    if (*s_abort) { failed = true; break; }
  }

  // ---- epilogue ---------------------------------------------------------------
  if (!failed) {
    const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
    uint16_t* orow = a.out + (q_row0 + r) * kHeadDim;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + lane_base + 32 * c, o);
      tmem_wait_ld();
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(o[8 * q8 + 0]) * inv_l, __uint_as_float(o[8 * q8 + 1]) * inv_l);
        w.y = pack_bf16x2(__uint_as_float(o[8 * q8 + 2]) * inv_l, __uint_as_float(o[8 * q8 + 3]) * inv_l);
        w.z = pack_bf16x2(__uint_as_float(o[8 * q8 + 4]) * inv_l, __uint_as_float(o[8 * q8 + 5]) * inv_l);
        w.w = pack_bf16x2(__uint_as_float(o[8 * q8 + 6]) * inv_l, __uint_as_float(o[8 * q8 + 7]) * inv_l);
        *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q8) = w;
      }
    }
    if (a.lse) a.lse[q_row0 + r] = l_sum > 0.f ? (m_used + __log2f(l_sum)) * kLn2 : -INFINITY;
  }
  if (GATHER) cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_pool_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const PoolArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* lse2 = reinterpret_cast<float*>(smem + kPoolMisc);                   // [kPoolHeads][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPoolMisc + kPoolHeads * kTile * 4);  // q, k0, k1, s
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  int* s_abort = reinterpret_cast<int*>(bars + 9);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int t = a.n_tiles - 1 - (int)blockIdx.x;  // t >= 1, longest first
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = a.G;
  const uint32_t bar_q = smem_u32(&bars[0]);
  const uint32_t bar_s = smem_u32(&bars[3]);
  const int64_t kv_row0 = ((int64_t)b * a.Hkv + h) * a.N;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars[i]), 1);
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t idesc = idesc_bf16(128, 128, false, false);
  float* prow = a.pooled + (((int64_t)b * a.n_tiles + t) * a.Hkv + h) * a.N;
  const float inv_count = 1.f / (float)(kTile * G);

  int it = 0;        // global block counter (K stage / phase bookkeeping)
  int q_phase = 0;
  bool failed = false;
  for (int g0 = 0; g0 < G && !failed; g0 += kPoolHeads) {
    const int hg = min(kPoolHeads, G - g0);
    // queries of the heads in this round, and their log2-domain LSE
    if (tid == 0) {
      mbar_expect_tx(bar_q, hg * kTileBytes);
      for (int j = 0; j < hg; ++j) {
        const int y = (int)(((int64_t)b * a.Hq + h * G + g0 + j) * a.N + (int64_t)kTile * t);
        tma_load_2d(sbase + kPoolQ + j * kTileBytes, &tm_q, 0, y, bar_q);
        tma_load_2d(sbase + kPoolQ + j * kTileBytes + kHalfBytes, &tm_q, 64, y, bar_q);
      }
    }
    for (int e = tid; e < hg * kTile; e += kThreads) {
      const int j = e / kTile, i = e % kTile;
      lse2[e] = a.lse[((int64_t)b * a.Hq + h * G + g0 + j) * a.N + (int64_t)kTile * t + i] * kLog2e;
    }
    auto load_k = [&](int jb, int stage) {
      if (tid == 0) {
        const uint32_t bar = smem_u32(&bars[1 + stage]);
        mbar_expect_tx(bar, kTileBytes);
        const int y = (int)(kv_row0 + (int64_t)kTile * jb);
        const uint32_t ks = sbase + kPoolK + stage * kTileBytes;
        tma_load_2d(ks, &tm_k, 0, y, bar);
        tma_load_2d(ks + kHalfBytes, &tm_k, 64, y, bar);
      }
    };
    load_k(0, it & 1);
    __syncthreads();  // lse2 visible
    for (int jb = 0; jb < t; ++jb, ++it) {
      const int stage = it & 1;
      if (jb + 1 < t) load_k(jb + 1, stage ^ 1);
      if (tid == 0) {
        bool ok = true;
        if (jb == 0) ok = mbar_wait(bar_q, q_phase, a.status);
        if (ok) ok = mbar_wait(smem_u32(&bars[1 + stage]), (it >> 1) & 1, a.status);
        if (ok) {
          tc_fence_after();
          const uint32_t ks = sbase + kPoolK + stage * kTileBytes;
          for (int j = 0; j < hg; ++j) {
            const uint32_t qs = sbase + kPoolQ + j * kTileBytes;
#pragma unroll
            for (int k16 = 0; k16 < 8; ++k16)
              umma_ss(tmem + 128 * j, kmajor_desc(ks, k16), kmajor_desc(qs, k16), idesc,
                      k16 > 0 ? 1u : 0u);
          }
          umma_commit(bar_s);
        } else {
          *s_abort = 1;
        }
      }
      __syncthreads();
      if (*s_abort) { failed = true; break; }
      if (!mbar_wait(bar_s, it & 1, a.status)) { failed = true; }
      tc_fence_after();
      float acc = 0.f;
      for (int j = 0; j < hg; ++j) {
        const float* l2 = lse2 + j * kTile;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sv[32];
          tmem_ld32(tmem + 128 * j + lane_base + 32 * c, sv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            acc += fast_exp2(__uint_as_float(sv[e]) * a.scale_log2 - l2[32 * c + e]);
        }
      }
      const int key = kTile * jb + tid;
      if (g0 == 0) prow[key] = acc * inv_count;
      else prow[key] += acc * inv_count;
      tc_fence_before();
      __syncthreads();
      if (failed) *s_abort = 1;
      __syncthreads();
      if (*s_abort) { failed = true; break; }
    }
    q_phase ^= 1;
    __syncthreads();  // Q tiles and lse2 are replaced by the next round
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D view [rows, 128] bf16, box of 64 columns x 128 rows, 128-byte swizzle.
bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_anchor_workspace_bytes(int, int, int, int) { return 0; }
size_t prefill_reuse_workspace_bytes(int, int, int, int, int) { return 0; }

static cudaError_t launch_attn(const PrefillParams& p, bool gather, cudaStream_t st) {
  const int n_tiles = p.N / kTile;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, p.q, (uint64_t)p.B * p.Hq * p.N) ||
      !make_tile_map(&tk, p.k, (uint64_t)p.B * p.Hkv * p.N) ||
      !make_tile_map(&tv, p.v, (uint64_t)p.B * p.Hkv * p.N))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.G = p.G; a.N = p.N; a.n_tiles = n_tiles;
  a.k = p.k; a.v = p.v; a.idx = p.idx; a.idx_k = p.idx_k; a.head_map = p.head_map;
  a.k_max = p.k_max;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.out = p.out; a.lse = p.lse; a.status = p.status;
  dim3 grid(n_tiles, p.Hq, p.B);
  if (gather) {
    cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
    if (e != cudaSuccess) return e;
    prefill_attn_kernel<true><<<grid, kThreads, kAttnSmem, st>>>(tq, tk, tv, a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
    if (e != cudaSuccess) return e;
    prefill_attn_kernel<false><<<grid, kThreads, kAttnSmem, st>>>(tq, tk, tv, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_prefill_anchor(const PrefillParams& p, cudaStream_t st) {
  cudaError_t e = launch_attn(p, false, st);
  if (e != cudaSuccess) return e;
  const int n_tiles = p.N / kTile;
  if (n_tiles < 2) return cudaSuccess;
  CUtensorMap tq, tk;
  if (!make_tile_map(&tq, p.q, (uint64_t)p.B * p.Hq * p.N) ||
      !make_tile_map(&tk, p.k, (uint64_t)p.B * p.Hkv * p.N))
    return cudaErrorInvalidValue;
  PoolArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.G = p.G; a.N = p.N; a.n_tiles = n_tiles;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.lse = p.lse; a.pooled = p.pooled; a.status = p.status;
  e = cudaFuncSetAttribute(prefill_pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPoolSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_tiles - 1, p.Hkv, p.B);
  prefill_pool_kernel<<<grid, kThreads, kPoolSmem, st>>>(tq, tk, a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_reuse(const PrefillParams& p, cudaStream_t st) {
  return launch_attn(p, true, st);
}

}  // namespace kascade
