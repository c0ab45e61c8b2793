// Prefill-phase Kascade kernels on the 5th-generation tensor cores
// (tcgen05.mma with accumulators in tensor memory, operands in 128-byte-
// swizzled shared memory filled by TMA).
//
// Method: Kascade explainer (0h-n0.github.io), 主要な貢献 (tile-level
// post-softmax pooling in prefill), 実装のポイント (128-query tiles),
// 技術的詳細 › アンカーレイヤーと再利用レイヤー and › ヘッドリマッピング.
//
// prefill_attn_kernel<GATHER, F16>  (F16: fp16 data, else bf16)
//   Work item: (query tile t, pair of query heads of one GQA group, sequence);
//   the grid has one CTA per item, in item order (longest tiles first).  CTAs
//   are persistent: when a CTA's producer reaches the last key block of its
//   item it asks the hardware (cluster launch control) to cancel the launch of
//   the next CTA that has not started and takes over that CTA's item, so
//   about one CTA per SM runs all items in launch order, and the next item's
//   query tiles and key blocks load while the current item finishes.
//   The two heads share every K/V block, so each block is loaded once for two
//   128 x 128 attention tiles.  Warp roles (384 threads, three warpgroups):
//     warp 8      TMA producer: Q tiles, then K/V blocks into a 2-stage ring
//                 that continues across the CTA's items; scheduling requests.
//                 anchor: dense key blocks 0..t (block t is the diagonal);
//                 reuse: the anchor's indices of row (t, head_map[h]) gathered
//                 with cp.async (two whole rows per warp instruction) into the
//                 same swizzled layout by warps 8, 10 and 11 together, then the
//                 diagonal block by TMA.
//     warp 9      MMA issuer (one thread): S_i = Q_i K^T into TMEM, and
//                 O_i += P_i V with P_i read from TMEM (it overwrites S_i).
//     warps 0-7   softmax, one warpgroup per tile, one query row (TMEM lane)
//                 per thread: the row's 128 scores are loaded into registers
//                 at once, so the row maximum needs no exchange between
//                 threads.  Online softmax in base 2 (the running maximum is
//                 raised only when a block exceeds it by 2^8, so O is rarely
//                 rescaled); P goes back to TMEM as bf16 over the row's S, in
//                 two halves of 64 keys, each handed to the MMA as soon as it
//                 is stored (PV of the first half overlaps the exponentials of
//                 the second).  Each warp writes its 32 rows of O through a
//                 swizzled shared-memory stage and TMA stores.
//   The MMA thread alternates between the tiles, so the tensor cores work on
//   one tile while the other tile's softmax runs.  The softmax warpgroups take
//   registers from the third one (setmaxnreg; the launch checks the split).
//   TMEM (512 columns): S0|P0 [0,128), O0 [128,256), S1|P1 [256,384), O1 [384,512).
//
// prefill_pool_kernel
//   One CTA per (tile t >= 1, KV head, sequence), longest tiles first.  For each key block before
//   the tile it computes S^T = K Q_g^T for the group's query heads (keys on
//   TMEM lanes, queries on columns, one 128-column TMEM tile per head), so a
//   thread owns one key and sums exp2(s - lse2) over the tile's queries in
//   registers (2 of 8 exponentials on the FMA pipe, the rest on the SFU).
//   The -lse term enters through one extra K16 step of the MMA (ones on the
//   key side, -lse/scale split into three bf16 parts on the query side), so
//   the summing loop reads no per-query values from shared memory.
//   Warp roles (640 threads): a TMA producer and an MMA issuer in warpgroup 0,
//   and four summing warpgroups, one per head of the round; a head's tile goes
//   back to the MMA as soon as its scores are in registers.  The heads' sums
//   are added through shared memory and pooled = sum / (128 G) is written
//   once, without atomics.
#include "exp2_poly.cuh"
#include "f32x2.cuh"
#include "tcgen05.cuh"
#include "internal.h"

#include <cudaTypedefs.h>

#include <cmath>


namespace kascade {

namespace {

constexpr int kTile = 128;
constexpr uint32_t kHalfBytes = 128u * 128u;     // 64 bf16 columns x 128 rows (one TMA box)
constexpr uint32_t kTileBytes = 2u * kHalfBytes;  // 128 x 128 bf16
constexpr float kRescaleLog2 = 8.f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- attention kernel layout ----
constexpr int kAttnThreads = 384;  // softmax warps 0-7, producer warp 8, MMA warp 9, 10-11 gather helpers
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kGatherWarps = 3;    // reuse: warps 8, 10 and 11 share the row gathers of a block
// setmaxnreg split: the launch gives every thread kLaunchRegs (the compiler's
// count, checked on the host); the third warpgroup releases down to kOtherRegs
// and the two softmax warpgroups take exactly what it releases.
constexpr int kLaunchRegs = 168, kSoftmaxRegs = 200, kOtherRegs = 104;
static_assert((kLaunchRegs - kOtherRegs) * 128 >= (kSoftmaxRegs - kLaunchRegs) * 256,
              "softmax register increase must fit in what the third warpgroup releases");
static_assert(kLaunchRegs * kAttnThreads <= 65536, "launch registers exceed the SM");
constexpr uint32_t kAttnQ = 0;                         // 2 query tiles
constexpr uint32_t kAttnKV = 2 * kTileBytes;           // stage s: K at +2s*tile, V at +(2s+1)*tile
// O staging for the TMA stores: per softmax warp 32 rows x 64 columns (4 KB)
constexpr uint32_t kAttnStage = kAttnKV + 4 * kTileBytes;
constexpr uint32_t kStageWarpBytes = 32u * 128u;
constexpr uint32_t kAttnMisc = kAttnStage + 8 * kStageWarpBytes;
// misc: barriers, TMEM address, abort flag, gather masks, scheduling responses
constexpr uint32_t kMiscTmem = 192, kMiscAbort = 200, kMiscMasks = 224, kMiscClc = 256, kMiscItem = 288;
constexpr uint32_t kAttnSmem = kAttnMisc + 512 + 1024;  // misc + alignment slack
static_assert(kAttnSmem <= 227u * 1024u, "attention shared memory exceeds the per-block limit");
// QFree: the item's S MMAs have read its query tiles; ClcFull: a scheduling
// response has landed (read by the producer); Item: the producer has
// published the next item in its slot; ClcEmpty: every other role has read it
enum { kBarQ = 0, kBarKvFull = 1, kBarKvEmpty = 3, kBarS = 5, kBarP = 7, kBarO = 11, kBarQFree = 13,
       kBarClcFull = 14, kBarClcEmpty = 16, kBarItem = 18, kAttnBars = 20 };
static_assert(kAttnBars * 8 <= kMiscTmem, "attention barriers overlap the misc fields");

// ---- pooling kernel layout ----
constexpr int kPoolThreads = 640;  // warpgroup 0: TMA (warp 0), MMA (warp 1), TMEM owner (warp 2);
                                   // warpgroups 1-4: summing, one per head of the round
constexpr int kPoolHeads = 4;                           // query heads resident at once
// setmaxnreg split of the 96 x 640 launch registers: warpgroup 0 releases down to
// 64, the four summing warpgroups take exactly that.
constexpr int kPoolLaunchRegs = 96, kPoolSumRegs = 104, kPoolCtlRegs = 64;
static_assert((kPoolLaunchRegs - kPoolCtlRegs) * 128 >= (kPoolSumRegs - kPoolLaunchRegs) * 512,
              "summing register increase must fit in what warpgroup 0 releases");
static_assert(kPoolLaunchRegs * kPoolThreads <= 65536, "launch registers exceed the SM");
// Q tiles as [64-dimension half][head][128 rows][128 B]: the rows of two
// consecutive heads are contiguous, so a pair of heads is one N = 256 operand.
constexpr uint32_t kPoolQ = 0;
constexpr uint32_t kPoolK = kPoolHeads * kTileBytes;    // 2 stages
// One extra K16 step folds -lse into the MMA: K-side rows [1, 1, 1, 0 ...],
// query-side rows [-v_hi, -v_mid, -v_lo, 0 ...] with v = lse / scale split into
// three bf16 terms (32-byte-swizzled K-major tiles of 128 rows x 16).
constexpr uint32_t kXBytes = 128u * 32u;
constexpr uint32_t kPoolKx = kPoolK + 2 * kTileBytes;
constexpr uint32_t kPoolQx = kPoolKx + kXBytes;         // [kPoolHeads] tiles
constexpr uint32_t kPoolRed = kPoolQx + kPoolHeads * kXBytes;  // [2 slots][3 heads][128] floats
constexpr uint32_t kPoolMisc = kPoolRed + 2 * 3 * kTile * 4;
constexpr uint32_t kPoolSmem = kPoolMisc + 256 + 1024;
// per TMEM buffer (two, alternating by sub-iteration): S^T full (MMA commit) /
// free (read into registers, one arrival per warp); partial-sum exchange:
// warpgroups 1.. -> warpgroup 0, double-buffered by block
enum { kPBarQ = 0, kPBarKFull = 1, kPBarKEmpty = 3, kPBarS = 5, kPBarFree = 7, kPBarRedFull = 9,
       kPBarRedEmpty = 11, kPoolBars = 13 };

struct AttnArgs {
  int B, Hq, Hkv, G, N, n_tiles;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  const int32_t* idx_k;
  const int32_t* head_map;
  int k_max;
  int head_major;  // anchor item order: key head by key head (set when K/V exceed half of L2)
  float scale_log2;
  uint16_t* out;
  float* lse;
  unsigned* status;
};

struct PoolArgs {
  int B, Hq, Hkv, G, N, n_tiles;
  float scale_log2;
  float inv_scale;  // 1 / scale
  const float* lse;
  float* pooled;
  unsigned* status;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sw128_desc(tile + (uint32_t)(ks >> 2) * kHalfBytes + (uint32_t)(ks & 3) * 32u, 16u, 1024u);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int ks) {
  return sw128_desc(tile + (uint32_t)ks * 2048u, kHalfBytes, 1024u);
}
// The start-address field is the low 14 bits of (address >> 4); shared
// addresses stay below 2^18, so a k-step is a constant added to a base
// descriptor (no carry out of the field).  Saves the MMA-issuing thread, which
// shares its scheduler with busy softmax warps, most of its instructions.
__device__ __forceinline__ constexpr uint64_t kmajor_step(int ks) {
  return (uint64_t)(((uint32_t)(ks >> 2) * kHalfBytes + (uint32_t)(ks & 3) * 32u) >> 4);
}
__device__ __forceinline__ constexpr uint64_t mnmajor_step(int ks) { return (uint64_t)(ks * 2048u >> 4); }
// k-step of the pooling kernel's [64-dim half][head][rows] Q layout
__device__ __forceinline__ constexpr uint64_t qpair_step(int ks) {
  return (uint64_t)(((uint32_t)(ks >> 2) * 4u * kHalfBytes + (uint32_t)(ks & 3) * 32u) >> 4);
}

// One unit of work of the attention kernel: query tile t of heads g0 .. g0 +
// ntile - 1 (one GQA group, key head h) of sequence b, with its key blocks.
// Item order (the grid's, kept by taking over pending CTAs in launch order):
// anchor: longest tiles first over the whole grid (every head group and
// sequence of tile t before any of tile t - 1), so no long tile starts late;
// when all heads' K/V exceed half of L2, key head by key head instead
// (longest tiles first within each), so the K/V being re-read by the running
// CTAs stays in L2 (131K tokens: 204.4 against 211.9 ms; at 16K the global
// order is 1-2% faster);
// reuse: tiles longest first within each head group, the head groups one
// after another (the CTAs running together then gather from the same key
// head's rows, which measured faster than the global order).
struct AttnItem {
  int t, g0, b, h;
  int nblk;      // key blocks: anchor 0..t; reuse n_gather gathered + the diagonal
  int n_gather;  // reuse: gathered blocks (kt keys of the anchor's row)
  int kt;
  const int32_t* irow;
  int64_t q_row0;
  int kv_row0;
};

// The item's fields from its index and (reuse) the two values read from
// device memory: kt keys in the anchor's index row and the anchor key head am
// (already checked; kt = 0 when the row was unusable).
template <bool GATHER>
__device__ __forceinline__ AttnItem attn_item_of(const AttnArgs& a, int item, int ntile, int kt, int am) {
  AttnItem w;
  const int HG = a.Hq / ntile;
  int rem;
  if (GATHER) {
    w.t = a.n_tiles - 1 - item % a.n_tiles;
    rem = item / a.n_tiles;
  } else if (a.head_major) {
    const int PH = HG / a.Hkv;  // head pairs per key head
    const int p = item % PH, rest = item / PH;
    w.t = a.n_tiles - 1 - rest % a.n_tiles;
    const int bh = rest / a.n_tiles;
    rem = (bh / a.Hkv) * HG + (bh % a.Hkv) * PH + p;
  } else {
    w.t = a.n_tiles - 1 - item / (HG * a.B);
    rem = item % (HG * a.B);
  }
  w.g0 = (rem % HG) * ntile;
  w.b = rem / HG;
  w.h = w.g0 / a.G;
  w.kt = GATHER ? kt : 0;
  w.irow = GATHER ? a.idx + (((int64_t)w.b * a.n_tiles + w.t) * a.Hkv + am) * a.k_max : nullptr;
  w.n_gather = (w.kt + kTile - 1) / kTile;
  w.nblk = GATHER ? w.n_gather + 1 : w.t + 1;
  w.q_row0 = ((int64_t)w.b * a.Hq + w.g0) * a.N + (int64_t)kTile * w.t;
  w.kv_row0 = (int)(((int64_t)w.b * a.Hkv + w.h) * a.N);
  return w;
}

// Reads (reuse) the item's anchor head and index count and checks them;
// returns kt and am for attn_item_of.
template <bool GATHER>
__device__ __forceinline__ void attn_item_load(const AttnArgs& a, int item, int ntile, bool flag_errors,
                                               int& kt, int& am) {
  kt = 0;
  am = 0;
  if (GATHER) {
    const int HG = a.Hq / ntile;
    const int t = a.n_tiles - 1 - item % a.n_tiles;
    const int rem = item / a.n_tiles;
    const int b = rem / HG, h = (rem % HG) * ntile / a.G;
    const int m = a.head_map[h];
    bool ok = m >= 0 && m < a.Hkv;
    if (ok) {
      const int64_t row = ((int64_t)b * a.n_tiles + t) * a.Hkv + m;
      kt = a.idx_k[row];
      ok = kt >= 0 && kt <= a.k_max && kt <= kTile * t;
      am = m;
    }
    if (!ok) {
      if (flag_errors) flag_status(a.status, kStatusBadIndex);
      kt = 0;
      am = 0;
    }
  }
}

template <bool GATHER>
__device__ __forceinline__ AttnItem attn_item(const AttnArgs& a, int item, int ntile, bool flag_errors) {
  int kt, am;
  attn_item_load<GATHER>(a, item, ntile, flag_errors, kt, am);
  return attn_item_of<GATHER>(a, item, ntile, kt, am);
}

template <bool GATHER, bool F16>
__global__ void __launch_bounds__(kAttnThreads, 1)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* misc = smem + kAttnMisc;
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + kMiscTmem);
  volatile int* s_abort = reinterpret_cast<volatile int*>(misc + kMiscAbort);
  uint32_t* masks = reinterpret_cast<uint32_t*>(misc + kMiscMasks);  // [2 stages][4]
  const uint32_t clc_resp = smem_u32(misc + kMiscClc);                // [2] x 16 bytes
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntile = a.G >= 2 ? 2 : 1;
  // Persistent CTAs: a CTA starts with item blockIdx.x; while working on its
  // item at position pos of its sequence it asks (request pos) to take over
  // the next CTA of the grid that has not started, and continues with that
  // CTA's item.  The K/V stage ring and the per-block barriers run on one
  // block counter g over all the CTA's items, so the next item's loads and
  // its first S MMAs overlap the current item's last blocks and epilogue.
  // The producer asks for the next item when it reaches the current item's
  // last key block (late enough that the item taken is the next one due, early
  // enough that its loads start before this item's compute ends), reads the
  // item's anchor head and index count, and publishes {item, kt, am} in slot
  // pos & 1 of shared memory.  Readers of a slot besides the producer warp:
  // the MMA warp, the softmax warps in use and (reuse) the two gather helpers.
  int* item_slot = reinterpret_cast<int*>(misc + kMiscItem);  // [2][4]
  const uint32_t n_clc_readers = 1u + 4u * (uint32_t)ntile + (GATHER ? 2u : 0u);
  auto read_item = [&](int pos, int& kt, int& am) -> int {  // one thread
    int nx = -1;
    kt = 0;
    am = 0;
    if (mbar_wait(bar(kBarItem + (pos & 1)), (pos >> 1) & 1, a.status)) {
      const volatile int* sl = item_slot + 4 * (pos & 1);
      nx = sl[0];
      kt = sl[1];
      am = sl[2];
    } else {
      *s_abort = 1;
    }
    mbar_arrive(bar(kBarClcEmpty + (pos & 1)));
    return nx;
  };

  if (tid == 0) {
    for (int i = 0; i < kAttnBars; ++i) {
      uint32_t count = 1;
      if (i >= kBarP && i < kBarP + 4) count = 4;  // 4 softmax warps per tile
      if (GATHER && i >= kBarKvFull && i < kBarKvFull + 2) count = kGatherWarps;  // one arrival per gather warp
      if (i >= kBarClcEmpty && i < kBarClcEmpty + 2) count = n_clc_readers;  // (Item: the producer, 1)
      mbar_init(bar(i), count);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    setmaxnreg_dec<kOtherRegs>();
    // gather warp index: producer warp 8 is 0, warps 10 and 11 are 1 and 2 (reuse only)
    const int gw = warp == kProducerWarp ? 0 : (warp >= 10 ? warp - 9 : -1);
    if (gw == 0 || (GATHER && gw > 0)) {
      // ================================ TMA producer ================================
      const bool leader = gw == 0 && lane == 0;  // issues TMA copies and the scheduling requests
      // Reuse: the gathered rows of a layer are first read from DRAM at scattered
      // positions; their latency would exceed a block's compute.  Each gather warp
      // pulls its share of the rows of block j + 2 into L2 before it waits for
      // the stage of block j, so the later copies are L2 hits.
      auto prefetch_rows = [&](const AttnItem& w, int jp) {
        if constexpr (GATHER) {
          if (jp >= w.n_gather) return;
          for (int r = gw + kGatherWarps * lane; r < kTile; r += kGatherWarps * 32) {
            const int pos = kTile * jp + r;
            if (pos >= w.kt) break;
            const int key = __ldg(w.irow + pos);
            if (key < 0 || key >= kTile * w.t) continue;  // flagged when the block is gathered
            const int64_t off = ((int64_t)w.kv_row0 + key) * kHeadDim;
            prefetch_l2(a.k + off);
            prefetch_l2(a.k + off + 64);
            prefetch_l2(a.v + off);
            prefetch_l2(a.v + off + 64);
          }
        }
      };
      // The item's query tiles (leader).  Their buffer is free once the previous
      // item's S MMAs have read it.
      // leader: the loads an abort must wait for, two bits per barrier (issued,
      // phase parity): field 0 the query tiles (kBarQ), 1 + s K/V stage s
      uint32_t inflight = 0u;
      auto note_load = [&](int field, uint32_t parity) {
        inflight = (inflight & ~(3u << (2 * field))) | ((1u | (parity << 1)) << (2 * field));
      };
      auto load_q = [&](const AttnItem& w) {
        const uint32_t qf = inflight & 3u;
        note_load(0, (qf & 1u) ? ((qf >> 1) ^ 1u) : 0u);  // the next kBarQ phase
        mbar_expect_tx(bar(kBarQ), ntile * kTileBytes);
        for (int i = 0; i < ntile; ++i) {
          const int y = (int)(w.q_row0 + (int64_t)i * a.N);
          tma_load_2d(sbase + kAttnQ + i * kTileBytes, &tm_q, 0, y, bar(kBarQ));
          tma_load_2d(sbase + kAttnQ + i * kTileBytes + kHalfBytes, &tm_q, 64, y, bar(kBarQ));
        }
      };
      AttnItem it = attn_item<GATHER>(a, blockIdx.x, ntile, leader);
      prefetch_rows(it, 0);
      prefetch_rows(it, 1);
      uint32_t g = 0;            // key blocks of the CTA's earlier items
      int unread = -1;           // leader: a request whose response it has not read
      bool q_pending = false;    // leader: this item's query tiles still to load
      if (leader) load_q(it);  // later items' tiles are loaded as the previous item ends
      for (int pos = 0;; ++pos) {
        bool ok = !__any_sync(0xffffffffu, *s_abort != 0);
        for (int j = 0; ok && j < it.nblk; ++j) {
          const uint32_t gb = g + (uint32_t)j;
          const int st = (int)(gb & 1u);
          const bool dense = !GATHER || j == it.n_gather;
          // Gathered block: every gather warp loads the block's 128 key indices in
          // one coalesced round (row 32e + lane in kix[e], its validity in bit lane
          // of m[e]) before it waits for the stage, so their latency overlaps the
          // block in flight instead of preceding the copies.
          int kix[4] = {0, 0, 0, 0};
          uint32_t m[4] = {0u, 0u, 0u, 0u};
          if (GATHER && !dense) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int pos_k = kTile * j + 32 * e + lane;
              kix[e] = pos_k < it.kt ? __ldg(it.irow + pos_k) : -1;
            }
          }
          prefetch_rows(it, j + 2);
          if (leader && j == it.nblk - 1) {
            // request the item after this one (slot pos & 1, free once every
            // reader has taken item pos - 1 from it)
            if (pos < 2 || mbar_wait(bar(kBarClcEmpty + (pos & 1)), ((pos >> 1) - 1) & 1, a.status)) {
              mbar_expect_tx(bar(kBarClcFull + (pos & 1)), 16);
              clc_try_cancel(clc_resp + 16u * (uint32_t)(pos & 1), bar(kBarClcFull + (pos & 1)));
              unread = pos;
            } else {
              *s_abort = 1;
            }
          }
          if (GATHER && !dense) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int pos_k = kTile * j + 32 * e + lane;
              const bool v = kix[e] >= 0 && kix[e] < kTile * it.t;
              if (gw == 0 && pos_k < it.kt && !v) flag_status(a.status, kStatusBadIndex);
              m[e] = __ballot_sync(0xffffffffu, v);
              if (!v) kix[e] = kTile * it.t;  // a valid row; the copy of a masked row is zero-filled
            }
          }
          if (gb >= 2 && !mbar_wait(bar(kBarKvEmpty + st), ((gb >> 1) - 1) & 1, a.status)) *s_abort = 1;
          if (__any_sync(0xffffffffu, *s_abort != 0)) {
            ok = false;
            break;
          }
          const uint32_t kb = sbase + kAttnKV + (2 * st) * kTileBytes;
          const uint32_t vb = kb + kTileBytes;
          if (dense) {
            if (gw > 0) {
              if (lane == 0) mbar_arrive(bar(kBarKvFull + st));  // helpers complete the count
            } else if (lane == 0) {
              mbar_expect_tx(bar(kBarKvFull + st), 2 * kTileBytes);
              note_load(1 + st, (gb >> 1) & 1u);
              const int y = it.kv_row0 + kTile * (GATHER ? it.t : j);
              tma_load_2d(kb, &tm_k, 0, y, bar(kBarKvFull + st));
              tma_load_2d(kb + kHalfBytes, &tm_k, 64, y, bar(kBarKvFull + st));
              tma_load_2d(vb, &tm_v, 0, y, bar(kBarKvFull + st));
              tma_load_2d(vb + kHalfBytes, &tm_v, 64, y, bar(kBarKvFull + st));
            }
            if (leader && q_pending) {
              if (mbar_wait(bar(kBarQFree), (pos - 1) & 1, a.status)) load_q(it);
              else *s_abort = 1;
              q_pending = false;
            }
          } else {
            // Copy: each warp instruction moves two whole 256-byte rows (16 lanes per
            // row, one 16-byte chunk each) into the swizzled layout; masked rows are
            // zero-filled from a valid address.  The gather warps take every third
            // pair of rows; a row's index comes from the lane that loaded it.
            const int c16 = lane & 15;
            const uint32_t half = (uint32_t)(c16 >> 3) * kHalfBytes;
#pragma unroll
            for (int i = 0; i < (kTile / 2 + kGatherWarps - 1) / kGatherWarps; ++i) {
              const int s2 = gw + kGatherWarps * i;  // warp-uniform
              if (s2 < kTile / 2) {
                const int row = 2 * s2 + (lane >> 4);
                const int e = s2 >> 4;  // = row >> 5 for both rows of the pair
                const int ke = e == 0 ? kix[0] : e == 1 ? kix[1] : e == 2 ? kix[2] : kix[3];
                const uint32_t me = e == 0 ? m[0] : e == 1 ? m[1] : e == 2 ? m[2] : m[3];
                const int key = __shfl_sync(0xffffffffu, ke, row & 31);
                const bool v = (me >> (row & 31)) & 1u;
                const int64_t src = (int64_t)it.kv_row0 + key;
                const uint32_t off = half + (uint32_t)row * 128u + ((uint32_t)((c16 & 7) ^ (row & 7)) << 4);
                cp_async16(kb + off, a.k + src * kHeadDim + c16 * 8, v ? 16u : 0u);
                cp_async16(vb + off, a.v + src * kHeadDim + c16 * 8, v ? 16u : 0u);
              }
            }
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();  // the tensor cores read these rows through the async proxy
            __syncwarp();
            if (lane == 0) {
              if (gw == 0) {
#pragma unroll
                for (int e = 0; e < 4; ++e) masks[st * 4 + e] = m[e];
              }
              mbar_arrive(bar(kBarKvFull + st));  // release: rows (and masks) visible
            }
            if (leader && q_pending) {
              if (mbar_wait(bar(kBarQFree), (pos - 1) & 1, a.status)) load_q(it);
              else *s_abort = 1;
              q_pending = false;
            }
          }
        }
        if (!ok) break;
        g += (uint32_t)it.nblk;
        // the next item: the leader reads the response, the item's index row
        // and publishes it; the helpers take it from the slot
        int nx = -1, nkt = 0, nam = 0;
        if (leader) {
          if (mbar_wait(bar(kBarClcFull + (pos & 1)), (pos >> 1) & 1, a.status)) {
            nx = clc_response_x(clc_resp + 16u * (uint32_t)(pos & 1));
            fence_proxy_async_smem();  // read before the slot is written again by the async unit
            if (nx >= (int)gridDim.x) {  // not a CTA of this grid: stop rather than index with it
              flag_status(a.status, kStatusBadIndex);
              *s_abort = 1;
              nx = -1;
            }
          } else {
            *s_abort = 1;
          }
          unread = -1;
          if (nx >= 0) attn_item_load<GATHER>(a, nx, ntile, true, nkt, nam);
          int* sl = item_slot + 4 * (pos & 1);
          sl[0] = nx;
          sl[1] = nkt;
          sl[2] = nam;
          mbar_arrive(bar(kBarItem + (pos & 1)));  // release: the slot's fields
        } else if (gw > 0 && lane == 0) {
          nx = read_item(pos, nkt, nam);
        }
        nx = __shfl_sync(0xffffffffu, nx, 0);
        nkt = __shfl_sync(0xffffffffu, nkt, 0);
        nam = __shfl_sync(0xffffffffu, nam, 0);
        if (nx < 0 || __any_sync(0xffffffffu, *s_abort != 0)) break;
        it = attn_item_of<GATHER>(a, nx, ntile, nkt, nam);
        if (leader) {
          // its query tiles: toward L2 at once; into shared memory once its first
          // K/V block is on its way and this item's last S MMAs have completed
          // (both are needed by the item's first S MMA, so their loads overlap)
          for (int i = 0; i < ntile; ++i) {
            const int y = (int)(it.q_row0 + (int64_t)i * a.N);
            tma_prefetch_l2_2d(&tm_q, 0, y);
            tma_prefetch_l2_2d(&tm_q, 64, y);
          }
          q_pending = true;  // loaded once this item's first K/V block is on its way
        }
        if (__any_sync(0xffffffffu, *s_abort != 0)) break;
        prefetch_rows(it, 0);
        prefetch_rows(it, 1);
      }
      // never leave with a response still to land in shared memory
      if (leader && unread >= 0) mbar_wait(bar(kBarClcFull + (unread & 1)), (unread >> 1) & 1, a.status);
      // after an abort, wait (bounded) for the copies this thread started: the
      // last query-tile load and the last TMA load into each stage (a gathered
      // block's cp.async copies are waited for by the warps that issue them)
      if (leader && *s_abort) {
        for (int f = 0; f < 3; ++f)
          if ((inflight >> (2 * f)) & 1u)
            mbar_wait(bar(f == 0 ? kBarQ : kBarKvFull + f - 1), (inflight >> (2 * f + 1)) & 1u, a.status);
      }
    } else if (warp == kMmaWarp) {
      // ================================ MMA issuer ==================================
      if (lane == 0) {
        const uint32_t idesc_s = idesc_f16kind(128, 128, false, false, F16);
        const uint32_t idesc_o = idesc_f16kind(128, 128, false, true, F16);
        // base descriptors: query tiles, and K / V of the two stages
        const uint64_t dq0 = kmajor_desc(sbase + kAttnQ, 0);
        const uint64_t dq1 = kmajor_desc(sbase + kAttnQ + kTileBytes, 0);
        const uint64_t dk0 = kmajor_desc(sbase + kAttnKV, 0);
        const uint64_t dk1 = kmajor_desc(sbase + kAttnKV + 2 * kTileBytes, 0);
        const uint64_t dv0 = mnmajor_desc(sbase + kAttnKV + kTileBytes, 0);
        const uint64_t dv1 = mnmajor_desc(sbase + kAttnKV + 3 * kTileBytes, 0);
        auto issue_s = [&](int i, int st) {
          const uint64_t dq = i ? dq1 : dq0, dk = st ? dk1 : dk0;
          const uint32_t d = tmem + 256 * i;
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            umma_ss(d, dq + kmajor_step(k16), dk + kmajor_step(k16), idesc_s, k16 > 0 ? 1u : 0u);
        };
        // P (128 keys as bf16 pairs) sits in columns 0..63 of the tile's S region.
        // The first PV of an item overwrites O: the softmax warps arrive on P
        // only after the previous item's epilogue has read O out of TMEM.
        auto issue_pv = [&](int i, int st, bool acc, int k0) {  // keys 16*k0 .. 16*k0+63
          const uint64_t dv = st ? dv1 : dv0;
          const uint32_t d = tmem + 256 * i + 128, pa = tmem + 256 * i;
#pragma unroll
          for (int k16 = k0; k16 < k0 + 4; ++k16)
            umma_ts(d, pa + 8 * k16, dv + mnmajor_step(k16), idesc_o, (acc || k16 > 0) ? 1u : 0u);
        };
        int item = blockIdx.x, kt, am;
        attn_item_load<GATHER>(a, item, ntile, false, kt, am);
        uint32_t g = 0;
        for (int pos = 0;; ++pos) {
          const int nblk = attn_item_of<GATHER>(a, item, ntile, kt, am).nblk;
          bool ok = mbar_wait(bar(kBarQ), pos & 1, a.status);
          for (int j = 0; ok && j < nblk; ++j) {
            const uint32_t gb = g + (uint32_t)j;
            const int st = (int)(gb & 1u);
            const uint32_t ph = gb & 1u;
            if (!(ok = mbar_wait(bar(kBarKvFull + st), (gb >> 1) & 1, a.status))) break;
            tc_fence_after();
            if (j == 0) {
              for (int i = 0; i < ntile; ++i) {
                issue_s(i, st);
                umma_commit(bar(kBarS + i));
              }
              if (nblk == 1) umma_commit(bar(kBarQFree));  // the item's last reads of Q
            }
            const bool more = j + 1 < nblk;
            // tile 0: PV of this block, then S of the next block
            if (!(ok = mbar_spin(bar(kBarP + 0), ph, a.status))) break;
            tc_fence_after();
            issue_pv(0, st, j > 0, 0);
            if (!(ok = mbar_spin(bar(kBarP + 1), ph, a.status))) break;
            tc_fence_after();
            issue_pv(0, st, j > 0, 4);
            if (more) {
              if (!(ok = mbar_wait(bar(kBarKvFull + (st ^ 1)), ((gb + 1) >> 1) & 1, a.status))) break;
              tc_fence_after();
              issue_s(0, st ^ 1);
              umma_commit(bar(kBarS + 0));
              if (ntile == 1 && j + 2 == nblk) umma_commit(bar(kBarQFree));
            }
            if (ntile == 2) {
              if (!(ok = mbar_spin(bar(kBarP + 2), ph, a.status))) break;
              tc_fence_after();
              issue_pv(1, st, j > 0, 0);
              if (!(ok = mbar_spin(bar(kBarP + 3), ph, a.status))) break;
              tc_fence_after();
              issue_pv(1, st, j > 0, 4);
            }
            umma_commit(bar(kBarKvEmpty + st));  // K/V stage free once these MMAs complete
            if (ntile == 2 && more) {
              issue_s(1, st ^ 1);
              umma_commit(bar(kBarS + 1));
              if (j + 2 == nblk) umma_commit(bar(kBarQFree));
            }
            if (*s_abort) { ok = false; break; }
          }
          if (!ok) *s_abort = 1;
          for (int i = 0; i < ntile; ++i) umma_commit(bar(kBarO + i));
          if (!ok) break;
          g += (uint32_t)nblk;
          item = read_item(pos, kt, am);
          if (item < 0 || *s_abort) break;
        }
      }
    }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ================================ softmax =====================================
    // Warpgroup i handles tile i; thread = query row r = TMEM lane.
    const int i = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    if (i < ntile) {
      const uint32_t tS = tmem + 256 * i + ((uint32_t)((warp & 3) * 32) << 16);  // S (and P)
      const uint32_t tO = tS + 128;
      const float sc = a.scale_log2;  // > 0, so max(s) * sc = max(s * sc)
      int item = blockIdx.x, kt, am;
      attn_item_load<GATHER>(a, item, ntile, false, kt, am);
      uint32_t g = 0;
      for (int pos = 0;; ++pos) {
        // only the block count and the diagonal block's position stay live
        // through the block loop (the loop is register-bound)
        int nblk, jdiag;
        {
          const AttnItem it = attn_item_of<GATHER>(a, item, ntile, kt, am);
          nblk = it.nblk;
          jdiag = GATHER ? it.n_gather : it.t;
        }
        float m_used = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
          const uint32_t gb = g + (uint32_t)j;
          if (!(ok = mbar_wait(bar(kBarS + i), gb & 1u, a.status)) || *s_abort) { ok = false; break; }
          tc_fence_after();
          const bool diag = j == jdiag;
          uint32_t mk[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
          if (GATHER && !diag) {
            // masks of the gathered rows (written before the stage's full barrier completed)
            if (!(ok = mbar_wait(bar(kBarKvFull + (gb & 1u)), (gb >> 1) & 1, a.status))) break;
#pragma unroll
            for (int e = 0; e < 4; ++e) mk[e] = masks[(gb & 1u) * 4 + e];
          }
          if (diag) {
            // causal diagonal block: key col is visible to row r if col <= r
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int n = r - 32 * c + 1;  // visible keys of this chunk
              mk[c] = n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : (1u << n) - 1u);
            }
          }
          uint32_t v[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, v[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) reg_fence32(v[c]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (mk[c] != 0xffffffffu) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (!((mk[c] >> e) & 1u)) v[c][e] = __float_as_uint(-INFINITY);
            }
          }
          // ---- row maximum of the raw scores
          float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2)
              mp[e2 & 3] = fmax3(mp[e2 & 3], __uint_as_float(v[c][2 * e2]), __uint_as_float(v[c][2 * e2 + 1]));
          const float mr = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
          const float mloc = mr == -INFINITY ? -INFINITY : mr * sc;
          float alpha = 1.f;
          bool rescale = false;
          if (m_used == -INFINITY) {
            m_used = mloc;  // first visible key of the row: O and l are still zero
          } else if (mloc > m_used + kRescaleLog2) {
            alpha = fast_exp2(m_used - mloc);
            m_used = mloc;
            rescale = true;
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // the previous PV of this tile completed before S of this block was committed
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * c, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + 32 * c, o);
            }
          }
          l_sum *= alpha;
          const float base = (m_used == -INFINITY) ? 0.f : m_used;
          // ---- p = exp2(s*sc - base), two scores per packed f32x2 FMA; P goes
          // back as bf16 pairs into columns 0..63 of the row's S (all read).
          uint64_t L[4] = {0ull, 0ull, 0ull, 0ull};
          const uint64_t SC = f2_pack(sc, sc), NB = f2_pack(-base, -base);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pw[16];
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(v[c][2 * e2]), __uint_as_float(v[c][2 * e2 + 1])), SC, NB),
                        x0, x1);
              const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              L[e2 & 3] = f2_add(L[e2 & 3], f2_pack(p0, p1));
              pw[e2] = pack_x2<F16>(p0, p1);
            }
            if (c == 2) {
              // keys 0..63 are stored: hand them to the MMA before the rest
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(kBarP + 2 * i));
            }
            tmem_st16(tS + 16 * c, pw);
          }
          float l0, l1, l2, l3;
          f2_unpack(f2_add(L[0], L[1]), l0, l1);
          f2_unpack(f2_add(L[2], L[3]), l2, l3);
          l_sum += (l0 + l1) + (l2 + l3);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarP + 2 * i + 1));  // one arrival per warp, 4 per tile
        }
        ok = __all_sync(0xffffffffu, ok && !*s_abort);
        if (!ok) *s_abort = 1;
        // ---- epilogue: O / l ------------------------------------------------------
        // Each warp stages its 32 rows, 64 columns at a time, in the 128-byte-
        // swizzled box layout and writes them with a TMA store (whole lines,
        // asynchronous); before refilling its buffer it waits until the previous
        // store has read it.  Only warp-level synchronisation is involved.
        const bool ep = __all_sync(0xffffffffu, mbar_wait(bar(kBarO + i), pos & 1, a.status) && ok && !*s_abort);
        if (ep) {
          tc_fence_after();
          const AttnItem it = attn_item_of<GATHER>(a, item, ntile, kt, am);
          const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
          const uint32_t stg = sbase + kAttnStage + (uint32_t)warp * kStageWarpBytes;  // warps 0-7
          const int y = (int)(it.q_row0 + (int64_t)i * a.N) + 32 * (warp & 3);
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * (2 * hh + c2), o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) {
                uint4 w;
                w.x = pack_x2<F16>(__uint_as_float(o[8 * q8 + 0]) * inv_l, __uint_as_float(o[8 * q8 + 1]) * inv_l);
                w.y = pack_x2<F16>(__uint_as_float(o[8 * q8 + 2]) * inv_l, __uint_as_float(o[8 * q8 + 3]) * inv_l);
                w.z = pack_x2<F16>(__uint_as_float(o[8 * q8 + 4]) * inv_l, __uint_as_float(o[8 * q8 + 5]) * inv_l);
                w.w = pack_x2<F16>(__uint_as_float(o[8 * q8 + 6]) * inv_l, __uint_as_float(o[8 * q8 + 7]) * inv_l);
                const uint32_t chunk = (uint32_t)(4 * c2 + q8) ^ (uint32_t)(lane & 7);
                sts128(stg + (uint32_t)lane * 128u + (chunk << 4), w);
              }
            }
            fence_proxy_async_smem();  // the TMA store reads the staged rows through the async proxy
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_o, stg, 64 * hh, y);
              bulk_commit();
            }
          }
          if (a.lse) a.lse[it.q_row0 + (int64_t)i * a.N + r] = l_sum > 0.f ? (m_used + __log2f(l_sum)) * kLn2 : -INFINITY;
        } else {
          ok = false;
        }
        if (!__all_sync(0xffffffffu, ok)) break;
        g += (uint32_t)nblk;
        int nx = -1;
        if (lane == 0) nx = read_item(pos, kt, am);
        nx = __shfl_sync(0xffffffffu, nx, 0);
        kt = __shfl_sync(0xffffffffu, kt, 0);
        am = __shfl_sync(0xffffffffu, am, 0);
        if (nx < 0) break;
        item = nx;
      }
      if (lane == 0) bulk_wait0();  // this warp's O stores have completed
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool F16>
__global__ void __launch_bounds__(kPoolThreads, 1)
prefill_pool_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const PoolArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* red = reinterpret_cast<float*>(smem + kPoolRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPoolMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kPoolMisc + 224);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kPoolMisc + 232);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1-D grid, longest tiles first over the whole grid (t >= 1)
  const int per_t = a.Hkv * a.B;
  const int t = a.n_tiles - 1 - (int)(blockIdx.x / per_t);
  const int h = (int)(blockIdx.x % per_t) % a.Hkv, b = (int)(blockIdx.x % per_t) / a.Hkv;
  const int G = a.G;
  const int kv_row0 = (int)(((int64_t)b * a.Hkv + h) * a.N);
  const int n_rounds = (G + kPoolHeads - 1) / kPoolHeads;
  const int nblk = t;  // key blocks before the tile, per round
  const int hg = G < kPoolHeads ? G : kPoolHeads;  // heads per round: 1, 2 or 4
  const int n_sub = hg >= 2 ? hg / 2 : 1;         // head pairs per round
  const int nwg = hg >= 2 ? 4 : 2;                // summing warpgroups in use

  if (tid == 0) {
    for (int i = 0; i < kPoolBars; ++i) {
      // buffer free: every warp of the summing warpgroups in use; exchange full:
      // the warps of warpgroups 1..; exchange empty: warpgroup 0's 4 warps
      uint32_t count = 1;
      if (i >= kPBarFree && i < kPBarFree + 2) count = 4u * nwg;
      if (i >= kPBarRedFull && i < kPBarRedFull + 2) count = 4u * (nwg - 1);
      if (i >= kPBarRedEmpty && i < kPBarRedEmpty + 2) count = 4u;
      mbar_init(bar(i), count);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  float* prow = a.pooled + (((int64_t)b * a.n_tiles + t) * a.Hkv + h) * a.N;
  const float inv_count = 1.f / (float)(kTile * G);
  // The extra K16 step: the K side once per CTA, the query side of a round's
  // heads from their log-sum-exp (every thread writes its share, then the CTA
  // synchronises; the tensor cores read these through the async proxy).
  for (int r = tid; r < kTile; r += kPoolThreads) {
    const uint32_t one = 0x3F80u;  // bf16 1.0
    *reinterpret_cast<uint4*>(smem + kPoolKx + sw32_chunk_offset(r, 0)) =
        make_uint4(one | (one << 16), one, 0u, 0u);
    *reinterpret_cast<uint4*>(smem + kPoolKx + sw32_chunk_offset(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
  }
  auto load_lse = [&](int hg, int gbase) {
    for (int e = tid; e < hg * kTile; e += kPoolThreads) {
      const int j = e / kTile, q = e % kTile;
      const float lse = a.lse[((int64_t)b * a.Hq + gbase + j) * a.N + (int64_t)kTile * t + q];
      const float nv = -lse * a.inv_scale;  // the MMA adds -v to q.k; x = scale log2(e) (q.k - v)
      const uint16_t hi = to_bf16_bits(nv);
      const float r1 = nv - __uint_as_float((uint32_t)hi << 16);
      const uint16_t mid = to_bf16_bits(r1);
      const uint16_t lo = to_bf16_bits(r1 - __uint_as_float((uint32_t)mid << 16));
      uint8_t* row = smem + kPoolQx + j * kXBytes;
      *reinterpret_cast<uint4*>(row + sw32_chunk_offset(q, 0)) =
          make_uint4((uint32_t)hi | ((uint32_t)mid << 16), (uint32_t)lo, 0u, 0u);
      *reinterpret_cast<uint4*>(row + sw32_chunk_offset(q, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    __syncthreads();
  };
  // Each role runs its own copy of the round loop, so the compiler sizes every
  // role's code for that role's register budget (setmaxnreg below).
  //
  // Within a round, the key blocks are the outer loop and the round's head
  // pairs ("sub-rounds") the inner one; sub-iteration it = (rd*nblk + jb)*n_sub
  // + sub computes S^T of one head pair into TMEM buffer it & 1 (columns
  // [256 (it&1), 256 (it&1) + 256): the pair's first head, then its second),
  // so the MMA fills one buffer while the summing warps work on the other.
  if (warp < 4) {
    setmaxnreg_dec<kPoolCtlRegs>();
    int q_loads = 0;             // warp 0 lane 0: query-tile loads issued (one kPBarQ phase each)
    int last_k0 = -1, last_k1 = -1;  // warp 0 lane 0: K-block counter of the last load into stage 0 / 1
    for (int rd = 0; rd < n_rounds; ++rd) {
      const int gbase = h * G + rd * kPoolHeads;
      const int kit0 = rd * nblk;  // running K-block counter (stage / phase bookkeeping)
      load_lse(hg, gbase);
      if (warp == 0) {
        // ---------------------------- TMA producer ----------------------------
        if (lane == 0) {
          ++q_loads;
          mbar_expect_tx(bar(kPBarQ), hg * kTileBytes);
          for (int j = 0; j < hg; ++j) {
            const int y = (int)(((int64_t)b * a.Hq + gbase + j) * a.N + (int64_t)kTile * t);
            tma_load_2d(sbase + kPoolQ + j * kHalfBytes, &tm_q, 0, y, bar(kPBarQ));
            tma_load_2d(sbase + kPoolQ + (kPoolHeads + j) * kHalfBytes, &tm_q, 64, y, bar(kPBarQ));
          }
          for (int jb = 0; jb < nblk; ++jb) {
            const int kit = kit0 + jb, st = kit & 1;
            if (kit >= 2 && !mbar_wait(bar(kPBarKEmpty + st), ((kit >> 1) - 1) & 1, a.status)) { *s_abort = 1; break; }
            if (*s_abort) break;
            const uint32_t ks = sbase + kPoolK + st * kTileBytes;
            mbar_expect_tx(bar(kPBarKFull + st), kTileBytes);
            if (st) last_k1 = kit; else last_k0 = kit;
            tma_load_2d(ks, &tm_k, 0, kv_row0 + kTile * jb, bar(kPBarKFull + st));
            tma_load_2d(ks + kHalfBytes, &tm_k, 64, kv_row0 + kTile * jb, bar(kPBarKFull + st));
          }
        }
      } else if (warp == 1) {
        // ---------------------------- MMA issuer ------------------------------
        // S^T = K [Q_g; Q_g+1]^T of each head pair (N = 256; a single head uses
        // N = 128) into buffer it & 1, once the summing warps freed it.
        if (lane == 0) {
          // Q and K in the data's type; the extra -lse step below is a separate
          // instruction with bf16 operands on both sides
          const uint32_t idesc = idesc_f16kind(128, hg >= 2 ? 256 : 128, false, false, F16);
          const uint32_t idesc_x = idesc_bf16(128, hg >= 2 ? 256 : 128, false, false);
          bool ok = mbar_wait(bar(kPBarQ), rd & 1, a.status);
          for (int jb = 0; ok && jb < nblk; ++jb) {
            const int kit = kit0 + jb, st = kit & 1;
            if (!(ok = mbar_wait(bar(kPBarKFull + st), (kit >> 1) & 1, a.status))) break;
            const uint64_t dk = kmajor_desc(sbase + kPoolK + st * kTileBytes, 0);
            for (int sub = 0; sub < n_sub; ++sub) {
              const int it = kit * n_sub + sub, buf = it & 1;
              if (it >= 2 && !(ok = mbar_spin(bar(kPBarFree + buf), ((it >> 1) - 1) & 1, a.status))) break;
              tc_fence_after();
              const uint64_t dq = kmajor_desc(sbase + kPoolQ + 2 * sub * kHalfBytes, 0);
#pragma unroll
              for (int k16 = 0; k16 < 8; ++k16)
                umma_ss(tmem + 256 * buf, dk + kmajor_step(k16), dq + qpair_step(k16), idesc, k16 > 0 ? 1u : 0u);
              umma_ss(tmem + 256 * buf, sw32_desc(sbase + kPoolKx), sw32_desc(sbase + kPoolQx + 2 * sub * kXBytes),
                      idesc_x, 1u);
              umma_commit(bar(kPBarS + buf));
            }
            if (!ok) break;
            umma_commit(bar(kPBarKEmpty + st));
            if (*s_abort) { ok = false; break; }
          }
          if (!ok) *s_abort = 1;
        }
      }
      __syncthreads();  // round done: Q tiles and the -lse tiles may be replaced
    }
    // after an abort, wait (bounded) for the copies the producer started: the
    // last query-tile load and the last K load into each stage
    if (warp == 0 && lane == 0 && *s_abort) {
      if (q_loads > 0) mbar_wait(bar(kPBarQ), (uint32_t)(q_loads - 1) & 1u, a.status);
      if (last_k0 >= 0) mbar_wait(bar(kPBarKFull + 0), ((uint32_t)last_k0 >> 1) & 1u, a.status);
      if (last_k1 >= 0) mbar_wait(bar(kPBarKFull + 1), ((uint32_t)last_k1 >> 1) & 1u, a.status);
    }
  } else {
    setmaxnreg_inc<kPoolSumRegs>();
    // ------------------- summing warpgroups ---------------------------------
    // Warpgroup w takes head (w >> 1) of each pair and query half (w & 1):
    // thread = key (TMEM lane) sums exp2(sc (q.k - lse/scale)) over 64 queries
    // of that head, read 16 at a time, one load ahead of the summing; the
    // buffer is released once the last columns are in registers.
    const int w = (warp >> 2) - 1;
    const int hl = w >> 1, qh = w & 1;
    const bool active = w < nwg;
    const int key = (warp & 3) * 32 + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint64_t SC = f2_pack(a.scale_log2, a.scale_log2);
    for (int rd = 0; rd < n_rounds; ++rd) {
      const int gbase = h * G + rd * kPoolHeads;
      const int kit0 = rd * nblk;
      load_lse(hg, gbase);
      float pend = 0.f;  // warpgroup 0: its own sum of the previous block
      // adds warpgroups 1.. of block kitp (block jbp of the round) to `mine`, writes pooled
      auto combine = [&](int rdp, int kitp, int jbp, float mine) -> bool {
        const int sl = kitp & 1;
        if (!mbar_wait(bar(kPBarRedFull + sl), (kitp >> 1) & 1, a.status)) {
          *s_abort = 1;
          return false;
        }
        const float* slot = red + sl * 3 * kTile;
        float tot = mine;
        for (int o = 0; o < nwg - 1; ++o) tot += slot[o * kTile + key];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kPBarRedEmpty + sl));
        const int col = kTile * jbp + key;
        if (rdp == 0) prow[col] = tot * inv_count;
        else prow[col] += tot * inv_count;
        return true;
      };
      for (int jb = 0; jb < nblk; ++jb) {
        const int kit = kit0 + jb;
        uint64_t A[4] = {0ull, 0ull, 0ull, 0ull};
        // sum over 16 queries of exp2(sc * (q.k - lse/scale)), two per packed
        // instruction; 2 of every 8 pairs on the FMA pipe, the rest on the SFU
        auto sum16 = [&](const uint32_t (&v)[16]) {
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) {
            float x0, x1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(v[2 * e2]), __uint_as_float(v[2 * e2 + 1])), SC), x0, x1);
            float p0, p1;
            if (e2 >= 6) {
              exp2_poly5_x2(x0, x1, p0, p1);
            } else {
              p0 = fast_exp2(x0);
              p1 = fast_exp2(x1);
            }
            A[e2 & 3] = f2_add(A[e2 & 3], f2_pack(p0, p1));
          }
        };
        bool ok = true;
        if (active) {
          for (int sub = 0; sub < n_sub; ++sub) {
            const int it = kit * n_sub + sub, buf = it & 1;
            if (!(ok = mbar_wait(bar(kPBarS + buf), (it >> 1) & 1, a.status)) || *s_abort) {
              ok = false;
              break;
            }
            tc_fence_after();
            // 64 scores in four loads of 16 columns, each in flight while the
            // previous ones are summed (a wait covers every earlier load; the
            // fence keeps the compiler from reading a register before it)
            const uint32_t tS = tmem + 256 * buf + 128 * hl + 64 * qh + lane_base;
            uint32_t v0[16], v1[16];
            tmem_ld16(tS, v0);
            tmem_wait_ld();
            reg_fence16(v0);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t (&cur)[16] = (c & 1) ? v1 : v0;
              uint32_t (&nxt)[16] = (c & 1) ? v0 : v1;
              if (c < 3) {
                tmem_ld16(tS + 16 * (c + 1), nxt);
              } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kPBarFree + buf));  // the buffer may be refilled
              }
              sum16(cur);
              if (c < 3) {
                tmem_wait_ld();
                reg_fence16(nxt);
              }
            }
          }
        }
        if (!ok) {
          *s_abort = 1;
          break;
        }
        float a0, a1, a2, a3;
        f2_unpack(f2_add(A[0], A[1]), a0, a1);
        f2_unpack(f2_add(A[2], A[3]), a2, a3);
        const float acc = (a0 + a1) + (a2 + a3);
        // Warpgroups 1.. hand their sums to warpgroup 0 through shared memory
        // (slot double-buffered by block parity, guarded by bounded mbarrier
        // waits).  Warpgroup 0 adds them one block late, while its own next
        // block is under way, so it never waits for the slowest one.
        if (w > 0) {
          if (active) {
            const int sl = kit & 1;
            if (kit >= 2 && !mbar_wait(bar(kPBarRedEmpty + sl), ((kit >> 1) - 1) & 1, a.status)) { *s_abort = 1; break; }
            red[(sl * 3 + w - 1) * kTile + key] = acc;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kPBarRedFull + sl));
          }
        } else {
          if (jb > 0 && !combine(rd, kit - 1, jb - 1, pend)) break;
          pend = acc;
        }
      }
      // warpgroup 0: the round's last block
      if (w == 0 && nblk > 0 && !*s_abort) combine(rd, kit0 + nblk - 1, nblk - 1, pend);
      __syncthreads();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host ----
// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised exactly once even when several host threads call at the same time).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// 2-D view [rows, 128] bf16, boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows, bool f16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_anchor_workspace_bytes(int, int, int, int) { return 0; }
size_t prefill_reuse_workspace_bytes(int, int, int, int, int) { return 0; }

static cudaError_t launch_attn(const PrefillParams& p, bool gather, cudaStream_t st) {
  const int n_tiles = p.N / kTile;
  const uint64_t kv_rows = (uint64_t)p.B * p.Hkv * p.N;
  if (kv_rows >= (1ull << 31) || (uint64_t)p.B * p.Hq * p.N >= (1ull << 31)) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv, to;
  if (!make_tile_map(&tq, p.q, (uint64_t)p.B * p.Hq * p.N, 128, p.f16) ||
      !make_tile_map(&tk, p.k, kv_rows, 128, p.f16) || !make_tile_map(&tv, p.v, kv_rows, 128, p.f16) ||
      !make_tile_map(&to, p.out, (uint64_t)p.B * p.Hq * p.N, 32, p.f16))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.G = p.G; a.N = p.N; a.n_tiles = n_tiles;
  a.k = p.k; a.v = p.v;
  a.idx = p.idx; a.idx_k = p.idx_k; a.head_map = p.head_map; a.k_max = p.k_max;
  a.head_major = !gather && kv_rows * (uint64_t)kHeadDim * 2u * 2u > (64ull << 20);
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.out = p.out; a.lse = p.lse; a.status = p.status;
  const int ntile = p.G >= 2 ? 2 : 1;
  const uint64_t n_ctas = (uint64_t)n_tiles * (uint64_t)(p.Hq / ntile) * (uint64_t)p.B;
  if (n_ctas >= (1ull << 31)) return cudaErrorNotSupported;
  dim3 grid((unsigned)n_ctas);
  // The kernel's setmaxnreg split assumes exactly kLaunchRegs registers per
  // thread at launch; with fewer, the softmax warpgroups' increase could never
  // be satisfied.  Refuse to launch a build that does not match.
  auto kern = gather ? (p.f16 ? prefill_attn_kernel<true, true> : prefill_attn_kernel<true, false>)
                     : (p.f16 ? prefill_attn_kernel<false, true> : prefill_attn_kernel<false, false>);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kAttnThreads, kAttnSmem, st>>>(tq, tk, tv, to, a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_anchor(const PrefillParams& p, cudaStream_t st) {
  cudaError_t e = launch_attn(p, false, st);
  if (e != cudaSuccess) return e;
  const int n_tiles = p.N / kTile;
  if (n_tiles < 2) return cudaSuccess;
  CUtensorMap tq, tk;
  if (!make_tile_map(&tq, p.q, (uint64_t)p.B * p.Hq * p.N, 128, p.f16) ||
      !make_tile_map(&tk, p.k, (uint64_t)p.B * p.Hkv * p.N, 128, p.f16))
    return cudaErrorInvalidValue;
  PoolArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.G = p.G; a.N = p.N; a.n_tiles = n_tiles;
  a.scale_log2 = (float)((double)p.scale * 1.4426950408889634);
  a.inv_scale = (float)(1.0 / (double)p.scale);
  a.lse = p.lse; a.pooled = p.pooled; a.status = p.status;
  auto pool = p.f16 ? prefill_pool_kernel<true> : prefill_pool_kernel<false>;
  cudaFuncAttributes fa;  // the setmaxnreg split assumes kPoolLaunchRegs at launch
  e = cudaFuncGetAttributes(&fa, pool);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kPoolLaunchRegs) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(pool, cudaFuncAttributeMaxDynamicSharedMemorySize, kPoolSmem);
  if (e != cudaSuccess) return e;
  const uint64_t n_pool = (uint64_t)(n_tiles - 1) * (uint64_t)p.Hkv * (uint64_t)p.B;
  if (n_pool >= (1ull << 31)) return cudaErrorNotSupported;
  pool<<<dim3((unsigned)n_pool), kPoolThreads, kPoolSmem, st>>>(tq, tk, a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_reuse(const PrefillParams& p, cudaStream_t st) {
  return launch_attn(p, true, st);
}

}  // namespace kascade
