// Tensor-core attention tiles on sm_100a (tcgen05 + TMEM + TMA), used by
// Phase 1 and by the Phase-2 query tokens.
//
// Phase 1 (hotaipapers.com page, Phase 1 paragraph; rebuttal to reviewer EMsM,
// "Size of Anchor Block"): block b_0 runs plain causal attention, every block
// b_i (i > 0) runs causal attention over [anchor = b_0 ; b_i] and keeps only its
// own rows. The anchor is never copied: a work item of block i first streams
// b_0's K/V tiles (all visible), then its own block's tiles up to the diagonal.
//
// Phase-2 query tokens (hotaipapers.com page, Phase 2 paragraph): every split
// (a chunk of one context block, or the query-local cache) returns a partial
// output and its LSE for all query rows; the merge kernel combines them.
//
// One CTA computes two 128-row Q tiles against the same sequence of 128-key K/V
// tiles, so every K/V tile loaded serves 256 rows:
//   Phase 1: the two tiles are two heads of one GQA group at the same block
//            rows (G >= 2), or two consecutive 128-row tiles of one head (G = 1;
//            the first tile then sees one fully masked extra K/V tile).
//   Query:   two consecutive tiles of packed rows, each 128/G query tokens x the
//            G heads of one kv-head; context splits see every key of their
//            chunk, the cache split is causal (query token j sees cache rows <= j).
// Work items are ordered so that the tiles of one block run together (their
// K/V and the anchor's stay in L2), blocks i > 0 before b_0, longer rows first.
//
// CTA = 3 warpgroups (12 warps; 5 with STAR_SOFTMAX_PARTS = 4):
//   warpgroup 0  warp 0: TMA producer (both Q tiles once, then K and V tiles
//                into 2-stage rings); warp 1: TMEM allocator and MMA issuer
//                (one thread); warps 2-3 idle. Registers trimmed to 104.
//   warpgroups 1, 2  the softmax, one thread per row (TMEM lane = row): each
//                takes one half (64 key columns) of both Q tiles' scores, tile 0
//                then tile 1 at every step, the halves of a row trading their
//                partial maxima through shared memory. Registers raised to 200.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256, 256+d), O_1 [256+d, 256+2d).
// MMA order (one thread): S_0(0), S_1(0), then for every K/V tile j
//   O_0 += P_0(j) V_j, S_0(j+1), O_1 += P_1(j) V_j, S_1(j+1),
// so the tensor core computes one tile's scores while the other tile's softmax
// runs. P_q(j) is written over S_q(j)'s columns as bf16 pairs and read by the
// MMA from TMEM. A commit after S_q(j+1) also covers O_q += P_q(j) V_j (a commit
// tracks every earlier MMA of the thread), so a softmax warp may rescale O_q as
// soon as it sees S_q(j+1). The running max is lazy: O is rescaled only when a
// row's max grows by more than 2^8; the final normalisation uses the same stale
// max, so the result is exact.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

// Softmax layout: the number of parts each tile's 128 key columns are split into.
// 1: warpgroup 1 takes Q tile 0 and warpgroup 2 Q tile 1, one thread per row with
// all 128 scores of a K/V tile. 2 or 4: each of 2 or 4 softmax warpgroups takes
// one part (64 or 32 columns) of both tiles' scores, the tiles in turn, so that
// all softmax warps of an SMSP work on the same tile and a tile's softmax takes
// less time; the parts of a row trade their partial maxima through shared memory.
#ifndef STAR_SOFTMAX_PARTS
#define STAR_SOFTMAX_PARTS 2
#endif
constexpr int kParts = STAR_SOFTMAX_PARTS;
static_assert(kParts == 1 || kParts == 2 || kParts == 4, "softmax parts: 1, 2 or 4");
constexpr int kSoftmaxWarpgroups = kParts == 4 ? 4 : 2;
constexpr int kThreads = 128 * (1 + kSoftmaxWarpgroups);
constexpr uint32_t kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle row each)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;          // lazy-rescale threshold (log2 units)
// Register split. Two softmax warpgroups: 384 threads launch with 168 registers
// (64512); warpgroup 0 gives back down to 104, the softmax warpgroups take 200.
// Four: 640 threads launch with 96 (61440); warpgroup 0 drops to 56 and the
// softmax warpgroups take 104.
constexpr int kLaunchRegs = kSoftmaxWarpgroups == 2 ? 168 : 96;
constexpr int kRegsLow = kSoftmaxWarpgroups == 2 ? 104 : 56;
constexpr int kRegsHigh = kSoftmaxWarpgroups == 2 ? 200 : 104;
static_assert(128 * kRegsLow + 128 * kSoftmaxWarpgroups * kRegsHigh <= kThreads * kLaunchRegs,
              "register split");
static_assert(kThreads * kLaunchRegs <= 65536, "register file");
// Of every 8 pairs of scores, this many take the FMA-pipe exponential; the MUFU
// (16 results per clock per SM) would otherwise pace the softmax at the same
// rate as the tensor core's MMAs.
#ifndef STAR_POLY_PAIRS
#define STAR_POLY_PAIRS 2
#endif
constexpr int kPolyPairs = STAR_POLY_PAIRS;

enum class Mode { kPhase1, kQuery };

struct AttnArgs {
  int32_t b, hq, hkv, G;
  int64_t L, B;
  float scale_log2;
  uint32_t* status;
  // Phase 1
  int32_t n_blocks, mt;   // blocks; 128-row q-tiles per block
  int32_t n_anchor;       // 128-column tiles covering the anchor b_0
  int32_t anchor_q;       // 1: the anchor tiles are scored with a second Q (map tk2)
  int32_t anchor_sep;     // 1: the anchor's K/V come from maps tk2/tv2 ([b, B, Hkv, d]) and
                          //    every block of this context is a block i > 0 (a host's share)
  __nv_bfloat16* o;       // [b, L, Hq, d]
  float* lse;             // [b, Hq, L] or null
  // Phase-2 query
  int64_t lq, chunk;
  int32_t spb, n_ctx, n_splits, n_qt;
  float* o_parts;    // [S, b, Lq, Hq, d]
  float* lse_parts;  // [S, b, Hq, Lq]
  // paged query-local cache (page_table == null: contiguous)
  const int32_t* page_table;  // [b, max_pages]
  int32_t page_size, max_pages;
  // Query pass of a uniform batch: the cache split reads the query tokens' K/V from
  // the inputs (maps tk2/tv2 over [b, Lq, Hkv, d]), and the cache append is done in
  // this kernel (cw_k == null: the cache was written before, the cache split reads it).
  const uint4* cw_k;  // [b, Lq, Hkv, d] as 16-byte words
  const uint4* cw_v;
  uint4* cw_kc;       // contiguous cache [b, cap, Hkv, d] or page pool [pages, P, Hkv, d]
  uint4* cw_vc;
  int64_t cw_cap;
  const int32_t* cw_table;  // [b, cw_max_pages] or null
  int32_t cw_page, cw_max_pages, cw_num_pages;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];  // per Q tile: S_q(j) (and every earlier MMA) complete
  uint64_t p_full[2];  // per Q tile: P_q(j) written to TMEM
  uint64_t o_bar[2];   // per Q tile: the last O_q += P V complete
  uint64_t drain;
  uint64_t q_free;     // the last anchor S MMAs are done: Q may be reloaded
  uint32_t tmem_base;
  int abort;
  float pmax[2][2][kParts][128];  // split columns: [tile][step parity][part][row] partial row maxima
  float psum[2][kParts][128];     // split columns: [tile][part][row] partial row sums at the end
};

// What one CTA computes.
struct Item {
  int bb, kvh;
  int n_tiles;
  int32_t qc1[2], qc2[2];  // Q tile coordinates: head (dim 1), token (dim 2)
  // Phase 1
  int h[2], rows_valid[2], n_anchor;
  int64_t bstart, t0[2];
  int64_t L, B;       // this sequence's length and block size
  int64_t tok_base;   // first token of this sequence in packed (varlen) tensors, else 0
  // query
  int split, tok0[2];
  bool cache;
  bool dual;           // both Q tiles hold the same rows; tile q takes K/V tiles 2j + q of the chunk
  int64_t k0, k1;
  int32_t lq;          // this sequence's query tokens
  int32_t q_c3;        // outer Q coordinate: the sequence, or 0 for packed queries
  int32_t ctx_tok, ctx_c3;  // context coordinates: packed offset and outer coordinate
  int64_t rbase;       // partial token-row of (this split, token 0)
};

template <Mode M>
__device__ __forceinline__ Item decode_item(const AttnArgs& a, const VarSeqs& vs) {
  Item it{};
  int64_t r = blockIdx.x;
  it.L = a.L;
  it.B = a.B;
  if constexpr (M == Mode::kPhase1) {
    int n_blocks = a.n_blocks, mt = a.mt, n_anchor = a.n_anchor;
    if (vs.n > 0) {
      // Varlen batch: the sequence whose work items hold this one (the last with
      // item0 <= r; empty sequences own no item), then its own block plan.
      int lo = 0, hi = vs.n;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (vs.item0[mid] <= r) lo = mid; else hi = mid;
      }
      r -= vs.item0[lo];
      it.tok_base = vs.start[lo];
      it.L = vs.start[lo + 1] - vs.start[lo];
      it.B = min(a.B, it.L);
      n_blocks = static_cast<int>((it.L + it.B - 1) / it.B);
      mt = static_cast<int>((it.B + 127) / 128);
      n_anchor = mt;
    }
    int i, m0, m1;
    if (a.G >= 2) {
      const int npair = a.G / 2;
      const int hp = static_cast<int>(r % npair);
      r /= npair;
      const int mp = static_cast<int>(r % mt);
      r /= mt;
      const int ip = static_cast<int>(r % n_blocks);
      r /= n_blocks;
      it.kvh = static_cast<int>(r % a.hkv);
      it.bb = static_cast<int>(r / a.hkv);
      i = (ip + 1) % n_blocks;  // blocks 1..n-1 first, b_0 (cheapest) last
      m0 = m1 = mt - 1 - mp;    // longest q-tiles first
      it.h[0] = it.kvh * a.G + 2 * hp;
      it.h[1] = it.h[0] + 1;
    } else {
      const int mt2 = (mt + 1) / 2;
      const int mp = static_cast<int>(r % mt2);
      r /= mt2;
      const int ip = static_cast<int>(r % n_blocks);
      r /= n_blocks;
      it.kvh = static_cast<int>(r % a.hkv);
      it.bb = static_cast<int>(r / a.hkv);
      i = (ip + 1) % n_blocks;
      m0 = 2 * (mt2 - 1 - mp);
      m1 = m0 + 1;
      it.h[0] = it.h[1] = it.kvh;
    }
    it.bstart = static_cast<int64_t>(i) * it.B;
    const int64_t bend = min(it.L, it.bstart + it.B);
    it.t0[0] = it.bstart + 128 * static_cast<int64_t>(m0);
    it.t0[1] = it.bstart + 128 * static_cast<int64_t>(m1);
#pragma unroll
    for (int q = 0; q < 2; ++q)
      it.rows_valid[q] = it.t0[q] >= bend ? 0 : static_cast<int>(bend - it.t0[q] < 128 ? bend - it.t0[q] : 128);
    const int m_last = it.rows_valid[1] > 0 ? m1 : m0;
    it.n_anchor = (i > 0 || a.anchor_sep) ? n_anchor : 0;
    it.n_tiles = it.rows_valid[0] > 0 ? it.n_anchor + m_last + 1 : 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      it.qc1[q] = it.h[q];
      it.qc2[q] = static_cast<int32_t>(it.tok_base + it.t0[q]);
    }
  } else {
    int n_qt = a.n_qt, n_splits = a.n_splits, n_ctx = a.n_ctx, spb = a.spb;
    int64_t chunk = a.chunk;
    it.lq = static_cast<int32_t>(a.lq);
    int32_t qbase = 0;
    int lo = 0;
    if (vs.n > 0) {
      // Varlen batch: the sequence that owns this item, then its own split plan
      // (packed queries and context; per-sequence caches).
      int hi = vs.n;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (vs.item0[mid] <= r) lo = mid; else hi = mid;
      }
      r -= vs.item0[lo];
      it.lq = vs.start[lo + 1] - vs.start[lo];
      qbase = vs.start[lo];
      it.L = vs.ctx0[lo + 1] - vs.ctx0[lo];
      it.B = min(a.B, it.L);
      spb = vs.spb[lo];
      n_ctx = it.L > 0 ? static_cast<int>((it.L + it.B - 1) / it.B) * spb : 0;
      n_splits = n_ctx + 1;
      chunk = it.L > 0 ? (it.B + spb - 1) / spb : 1;
      n_qt = (it.lq * a.G + 127) / 128;
    }
    const int npair = (n_qt + 1) / 2;
    const int qp = static_cast<int>(r % npair);
    r /= npair;
    it.split = static_cast<int>(r % n_splits);
    r /= n_splits;
    it.kvh = static_cast<int>(r % a.hkv);
    if (vs.n > 0) {
      it.bb = lo;
      it.q_c3 = 0;
      it.ctx_tok = vs.ctx0[lo];
      it.ctx_c3 = 0;
      it.rbase = static_cast<int64_t>(vs.rbase[lo]) + static_cast<int64_t>(it.split) * it.lq;
    } else {
      it.bb = static_cast<int>(r / a.hkv);
      it.q_c3 = it.bb;
      it.ctx_tok = 0;
      it.ctx_c3 = it.bb;
      it.rbase = (static_cast<int64_t>(it.split) * a.b + it.bb) * it.lq;
    }
    it.tok0[0] = 2 * qp * (128 / a.G);
    it.tok0[1] = it.tok0[0] + 128 / a.G;  // may lie past Lq: zero rows, never stored
    it.cache = it.split == n_ctx;
    if (!it.cache) {
      const int64_t blk = it.split / spb;
      const int64_t sub = it.split % spb;
      const int64_t bs = blk * it.B;
      const int64_t be = min(it.L, bs + it.B);
      it.k0 = min(be, bs + sub * chunk);
      it.k1 = min(be, it.k0 + chunk);
    } else {
      it.k0 = 0;
      it.k1 = it.lq;
    }
    const int n_kv = static_cast<int>((it.k1 - it.k0 + 127) / 128);
    // A context split whose second Q tile has no rows (all query rows fit one tile)
    // gives that tile the same rows and half of the chunk's K/V tiles: tile q takes
    // tiles 2j + q, so each step processes two K/V tiles for the one real Q tile and
    // the two partial softmaxes are combined in the epilogue. (Needs the column-part
    // layout, where each thread holds both tiles' state for its row.)
    it.dual = kParts > 1 && !it.cache && it.tok0[1] >= it.lq;
    if (it.dual) it.tok0[1] = it.tok0[0];
    it.n_tiles = it.dual ? (n_kv + 1) / 2 : n_kv;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      it.qc1[q] = it.kvh * a.G;
      it.qc2[q] = qbase + it.tok0[q];
    }
  }
  return it;
}

// Wait that also gives up when another role of the CTA has already given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Bars* bars,
                                              uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  volatile int* abort = &bars->abort;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitNs) {
      *abort = 1;
      report(status, kTimeoutFlag);
      return false;
    }
  }
}

template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Columns [0, limit) of K/V tile j are visible to a softmax row whose token is
// `tok` (Phase 1: absolute context position; query: query-token index).
template <Mode M>
__device__ __forceinline__ int visible_prefix(const Item& it, const AttnArgs& a, int64_t tok,
                                              int j, int q) {
  int64_t lim;
  if constexpr (M == Mode::kPhase1) {
    if (j < it.n_anchor) {
      lim = it.B - 128 * static_cast<int64_t>(j);  // the anchor ends at B
    } else {
      const int64_t kv0 = it.bstart + 128 * static_cast<int64_t>(j - it.n_anchor);
      lim = tok - kv0 + 1;  // causal inside the own block
    }
  } else {
    if (it.cache)
      lim = tok - 128 * static_cast<int64_t>(j) + 1;  // query token sees cache rows <= itself
    else
      lim = it.k1 - it.k0 - 128 * static_cast<int64_t>(it.dual ? 2 * j + q : j);  // end of the chunk
  }
  return lim < 0 ? 0 : (lim > 128 ? 128 : static_cast<int>(lim));
}

template <int D, Mode M>
__global__ void __launch_bounds__(kThreads, 1) attention_kernel(
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tk2,
    const __grid_constant__ CUtensorMap tv2, const AttnArgs a, const __grid_constant__ VarSeqs vs) {
  constexpr int CH = D / 64;
  constexpr uint32_t kTileBytes = CH * kChunkBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = base;                 // [2][kTileBytes]
  uint8_t* sk = sq + 2 * kTileBytes;  // [2][kTileBytes]
  uint8_t* sv = sk + 2 * kTileBytes;  // [2][kTileBytes]
  Bars* bars = reinterpret_cast<Bars*>(sv + 2 * kTileBytes);

  const Item it = decode_item<M>(a, vs);
  // Sizes of the buffers this CTA stores to (the debug build's index checks).
  // Phase 1: o [b, L, Hq, D] or [total, Hq, D], lse [b, Hq, L] or [Hq, total];
  // query: o_parts [rows, Hq, D], lse_parts [rows, Hq] with rows = all partial token-rows.
  const int64_t out_rows = M == Mode::kPhase1 ? (vs.n > 0 ? a.L : static_cast<int64_t>(a.b) * a.L)
                                              : (vs.n > 0 ? static_cast<int64_t>(vs.rbase[vs.n])
                                                          : static_cast<int64_t>(a.n_splits) * a.b * a.lq);
  if constexpr (M == Mode::kQuery) {
    // The query pass is launched programmatically: the merge that follows may be
    // scheduled now (it waits for this grid to finish). This kernel waits for the
    // previous one before it writes the partials (the previous kernel may be a merge
    // still reading them), appends to the cache (a decode step may still read it),
    // or, in the varlen pass, reads the cache rows its separate append just wrote.
    pdl_launch_dependents();
  }
  if (it.n_tiles == 0) {
    if constexpr (M == Mode::kQuery) {
      // A chunk past the end of a short last block: an empty partial.
      pdl_wait();
      for (int idx = threadIdx.x; idx < 256 * D; idx += kThreads) {
        const int row = idx / D, e = idx % D;
        const int tok = it.tok0[row >> 7] + (row & 127) / a.G;
        if (tok >= it.lq) continue;
        const int hq = it.kvh * a.G + (row & 127) % a.G;
        const int64_t oi = ((it.rbase + tok) * a.hq + hq) * D + e;
        if (STAR_IN_BOUNDS(a.status, oi, out_rows * a.hq * D)) a.o_parts[oi] = 0.f;
        const int64_t li = it.rbase * a.hq + static_cast<int64_t>(hq) * it.lq + tok;
        if (e == 0 && STAR_IN_BOUNDS(a.status, li, out_rows * a.hq)) a.lse_parts[li] = -INFINITY;
      }
    }
    return;  // before any barrier or TMEM allocation
  }
  const int n_tiles = it.n_tiles;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      // one arrival per softmax warp that holds a part of tile s: all of them when
      // the columns are split, tile s's own warpgroup otherwise
      mbar_init(&bars->p_full[s], 4 * (kParts > 1 ? kSoftmaxWarpgroups : 1));
      mbar_init(&bars->o_bar[s], 1);
    }
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->q_free, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (wg == 0) {
    setmaxnreg_dec<kRegsLow>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const CUtensorMap* mk = &tk;
      const CUtensorMap* mv = &tv;
      if constexpr (M == Mode::kQuery) {
        if (it.cache) {
          mk = &tk2;
          mv = &tv2;
        }
      }
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(mk);
      tma_prefetch_desc(mv);
      if constexpr (M == Mode::kPhase1) {
        if (a.anchor_sep) {
          tma_prefetch_desc(&tk2);
          tma_prefetch_desc(&tv2);
        }
      }
      if constexpr (M == Mode::kQuery) {
        // the cache rows this pass reads were just written by the previous kernel
        // (when they come from the inputs, nothing needs to wait)
        if (it.cache && a.cw_k == nullptr) pdl_wait();
      }
      // Anchor-position variant: the anchor tiles see Q rotated at the anchor
      // positions (map tk2); after them, Q is reloaded from tq for the own block.
      bool reload_q = false;
      const CUtensorMap* mq = &tq;
      if constexpr (M == Mode::kPhase1) {
        reload_q = a.anchor_q && it.n_anchor > 0;
        if (reload_q) mq = &tk2;
      }
      auto load_q = [&](const CUtensorMap* map) {
        mbar_arrive_expect_tx(&bars->q_full, 2 * kTileBytes);
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int c = 0; c < CH; ++c)
            tma_load_4d(sq + q * kTileBytes + c * kChunkBytes, map, &bars->q_full, c * 64,
                        it.qc1[q], it.qc2[q], M == Mode::kQuery ? it.q_c3 : it.bb);
      };
      load_q(mq);
      int q_loads = 1;
      int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};
      // Tile j goes to ring stage j & 1 (dual: stage q holds Q tile q's K/V tiles).
      const int n_loads = it.dual ? 2 * n_tiles : n_tiles;
      for (int j = 0; j < n_loads; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        int32_t kv0;
        const CUtensorMap* tkm = mk;
        const CUtensorMap* tvm = mv;
        if constexpr (M == Mode::kPhase1) {
          kv0 = static_cast<int32_t>(it.tok_base) +
                (j < it.n_anchor ? j * 128 : static_cast<int32_t>(it.bstart + 128 * (j - it.n_anchor)));
          if (a.anchor_sep && j < it.n_anchor) {  // the anchor's own buffer, rows [0, B)
            kv0 = j * 128;
            tkm = &tk2;
            tvm = &tv2;
          }
        } else {
          kv0 = static_cast<int32_t>(it.k0 + 128 * j);
        }
        // Outer TMA coordinate: the sequence, or for a paged cache the page holding
        // this 128-row tile (page sizes are multiples of 128).
        int32_t c3 = it.bb;
        if constexpr (M == Mode::kQuery) {
          if (!it.cache) {
            kv0 += it.ctx_tok;
            c3 = it.ctx_c3;
          } else if (a.page_table) {
            c3 = a.page_table[static_cast<int64_t>(it.bb) * a.max_pages + kv0 / a.page_size];
            kv0 %= a.page_size;
          }
        }
        if (j >= 2 && !wait_or_abort(&bars->k_empty[s], ph ^ 1, bars, a.status)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], kTileBytes);
#pragma unroll
        for (int c = 0; c < CH; ++c)
          tma_load_4d(sk + s * kTileBytes + c * kChunkBytes, tkm, &bars->k_full[s], c * 64, it.kvh, kv0, c3);
        last_k[s] = j;
        if (j >= 2 && !wait_or_abort(&bars->v_empty[s], ph ^ 1, bars, a.status)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], kTileBytes);
#pragma unroll
        for (int c = 0; c < CH; ++c)
          tma_load_4d(sv + s * kTileBytes + c * kChunkBytes, tvm, &bars->v_full[s], c * 64, it.kvh, kv0, c3);
        last_v[s] = j;
        if (reload_q && j == it.n_anchor) {
          if (!wait_or_abort(&bars->q_free, 0, bars, a.status)) break;
          load_q(&tq);
          q_loads = 2;
        }
      }
      // Every copy this thread issued has landed before the CTA may exit (on the
      // normal path these phases completed long ago).
      mbar_wait(&bars->q_full, (q_loads - 1) & 1, a.status);
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (last_k[s] >= 0) mbar_wait(&bars->k_full[s], (last_k[s] >> 1) & 1, a.status);
        if (last_v[s] >= 0) mbar_wait(&bars->v_full[s], (last_v[s] >> 1) & 1, a.status);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t kIdescQK = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescPV = make_idesc_bf16(128, D, false, true);
      const uint32_t sq_addr = smem_u32(sq);
      const uint32_t sk_addr = smem_u32(sk);
      const uint32_t sv_addr = smem_u32(sv);
      // Shared-memory descriptors of every tile this thread addresses, built once: a
      // step's descriptor is its tile's plus the step's offset in 16-byte units (the
      // address field cannot carry out: shared addresses stay below 256 KB). The
      // thread shares its SMSP with two busy softmax warps, so every instruction it
      // saves between MMAs shortens the hand-off.
      constexpr uint32_t kDescHi = sdesc_hi(1024);
      const uint32_t qd0 = sdesc_lo(sq_addr, 16), qd1 = sdesc_lo(sq_addr + kTileBytes, 16);
      const uint32_t kd0 = sdesc_lo(sk_addr, 16), kd1 = sdesc_lo(sk_addr + kTileBytes, 16);
      const uint32_t vd0 = sdesc_lo(sv_addr, kChunkBytes), vd1 = sdesc_lo(sv_addr + kTileBytes, kChunkBytes);
      // S_q = Q_q K_j^T: A = Q, B = K, both K-major 128-byte swizzled (16 columns = 32 bytes a step).
      bool reload_q = false;
      if constexpr (M == Mode::kPhase1) reload_q = a.anchor_q && it.n_anchor > 0;
      auto issue_s = [&](int q, int j) {
        const uint32_t qd = q ? qd1 : qd0;
        const uint32_t kd = (it.dual ? q : (j & 1)) ? kd1 : kd0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4;
          tc_mma_ss_lo(tmem + q * 128, qd + off16, kd + off16, kDescHi, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars->s_full[q]);
        if (reload_q && q == 1 && j == it.n_anchor - 1) tc_commit(&bars->q_free);
      };
      // O_q += P_q V_j: P from TMEM (bf16 pairs over S_q's columns); V MN-major
      // (d contiguous): 16 kv rows a step, the next 64 columns of d one chunk (LBO)
      // away, the next 8 kv rows 1024 B (SBO) away.
      auto issue_pv = [&](int q, int j) {
        const uint32_t vd = (it.dual ? q : (j & 1)) ? vd1 : vd0;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          tc_mma_ts_lo(tmem + 256 + q * D, tmem + q * 128 + kk * 8, vd + kk * (2048 >> 4), kDescHi,
                       kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok;
      if (it.dual) {
        // Both Q tiles hold the same rows; Q tile q's K/V tiles (2j + q) sit in ring
        // stage q, round j: S_q and PV_q each free their own stage.
        ok = wait_or_abort(&bars->q_full, 0, bars, a.status);
        for (int q = 0; ok && q < 2; ++q) {
          ok = wait_or_abort(&bars->k_full[q], 0, bars, a.status);
          if (!ok) break;
          tc_fence_after();
          issue_s(q, 0);
          tc_commit(&bars->k_empty[q]);
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const bool more = j + 1 < n_tiles;
          for (int q = 0; ok && q < 2; ++q) {
            ok = wait_or_abort(&bars->v_full[q], j & 1, bars, a.status) &&
                 wait_or_abort(&bars->p_full[q], j & 1, bars, a.status);
            if (!ok) break;
            tc_fence_after();
            issue_pv(q, j);
            tc_commit(&bars->v_empty[q]);
            if (!more) tc_commit(&bars->o_bar[q]);
            if (more) {
              ok = wait_or_abort(&bars->k_full[q], (j + 1) & 1, bars, a.status);
              if (!ok) break;
              tc_fence_after();
              issue_s(q, j + 1);
              tc_commit(&bars->k_empty[q]);
            }
          }
        }
      } else {
        ok = wait_or_abort(&bars->q_full, 0, bars, a.status) &&
             wait_or_abort(&bars->k_full[0], 0, bars, a.status);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          issue_s(1, 0);
          tc_commit(&bars->k_empty[0]);
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int s = j & 1;
          const bool more = j + 1 < n_tiles;
          ok = wait_or_abort(&bars->v_full[s], (j >> 1) & 1, bars, a.status) &&
               wait_or_abort(&bars->p_full[0], j & 1, bars, a.status);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, j);
          if (!more) tc_commit(&bars->o_bar[0]);
          if (more) {
            ok = wait_or_abort(&bars->k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, bars, a.status);
            // the first own-block tile needs the reloaded Q
            if (ok && reload_q && j + 1 == it.n_anchor) ok = wait_or_abort(&bars->q_full, 1, bars, a.status);
            if (!ok) break;
            tc_fence_after();
            issue_s(0, j + 1);
          }
          ok = wait_or_abort(&bars->p_full[1], j & 1, bars, a.status);
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, j);
          tc_commit(&bars->v_empty[s]);
          if (!more) tc_commit(&bars->o_bar[1]);
          if (more) {
            issue_s(1, j + 1);
            tc_commit(&bars->k_empty[(j + 1) & 1]);
          }
        }
      }
      // Every MMA this thread issued has completed before TMEM is released.
      tc_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, a.status);
    } else if (warp >= 2) {
      if constexpr (M == Mode::kQuery) {
        // ------------------------------------------------------------ cache append
        // The cache split's CTA of the first q-tile pair appends its (sequence,
        // kv-head)'s query K/V rows to the query-local cache: rows [0, Lq), and for
        // a paged cache zeros up to the end of the last page (later tiles read
        // those rows). It waits for the previous kernel, which may still read the
        // cache. A page id outside the pool is refused (bounds flag, no write).
        if (a.cw_k != nullptr && it.cache && it.tok0[0] == 0) {
          pdl_wait();
          constexpr int W = D / 8;  // 16-byte words of one row of one kv-head
          const int64_t lq = it.lq;
          const int64_t ext = a.cw_table ? (lq + a.cw_page - 1) / a.cw_page * a.cw_page : lq;
          const int64_t cache_rows = a.cw_table ? static_cast<int64_t>(a.cw_num_pages) * a.cw_page
                                                : static_cast<int64_t>(a.b) * a.cw_cap;
          for (int64_t i = (warp - 2) * 32 + lane; i < ext * W; i += 64) {
            const int64_t r = i / W;
            const int e = static_cast<int>(i % W);
            int64_t drow = static_cast<int64_t>(it.bb) * a.cw_cap + r;
            if (a.cw_table) {
              const int64_t page = a.cw_table[static_cast<int64_t>(it.bb) * a.cw_max_pages + r / a.cw_page];
              if (page < 0 || page >= a.cw_num_pages) {
                report(a.status, kBoundsFlag);
                continue;
              }
              drow = page * a.cw_page + r % a.cw_page;
            }
            if (!STAR_IN_BOUNDS(a.status, drow, cache_rows)) continue;
            const int64_t dst = (drow * a.hkv + it.kvh) * W + e;
            if (r < lq) {
              const int64_t src = ((static_cast<int64_t>(it.bb) * lq + r) * a.hkv + it.kvh) * W + e;
              a.cw_kc[dst] = a.cw_k[src];
              a.cw_vc[dst] = a.cw_v[src];
            } else {
              a.cw_kc[dst] = make_uint4(0u, 0u, 0u, 0u);
              a.cw_vc[dst] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    setmaxnreg_inc<kRegsHigh>();
    const int sw = wg - 1;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    // Layout: with the columns split (kParts > 1), warpgroup sw takes columns
    // [sw * 128 / kParts, (sw + 1) * 128 / kParts) of both Q tiles' scores (and D /
    // kParts output columns), the tiles in turn; with kParts = 1 warpgroup sw owns
    // Q tile sw whole.
    constexpr int kCols = 128 / kParts;         // scores per thread and tile
    constexpr int kChunks = kCols / 32;         // 32-column pieces of them
    constexpr int kOCols = D / kParts;          // output columns per thread
    constexpr int kOP = kOCols < 32 ? kOCols : 32;  // output columns per TMEM access
    constexpr int kTilesPerWarp = kParts > 1 ? 2 : 1;
    const int part = kParts > 1 ? sw : 0;
    const float sl2 = a.scale_log2;
    // This row's token and head in each of the warp's tiles (selected, so that Item
    // stays in registers). Phase 1: context position; query: query-token index.
    int64_t row_tok[kTilesPerWarp];
    int head[kTilesPerWarp], rows_valid[kTilesPerWarp];
#pragma unroll
    for (int i = 0; i < kTilesPerWarp; ++i) {
      const int q = kParts > 1 ? i : sw;
      if constexpr (M == Mode::kPhase1) {
        row_tok[i] = (q ? it.t0[1] : it.t0[0]) + row;
        head[i] = q ? it.h[1] : it.h[0];
        rows_valid[i] = q ? it.rows_valid[1] : it.rows_valid[0];
      } else {
        row_tok[i] = (q ? it.tok0[1] : it.tok0[0]) + row / a.G;
        head[i] = it.kvh * a.G + row % a.G;
        rows_valid[i] = 0;
      }
    }
    // K/V tiles [0, full_upto) are visible in full to every row of this warp, so
    // they need no mask and no visibility test. Phase 1: the anchor tiles when B is
    // a multiple of 128, then the own block's tiles wholly below the warp's first
    // row (row tiles start at multiples of 128 from the block start). Otherwise,
    // and for the query pass, every tile is tested.
    int full_upto = 0;
    if constexpr (M == Mode::kPhase1) {
      if (it.B % 128 == 0) {
        const int64_t first = (it.t0[0] < it.t0[1] ? it.t0[0] : it.t0[1]) + q4 * 32 - it.bstart;
        full_upto = it.n_anchor + static_cast<int>((first + 1) / 128);
      }
    }
    float m_run[kTilesPerWarp], l_run[kTilesPerWarp];
#pragma unroll
    for (int i = 0; i < kTilesPerWarp; ++i) {
      m_run[i] = -INFINITY;
      l_run[i] = 0.f;
    }
    // The kParts warps holding the parts of the same 32 rows meet on named barrier
    // 1 + q4. All of them take every barrier of the loop even after a wait has given
    // up, so none can be left waiting for another.
    auto parts_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + q4), "n"(32 * kParts) : "memory"); };
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
#pragma unroll
      for (int i = 0; i < kTilesPerWarp; ++i) {
        const int q = kParts > 1 ? i : sw;
        const uint32_t s_col = q * 128 + part * kCols;      // this thread's scores
        const uint32_t p_col = q * 128 + part * kCols / 2;  // its bf16 pairs of P
        const uint32_t o_col = 256 + q * D + part * kOCols;
        // Waits are per thread; the tcgen05 loads/stores below are warp-wide, so
        // the warp proceeds only if every lane's wait succeeded.
        if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(&bars->s_full[q], j & 1, bars, a.status));
        uint32_t sr[kChunks][32];
        float mt = -INFINITY;
        if (ok) {
          tc_fence_after();
          // Most tiles are fully visible: mask only when some row of the warp needs it.
          int limit = kCols;
          bool masked = false;
          if (j >= full_upto) {
            limit = visible_prefix<M>(it, a, row_tok[i], j, q) - part * kCols;  // in this part
            masked = __any_sync(0xffffffffu, limit < kCols);
          }
          // S in pieces of 32: the max over the first pieces overlaps the TMEM read of
          // the later ones. Row max with independent 3-input max chains.
          float mc[kChunks];
          tmem_ld32(lane_addr + s_col, sr[0]);
          if constexpr (kChunks >= 2) tmem_ld32(lane_addr + s_col + 32, sr[1 % kChunks]);
          tmem_wait_ld();
          if constexpr (kChunks == 4) {
            tmem_ld32(lane_addr + s_col + 64, sr[2 % kChunks]);
            tmem_ld32(lane_addr + s_col + 96, sr[3 % kChunks]);
          }
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            if (c == 2) tmem_wait_ld();
            if (masked) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e >= limit) sr[c][e] = __float_as_uint(-INFINITY);
            }
            mc[c] = fmaxf(__uint_as_float(sr[c][0]), __uint_as_float(sr[c][1]));
#pragma unroll
            for (int e = 2; e < 32; e += 2)
              mc[c] = fmax3(mc[c], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
          }
          mt = mc[0];
#pragma unroll
          for (int c = 1; c < kChunks; ++c) mt = fmaxf(mt, mc[c]);
        }
        if constexpr (kParts > 1) {
          // Trade partial maxima with the other parts of the row. Every part has its
          // scores in registers before any passes the barrier, so P (which the parts
          // write over S's first 64 columns) cannot overwrite unread scores.
          bars->pmax[q][j & 1][part][row] = mt;
          parts_sync();
#pragma unroll
          for (int o = 1; o < kParts; ++o) mt = fmaxf(mt, bars->pmax[q][j & 1][(part + o) % kParts][row]);
        }
        if (!ok) continue;
        const bool need = (m_run[i] == -INFINITY) || ((mt - m_run[i]) * sl2 > kRescaleLog2);
        const float m_new = need ? mt : m_run[i];
        const float m_use = m_new == -INFINITY ? 0.f : m_new;  // a row with nothing visible yet
        const float alpha = need ? ex2_approx((m_run[i] - m_use) * sl2) : 1.f;
        m_run[i] = m_new;
        const float ms = m_use * sl2;
        // p = 2^(s * scale * log2(e) - m'), two lanes per packed fp32 FMA / add.
        const float2 sl2v = make_float2(sl2, sl2);
        const float2 nms = make_float2(-ms, -ms);
        float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          // Chunk c (32 scores) -> 16 bf16 pairs, stored to TMEM at once (S is all
          // in registers already), so few P words are ever live.
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])),
                                   sl2v, nms);
            float p0, p1;
            if (((e >> 1) & 7) < kPolyPairs) {
              // a share of the exponentials on the FMA pipe, the rest on the MUFU
              const float2 pp = exp2_poly2(x);
              p0 = pp.x;
              p1 = pp.y;
            } else {
              p0 = ex2_approx(x.x);
              p1 = ex2_approx(x.y);
            }
            ps[(e >> 1) & 1] = fadd2(ps[(e >> 1) & 1], make_float2(p0, p1));
            pk[e / 2] = pack_bf16x2(p0, p1);
          }
          tmem_st16(lane_addr + p_col + c * 16, pk);
        }
        const float psum = (ps[0].x + ps[0].y) + (ps[1].x + ps[1].y);
        l_run[i] = l_run[i] * alpha + psum;
        // S_q(j) complete implies O_q += P_q(j-1) V complete: O may be rescaled now.
        if (j >= 1 && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < kOCols / kOP; ++c) {
            if constexpr (kOP == 32) {
              uint32_t ob[32];
              tmem_ld32(lane_addr + o_col + c * 32, ob);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * alpha);
              tmem_st32(lane_addr + o_col + c * 32, ob);
            } else {
              uint32_t ob[16];
              tmem_ld16(lane_addr + o_col + c * 16, ob);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * alpha);
              tmem_st16(lane_addr + o_col + c * 16, ob);
            }
          }
        }
        // Every lane's P (and O rescale) stores are complete; one lane per warp tells
        // the MMA thread (32x fewer arrivals on the barrier than one per thread).
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[q]);
      }
    }
    if constexpr (kParts > 1) {
      // The row sum is the parts' sums (same running max in all of them).
#pragma unroll
      for (int i = 0; i < kTilesPerWarp; ++i) bars->psum[i][part][row] = l_run[i];
      parts_sync();
#pragma unroll
      for (int i = 0; i < kTilesPerWarp; ++i)
#pragma unroll
        for (int o = 1; o < kParts; ++o) l_run[i] += bars->psum[i][(part + o) % kParts][row];
    }
    bool dual = false;
    if constexpr (M == Mode::kQuery && kParts > 1) dual = it.dual;
    if (dual) {
      // Both tiles hold this row over disjoint halves of the chunk's keys: combine
      // the two partial softmaxes exactly (the Phase-2 merge within one CTA) and
      // store one partial.
#pragma unroll
      for (int q = 0; q < 2; ++q)
        if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(&bars->o_bar[q], 0, bars, a.status));
      tc_fence_after();
      if (ok) {
        pdl_wait();  // the partials may still be read by the previous kernel
        const float M2 = fmaxf(m_run[0], m_run[kTilesPerWarp - 1]);
        float wq[2];
#pragma unroll
        for (int q = 0; q < 2; ++q)
          wq[q] = (M2 == -INFINITY || m_run[q % kTilesPerWarp] == -INFINITY)
                      ? 0.f : ex2_approx((m_run[q % kTilesPerWarp] - M2) * sl2);
        const float l = l_run[0] * wq[0] + l_run[kTilesPerWarp - 1] * wq[1];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse2 = l > 0.f ? M2 * sl2 + log2f(l) : -INFINITY;
        const int tok = static_cast<int>(row_tok[0]);
        const int hq = head[0];
        const int64_t o_off = ((it.rbase + tok) * a.hq + hq) * D + part * kOCols;
        const bool valid = tok < it.lq && STAR_IN_BOUNDS(a.status, o_off + kOCols - 1, out_rows * a.hq * D);
        float* dst = a.o_parts + o_off;
#pragma unroll
        for (int c = 0; c < kOCols / kOP; ++c) {
          uint32_t o0[kOP], o1[kOP];
          if constexpr (kOP == 32) {
            tmem_ld32(lane_addr + 256 + part * kOCols + c * 32, o0);
            tmem_ld32(lane_addr + 256 + D + part * kOCols + c * 32, o1);
          } else {
            tmem_ld16(lane_addr + 256 + part * kOCols + c * 16, o0);
            tmem_ld16(lane_addr + 256 + D + part * kOCols + c * 16, o1);
          }
          tmem_wait_ld();
          float v[kOP];
#pragma unroll
          for (int e = 0; e < kOP; ++e)
            v[e] = (__uint_as_float(o0[e]) * wq[0] + __uint_as_float(o1[e]) * wq[1]) * inv;
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * kOP);
#pragma unroll
            for (int u = 0; u < kOP / 4; ++u) d4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          }
        }
        const int64_t l_off = it.rbase * a.hq + static_cast<int64_t>(hq) * it.lq + tok;
        if (valid && part == 0 && STAR_IN_BOUNDS(a.status, l_off, out_rows * a.hq))
          a.lse_parts[l_off] = lse2 * 0.69314718055994531f;
      }
    }
#pragma unroll
    for (int i = 0; i < kTilesPerWarp; ++i) {
      if (dual) break;
      const int q = kParts > 1 ? i : sw;
      const uint32_t o_col = 256 + q * D + part * kOCols;
      if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(&bars->o_bar[q], 0, bars, a.status));
      tc_fence_after();
      if (!ok) continue;
      if constexpr (M == Mode::kQuery) pdl_wait();  // the partials may still be read by the previous kernel
      const bool has = l_run[i] > 0.f;
      const float inv = has ? 1.f / l_run[i] : 0.f;
      const float lse2 = has ? m_run[i] * sl2 + log2f(l_run[i]) : -INFINITY;
      // This thread's kOCols output columns, kOP at a time from TMEM, scaled by 1/l.
      auto load_scaled = [&](int c, float (&v)[kOP]) {
        uint32_t ob[kOP];
        if constexpr (kOP == 32) tmem_ld32(lane_addr + o_col + c * 32, ob);
        else tmem_ld16(lane_addr + o_col + c * 16, ob);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < kOP; ++e) v[e] = __uint_as_float(ob[e]) * inv;
      };
      if constexpr (M == Mode::kPhase1) {
        const int64_t t = row_tok[i];
        // uniform: row bb * L + t of [b, L, Hq, d]; varlen: row tok_base + t of [total, Hq, d]
        const int64_t o_off = ((static_cast<int64_t>(it.bb) * a.L + it.tok_base + t) * a.hq + head[i]) * D +
                              part * kOCols;
        const bool valid = row < rows_valid[i] &&
                           STAR_IN_BOUNDS(a.status, o_off + kOCols - 1, out_rows * a.hq * D);
        __nv_bfloat16* dst = a.o + o_off;
#pragma unroll
        for (int c = 0; c < kOCols / kOP; ++c) {
          float v[kOP];
          load_scaled(c, v);
          uint32_t w[kOP / 2];
#pragma unroll
          for (int e = 0; e < kOP / 2; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * kOP);
#pragma unroll
            for (int u = 0; u < kOP / 8; ++u)
              d4[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
          }
        }
        const int64_t l_off = (static_cast<int64_t>(it.bb) * a.hq + head[i]) * a.L + it.tok_base + t;
        if (a.lse && valid && part == 0 &&
            STAR_IN_BOUNDS(a.status, l_off, (vs.n > 0 ? 1 : static_cast<int64_t>(a.b)) * a.hq * a.L))
          a.lse[l_off] = lse2 * 0.69314718055994531f;
      } else {
        const int tok = static_cast<int>(row_tok[i]);
        const int hq = head[i];
        const int64_t o_off = ((it.rbase + tok) * a.hq + hq) * D + part * kOCols;
        const bool valid = tok < it.lq && STAR_IN_BOUNDS(a.status, o_off + kOCols - 1, out_rows * a.hq * D);
        float* dst = a.o_parts + o_off;
#pragma unroll
        for (int c = 0; c < kOCols / kOP; ++c) {
          float v[kOP];
          load_scaled(c, v);
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * kOP);
#pragma unroll
            for (int u = 0; u < kOP / 4; ++u) d4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          }
        }
        const int64_t l_off = it.rbase * a.hq + static_cast<int64_t>(hq) * it.lq + tok;
        if (valid && part == 0 && STAR_IN_BOUNDS(a.status, l_off, out_rows * a.hq))
          a.lse_parts[l_off] = lse2 * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

AttnArgs base_args(const Shape& s) {
  AttnArgs a{};
  a.b = s.b;
  a.hq = s.hq;
  a.hkv = s.hkv;
  a.G = s.group();
  a.L = s.L;
  a.B = s.B;
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.status = device_status_word();
  return a;
}

template <int D, Mode M>
cudaError_t launch(const AttnArgs& a, const CUtensorMap (&m)[5], int64_t items, const VarSeqs& vs,
                   cudaStream_t st) {
  constexpr uint32_t kTileBytes = (D / 64) * kChunkBytes;
  // 6 tiles (2 Q, 2 K, 2 V) + barriers + alignment slack; at least 120 KB so that
  // only one CTA (and one 512-column TMEM allocation) lives on an SM.
  size_t smem = 6 * kTileBytes + sizeof(Bars) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  auto kern = attention_kernel<D, M>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (items <= 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  if constexpr (M == Mode::kQuery) {
    e = launch_programmatic(kern, dim3(static_cast<unsigned>(items)), dim3(kThreads), smem, st, m[0],
                            m[1], m[2], m[3], m[4], a, vs);
    if (e != cudaSuccess) return e;
  } else {
    kern<<<static_cast<unsigned>(items), kThreads, smem, st>>>(m[0], m[1], m[2], m[3], m[4], a, vs);
  }
  count_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_phase1_t(const Shape& s, const void* q, const void* k, const void* v, void* o,
                            float* lse, cudaStream_t st) {
  alignas(64) CUtensorMap m[5];
  if (!encode_tma_bf16_4d(&m[0], q, D, s.hq, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[1], k, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[2], v, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true))
    return cudaErrorInvalidValue;
  m[3] = m[1];
  m[4] = m[2];
  AttnArgs a = base_args(s);
  a.n_blocks = static_cast<int32_t>(s.n_blocks());
  a.mt = static_cast<int32_t>((s.B + 127) / 128);
  a.n_anchor = a.mt;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  const int64_t pairs_per_block = a.G >= 2 ? static_cast<int64_t>(a.mt) * (a.G / 2) : (a.mt + 1) / 2;
  const int64_t items = static_cast<int64_t>(s.b) * s.hkv * a.n_blocks * pairs_per_block;
  VarSeqs vs;
  vs.n = 0;
  return launch<D, Mode::kPhase1>(a, m, items, vs, st);
}

template <int D>
cudaError_t launch_phase1_anchor_q_t(const Shape& s, const void* q, const void* qa, const void* k,
                                     const void* v, void* o, float* lse, cudaStream_t st) {
  alignas(64) CUtensorMap m[5];
  if (!encode_tma_bf16_4d(&m[0], q, D, s.hq, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[1], k, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[2], v, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[3], qa, D, s.hq, s.L, s.L, s.b, 64, 1, 128, true))
    return cudaErrorInvalidValue;
  m[4] = m[2];
  AttnArgs a = base_args(s);
  a.n_blocks = static_cast<int32_t>(s.n_blocks());
  a.mt = static_cast<int32_t>((s.B + 127) / 128);
  a.n_anchor = a.mt;
  a.anchor_q = 1;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  const int64_t pairs_per_block = a.G >= 2 ? static_cast<int64_t>(a.mt) * (a.G / 2) : (a.mt + 1) / 2;
  const int64_t items = static_cast<int64_t>(s.b) * s.hkv * a.n_blocks * pairs_per_block;
  VarSeqs vs;
  vs.n = 0;
  return launch<D, Mode::kPhase1>(a, m, items, vs, st);
}

// A host's share of Phase 1 in the multi-host form: the context holds blocks
// b_i .. b_k (i > 0) of the global context, and the anchor b_0's K/V [b, B, Hkv, d]
// is a separate buffer (received from the host holding b_0). Every local block
// attends to the anchor and causally to itself; s.B is the global block size (also
// the anchor's length), not clamped to the local context.
template <int D>
cudaError_t launch_phase1_anchored_t(const Shape& s, const void* q, const void* k, const void* v,
                                     const void* ka, const void* va, void* o, float* lse,
                                     cudaStream_t st) {
  alignas(64) CUtensorMap m[5];
  if (!encode_tma_bf16_4d(&m[0], q, D, s.hq, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[1], k, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[2], v, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[3], ka, D, s.hkv, s.B, s.B, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[4], va, D, s.hkv, s.B, s.B, s.b, 64, 1, 128, true))
    return cudaErrorInvalidValue;
  AttnArgs a = base_args(s);
  a.n_blocks = static_cast<int32_t>(s.n_blocks());
  a.mt = static_cast<int32_t>((s.B + 127) / 128);
  a.n_anchor = a.mt;
  a.anchor_sep = 1;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  const int64_t pairs_per_block = a.G >= 2 ? static_cast<int64_t>(a.mt) * (a.G / 2) : (a.mt + 1) / 2;
  const int64_t items = static_cast<int64_t>(s.b) * s.hkv * a.n_blocks * pairs_per_block;
  VarSeqs vs;
  vs.n = 0;
  return launch<D, Mode::kPhase1>(a, m, items, vs, st);
}

// Work items of one Phase-1 sequence of length L (blocks x q-tile pairs x kv-heads).
int64_t phase1_items(int64_t L, int64_t B, int G, int hkv) {
  if (L <= 0) return 0;
  const int64_t Bi = B < L ? B : L;
  const int64_t n_blocks = (L + Bi - 1) / Bi;
  const int64_t mt = (Bi + 127) / 128;
  const int64_t pairs = G >= 2 ? mt * (G / 2) : (mt + 1) / 2;
  return n_blocks * pairs * hkv;
}

template <int D>
cudaError_t launch_phase1_varlen_t(const Shape& s, const int64_t* cu, const void* q, const void* k,
                                   const void* v, void* o, float* lse, cudaStream_t st) {
  const int64_t total = cu[s.b];
  alignas(64) CUtensorMap m[5];
  if (!encode_tma_bf16_4d(&m[0], q, D, s.hq, total, total, 1, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[1], k, D, s.hkv, total, total, 1, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[2], v, D, s.hkv, total, total, 1, 64, 1, 128, true))
    return cudaErrorInvalidValue;
  m[3] = m[1];
  m[4] = m[2];
  AttnArgs a = base_args(s);
  a.L = total;  // row stride of the packed outputs (o rows, lse per head)
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  VarSeqs vs;
  vs.n = s.b;
  int64_t items = 0;
  for (int i = 0; i < s.b; ++i) {
    vs.item0[i] = static_cast<int32_t>(items);
    vs.start[i] = static_cast<int32_t>(cu[i]);
    items += phase1_items(cu[i + 1] - cu[i], s.B, a.G, s.hkv);
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  }
  vs.item0[s.b] = static_cast<int32_t>(items);
  vs.start[s.b] = static_cast<int32_t>(total);
  return launch<D, Mode::kPhase1>(a, m, items, vs, st);
}

template <int D>
cudaError_t launch_query_t(const Shape& s, const SplitPlan& p, const void* q, const void* k_new,
                           const void* v_new, int64_t lq, const void* kc, const void* vc,
                           const CacheRef& c, float* o_parts, float* lse_parts, cudaStream_t st,
                           bool write_cache) {
  const int G = s.group();
  alignas(64) CUtensorMap m[5];
  bool ok = encode_tma_bf16_4d(&m[0], q, D, s.hq, lq, lq, s.b, 64, G, 128 / G, true) &&
            encode_tma_bf16_4d(&m[1], kc, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) &&
            encode_tma_bf16_4d(&m[2], vc, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true);
  // The cache split's keys are exactly this call's query tokens: it reads them from
  // the inputs [b, Lq, Hkv, d] (rows past Lq read as zeros, so P = 0 never meets
  // whatever bytes the cache holds there). Without them (no cache split) the maps
  // only stand in.
  const void* ks = k_new ? k_new : kc;
  const void* vsrc = v_new ? v_new : vc;
  const int64_t rows = k_new ? lq : s.L;
  ok = ok && encode_tma_bf16_4d(&m[3], ks, D, s.hkv, rows, rows, s.b, 64, 1, 128, true) &&
       encode_tma_bf16_4d(&m[4], vsrc, D, s.hkv, rows, rows, s.b, 64, 1, 128, true);
  if (!ok) return cudaErrorInvalidValue;
  AttnArgs a = base_args(s);
  if (write_cache && k_new) {
    a.cw_k = static_cast<const uint4*>(k_new);
    a.cw_v = static_cast<const uint4*>(v_new);
    a.cw_kc = static_cast<uint4*>(c.k);
    a.cw_vc = static_cast<uint4*>(c.v);
    a.cw_cap = c.cap;
    a.cw_table = c.page_table;
    a.cw_page = c.page_size;
    a.cw_max_pages = c.max_pages;
    a.cw_num_pages = c.num_pages;
  }
  a.lq = lq;
  a.chunk = p.chunk;
  a.spb = p.spb;
  a.n_ctx = p.n_ctx;
  a.n_splits = p.n_splits;
  a.n_qt = static_cast<int32_t>(query_tiles(s, lq));
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  const int64_t items = static_cast<int64_t>(s.b) * s.hkv * a.n_splits * ((a.n_qt + 1) / 2);
  VarSeqs vs;
  vs.n = 0;
  return launch<D, Mode::kQuery>(a, m, items, vs, st);
}

template <int D>
cudaError_t launch_query_varlen_t(const Shape& s, const VarSeqs& vs, const void* q,
                                  const void* kc, const void* vc, const CacheRef& c,
                                  float* o_parts, float* lse_parts, cudaStream_t st) {
  const int G = s.group();
  const uint64_t total_q = static_cast<uint64_t>(vs.start[vs.n]);
  const uint64_t total_ctx = static_cast<uint64_t>(vs.ctx0[vs.n]);
  alignas(64) CUtensorMap m[5];
  bool ok = encode_tma_bf16_4d(&m[0], q, D, s.hq, total_q, total_q, 1, 64, G, 128 / G, true) &&
            encode_tma_bf16_4d(&m[1], kc, D, s.hkv, total_ctx, total_ctx, 1, 64, 1, 128, true) &&
            encode_tma_bf16_4d(&m[2], vc, D, s.hkv, total_ctx, total_ctx, 1, 64, 1, 128, true);
  if (c.paged()) {
    ok = ok &&
         encode_tma_bf16_4d(&m[3], c.k, D, s.hkv, c.page_size, c.page_size, c.num_pages, 64, 1, 128, true) &&
         encode_tma_bf16_4d(&m[4], c.v, D, s.hkv, c.page_size, c.page_size, c.num_pages, 64, 1, 128, true);
  } else {
    // every row of a sequence's cache is in bounds; the varlen cache write zeroed
    // the rows past its query rows up to the end of their 128-row tile
    ok = ok && encode_tma_bf16_4d(&m[3], c.k, D, s.hkv, c.cap, c.cap, s.b, 64, 1, 128, true) &&
         encode_tma_bf16_4d(&m[4], c.v, D, s.hkv, c.cap, c.cap, s.b, 64, 1, 128, true);
  }
  if (!ok) return cudaErrorInvalidValue;
  AttnArgs a = base_args(s);
  a.page_table = c.page_table;
  a.page_size = c.page_size;
  a.max_pages = c.max_pages;
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  return launch<D, Mode::kQuery>(a, m, vs.item0[vs.n], vs, st);
}

}  // namespace

int64_t query_tiles(const Shape& s, int64_t lq) { return (lq * s.group() + 127) / 128; }

int64_t plan_query_varlen(const Shape& s, const int64_t* cu_ctx, const int64_t* cu_q,
                          int64_t target_ctas, VarSeqs* vs) {
  // One chunk size for the batch, chosen so that all items (q-tile pairs x splits
  // x kv-heads) come to about target_ctas.
  int64_t work = 0, cache_items = 0;
  for (int i = 0; i < s.b; ++i) {
    const int64_t pairs = ((cu_q[i + 1] - cu_q[i]) * s.group() + 255) / 256;
    work += pairs * (cu_ctx[i + 1] - cu_ctx[i]) * s.hkv;
    cache_items += pairs * s.hkv;
  }
  const int64_t ctx_items = target_ctas - cache_items;
  int64_t C = ctx_items > 0 ? (work + ctx_items - 1) / ctx_items : work;
  if (C < 128) C = 128;
  vs->n = s.b;
  int64_t items = 0, rows = 0;
  for (int i = 0; i < s.b; ++i) {
    const int64_t L = cu_ctx[i + 1] - cu_ctx[i];
    const int64_t lq = cu_q[i + 1] - cu_q[i];
    int64_t spb = 1, n_ctx = 0;
    if (L > 0) {
      const int64_t B = s.B < L ? s.B : L;
      spb = (B + C - 1) / C;
      n_ctx = (L + B - 1) / B * spb;
    }
    const int64_t ns = n_ctx + 1;
    const int64_t pairs = (lq * s.group() + 255) / 256;
    vs->item0[i] = static_cast<int32_t>(items);
    vs->start[i] = static_cast<int32_t>(cu_q[i]);
    vs->ctx0[i] = static_cast<int32_t>(cu_ctx[i]);
    vs->rbase[i] = static_cast<int32_t>(rows);
    vs->spb[i] = static_cast<int32_t>(spb);
    items += pairs * ns * s.hkv;
    rows += ns * lq;
    if (items > 0x7fffffffLL || rows > 0x7fffffffLL) return -1;
  }
  vs->item0[s.b] = static_cast<int32_t>(items);
  vs->start[s.b] = static_cast<int32_t>(cu_q[s.b]);
  vs->ctx0[s.b] = static_cast<int32_t>(cu_ctx[s.b]);
  vs->rbase[s.b] = static_cast<int32_t>(rows);
  return rows;
}

cudaError_t launch_query_varlen(const Shape& s, const VarSeqs& vs, const void* q,
                                const void* kc, const void* vc, const CacheRef& c,
                                float* o_parts, float* lse_parts, void* o, float* lse,
                                cudaStream_t st) {
  cudaError_t e = s.d == 128 ? launch_query_varlen_t<128>(s, vs, q, kc, vc, c, o_parts, lse_parts, st)
                             : launch_query_varlen_t<64>(s, vs, q, kc, vc, c, o_parts, lse_parts, st);
  if (e != cudaSuccess) return e;
  return launch_merge_varlen(o_parts, lse_parts, vs, s.B, s.hq, s.d, o, lse, st);
}

cudaError_t launch_phase1_sm100(const Shape& s, const void* q, const void* k, const void* v,
                                void* o, float* lse, cudaStream_t st) {
  if (s.d == 128) return launch_phase1_t<128>(s, q, k, v, o, lse, st);
  return launch_phase1_t<64>(s, q, k, v, o, lse, st);
}

cudaError_t launch_phase1_anchor_q(const Shape& s, const void* q, const void* q_anchor,
                                   const void* k, const void* v, void* o, float* lse,
                                   cudaStream_t st) {
  if (s.d == 128) return launch_phase1_anchor_q_t<128>(s, q, q_anchor, k, v, o, lse, st);
  return launch_phase1_anchor_q_t<64>(s, q, q_anchor, k, v, o, lse, st);
}

cudaError_t launch_phase1_anchored(const Shape& s, const void* q, const void* k, const void* v,
                                   const void* k_anchor, const void* v_anchor, void* o, float* lse,
                                   cudaStream_t st) {
  if (s.d == 128) return launch_phase1_anchored_t<128>(s, q, k, v, k_anchor, v_anchor, o, lse, st);
  return launch_phase1_anchored_t<64>(s, q, k, v, k_anchor, v_anchor, o, lse, st);
}

cudaError_t launch_phase1_varlen(const Shape& s, const int64_t* cu_seqlens, const void* q,
                                 const void* k, const void* v, void* o, float* lse,
                                 cudaStream_t st) {
  if (s.d == 128) return launch_phase1_varlen_t<128>(s, cu_seqlens, q, k, v, o, lse, st);
  return launch_phase1_varlen_t<64>(s, cu_seqlens, q, k, v, o, lse, st);
}

cudaError_t launch_query_path(const Shape& s, const SplitPlan& p, const void* q,
                              const void* k_new, const void* v_new, int64_t lq,
                              const void* kc, const void* vc, const CacheRef& c, float* o_parts,
                              float* lse_parts, void* o, float* lse, cudaStream_t st,
                              bool o_fp32, bool write_cache) {
  cudaError_t e =
      s.d == 128 ? launch_query_t<128>(s, p, q, k_new, v_new, lq, kc, vc, c, o_parts, lse_parts, st, write_cache)
                 : launch_query_t<64>(s, p, q, k_new, v_new, lq, kc, vc, c, o_parts, lse_parts, st, write_cache);
  if (e != cudaSuccess) return e;
  return launch_merge(o_parts, lse_parts, p.n_splits, s.b, lq, s.hq, s.d, o, lse, st, o_fp32);
}

}  // namespace star
