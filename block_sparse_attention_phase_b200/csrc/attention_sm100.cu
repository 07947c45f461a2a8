// Tensor-core attention tiles on sm_100a (tcgen05 + TMEM + TMA), used by
// Phase 1 and by the Phase-2 query tokens.
//
// Phase 1 (hotaipapers.com page, Phase 1 paragraph; rebuttal to reviewer EMsM,
// "Size of Anchor Block"): block b_0 runs plain causal attention, every block
// b_i (i > 0) runs causal attention over [anchor = b_0 ; b_i] and keeps only its
// own rows. The anchor is never copied: a work item of block i first streams
// b_0's K/V tiles (all visible), then its own block's tiles up to the diagonal
// (the diagonal tile causally masked).
//   Work item = (batch, kv-head, block i, 128-row q-tile m, head in the GQA
//   group). Items are ordered so that the q-tiles and the G heads of one block
//   run together (their K/V and the anchor's stay in L2), blocks i > 0 before
//   b_0, larger m (longer rows) first.
//
// Phase-2 query tokens (hotaipapers.com page, Phase 2 paragraph): every split
// (a chunk of one context block, or the query-local cache) returns a partial
// output and its LSE for all query rows; the merge kernel combines them.
//   Work item = (batch, kv-head, split, q-tile). A q-tile packs 128/G query
//   tokens x the G heads of one kv-head into 128 rows, so each K/V tile feeds
//   all G heads. Context splits see every key of their chunk; the cache split is
//   causal: query token j sees cache rows 0..j.
//
// CTA = 6 warps:
//   warp 0     TMA producer: Q once, then K and V tiles into 2-stage rings
//   warp 1     TMEM allocator and MMA issuer (one thread):
//                S_j = Q K_j^T  (SS MMA, fp32 into TMEM, double-buffered)
//                O  += P_j V_j  (TS MMA: P read from TMEM, V from smem)
//   warps 2-5  softmax, one thread per row (TMEM lane = row): read S_j, mask,
//              running max with lazy rescaling (O is rescaled only when the max
//              grows by more than 2^8), P_j = exp2(...) written back to TMEM as
//              bf16 over S_j's columns; epilogue O / l and LSE.
// TMEM columns: S_0 [0,128), S_1 [128,256), O [256, 256+d).
// The QK^T MMA of tile j+1 overlaps the softmax of tile j.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int kThreads = 192;
constexpr uint32_t kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle row each)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;          // lazy-rescale threshold (log2 units)
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
  int32_t anchor_tail;    // visible columns of the last anchor tile
  __nv_bfloat16* o;       // [b, L, Hq, d]
  float* lse;             // [b, Hq, L] or null
  // Phase-2 query
  int64_t lq, chunk;
  int32_t spb, n_ctx, n_splits, n_qt;
  float* o_parts;    // [S, b, Lq, Hq, d]
  float* lse_parts;  // [S, b, Hq, Lq]
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t o_bar;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// What one CTA computes.
struct Item {
  int bb, kvh;
  int32_t qc1, qc2;  // Q tile coordinates: head (dim 1), token (dim 2)
  int n_tiles;
  // Phase 1
  int h, n_anchor, rows_valid;
  int64_t bstart, t0;
  // query
  int split, tok0;
  bool cache;
  int64_t k0, k1;
};

template <Mode M>
__device__ __forceinline__ Item decode_item(const AttnArgs& a) {
  Item it{};
  int64_t r = blockIdx.x;
  if constexpr (M == Mode::kPhase1) {
    const int hg = static_cast<int>(r % a.G);
    r /= a.G;
    const int mp = static_cast<int>(r % a.mt);
    r /= a.mt;
    const int ip = static_cast<int>(r % a.n_blocks);
    r /= a.n_blocks;
    it.kvh = static_cast<int>(r % a.hkv);
    it.bb = static_cast<int>(r / a.hkv);
    const int i = (ip + 1) % a.n_blocks;  // blocks 1..n-1 first, b_0 (cheapest) last
    const int m = a.mt - 1 - mp;          // longest q-tiles first
    it.h = it.kvh * a.G + hg;
    it.bstart = static_cast<int64_t>(i) * a.B;
    const int64_t bend = min(a.L, it.bstart + a.B);
    it.t0 = it.bstart + 128 * static_cast<int64_t>(m);
    it.rows_valid = it.t0 >= bend ? 0 : static_cast<int>(bend - it.t0 < 128 ? bend - it.t0 : 128);
    it.n_anchor = i > 0 ? a.n_anchor : 0;
    it.n_tiles = it.rows_valid > 0 ? it.n_anchor + m + 1 : 0;
    it.qc1 = it.h;
    it.qc2 = static_cast<int32_t>(it.t0);
  } else {
    const int qt = static_cast<int>(r % a.n_qt);
    r /= a.n_qt;
    it.split = static_cast<int>(r % a.n_splits);
    r /= a.n_splits;
    it.kvh = static_cast<int>(r % a.hkv);
    it.bb = static_cast<int>(r / a.hkv);
    it.tok0 = qt * (128 / a.G);
    it.cache = it.split == a.n_ctx;
    if (!it.cache) {
      const int64_t blk = it.split / a.spb;
      const int64_t sub = it.split % a.spb;
      const int64_t bs = blk * a.B;
      const int64_t be = min(a.L, bs + a.B);
      it.k0 = min(be, bs + sub * a.chunk);
      it.k1 = min(be, it.k0 + a.chunk);
    } else {
      it.k0 = 0;
      it.k1 = a.lq;
    }
    it.n_tiles = static_cast<int>((it.k1 - it.k0 + 127) / 128);
    it.qc1 = it.kvh * a.G;
    it.qc2 = it.tok0;
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

template <int D, Mode M>
__global__ void __launch_bounds__(kThreads, 1) attention_kernel(
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tk2,
    const __grid_constant__ CUtensorMap tv2, const AttnArgs a) {
  constexpr int CH = D / 64;
  constexpr uint32_t kTileBytes = CH * kChunkBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk = sq + kTileBytes;      // [2][kTileBytes]
  uint8_t* sv = sk + 2 * kTileBytes;  // [2][kTileBytes]
  Bars* bars = reinterpret_cast<Bars*>(sv + 2 * kTileBytes);

  const Item it = decode_item<M>(a);
  if (it.n_tiles == 0) {
    if constexpr (M == Mode::kQuery) {
      // A chunk past the end of a short last block: an empty partial.
      for (int idx = threadIdx.x; idx < 128 * D; idx += kThreads) {
        const int row = idx / D, e = idx % D;
        const int tok = it.tok0 + row / a.G;
        if (tok >= a.lq) continue;
        const int hq = it.kvh * a.G + row % a.G;
        const int64_t prow = static_cast<int64_t>(it.split) * a.b + it.bb;
        a.o_parts[((prow * a.lq + tok) * a.hq + hq) * D + e] = 0.f;
        if (e == 0) a.lse_parts[(prow * a.hq + hq) * a.lq + tok] = -INFINITY;
      }
    }
    return;  // before any barrier or TMEM allocation
  }
  const int n_tiles = it.n_tiles;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
    }
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_bar, 1);
    mbar_init(&bars->drain, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
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
      mbar_arrive_expect_tx(&bars->q_full, kTileBytes);
#pragma unroll
      for (int c = 0; c < CH; ++c)
        tma_load_4d(sq + c * kChunkBytes, &tq, &bars->q_full, c * 64, it.qc1, it.qc2, it.bb);
      int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        int32_t kv0;
        if constexpr (M == Mode::kPhase1) {
          kv0 = j < it.n_anchor ? j * 128 : static_cast<int32_t>(it.bstart + 128 * (j - it.n_anchor));
        } else {
          kv0 = static_cast<int32_t>(it.k0 + 128 * j);
        }
        if (j >= 2 && !wait_or_abort(&bars->k_empty[s], ph ^ 1, bars, a.status)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], kTileBytes);
#pragma unroll
        for (int c = 0; c < CH; ++c)
          tma_load_4d(sk + s * kTileBytes + c * kChunkBytes, mk, &bars->k_full[s], c * 64, it.kvh, kv0, it.bb);
        last_k[s] = j;
        if (j >= 2 && !wait_or_abort(&bars->v_empty[s], ph ^ 1, bars, a.status)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], kTileBytes);
#pragma unroll
        for (int c = 0; c < CH; ++c)
          tma_load_4d(sv + s * kTileBytes + c * kChunkBytes, mv, &bars->v_full[s], c * 64, it.kvh, kv0, it.bb);
        last_v[s] = j;
      }
      // Every copy this thread issued has landed before the CTA may exit (on the
      // normal path these phases completed long ago).
      mbar_wait(&bars->q_full, 0, a.status);
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (last_k[s] >= 0) mbar_wait(&bars->k_full[s], (last_k[s] >> 1) & 1, a.status);
        if (last_v[s] >= 0) mbar_wait(&bars->v_full[s], (last_v[s] >> 1) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescPV = make_idesc_bf16(128, D, false, true);
      const uint32_t sq_addr = smem_u32(sq);
      auto issue_pv = [&](int jp) -> bool {
        const int sp = jp & 1;
        if (!wait_or_abort(&bars->p_full, jp & 1, bars, a.status)) return false;
        if (!wait_or_abort(&bars->v_full[sp], (jp >> 1) & 1, bars, a.status)) return false;
        tc_fence_after();
        const uint32_t sv_addr = smem_u32(sv + sp * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          // B = V tile, MN-major (d contiguous): 16 kv rows per step; the next 64
          // columns of d sit one chunk (LBO) away, the next 8 kv rows 1024 B (SBO).
          tc_mma_ts(tmem + 256, tmem + sp * 128 + kk * 8,
                    make_sdesc(sv_addr + kk * 2048, kChunkBytes, 1024), kIdescPV,
                    (jp > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars->o_bar);
        tc_commit(&bars->v_empty[sp]);
        return true;
      };
      bool ok = wait_or_abort(&bars->q_full, 0, bars, a.status);
      tc_fence_after();
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j & 1;
        if (!wait_or_abort(&bars->k_full[s], (j >> 1) & 1, bars, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sk_addr = smem_u32(sk + s * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // A = Q, B = K, both K-major 128-byte swizzled: 16 columns = 32 bytes per step.
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          tc_mma_ss(tmem + s * 128, make_sdesc(sq_addr + off, 16, 1024),
                    make_sdesc(sk_addr + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars->s_full[s]);
        tc_commit(&bars->k_empty[s]);
        if (j >= 1 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) issue_pv(n_tiles - 1);
      // Every MMA this thread issued has completed before TMEM is released.
      tc_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      // Waits are per thread; the tcgen05 loads/stores below are warp-wide, so
      // the warp proceeds only if every lane's wait succeeded.
      ok = __all_sync(0xffffffffu, wait_or_abort(&bars->s_full[s], (j >> 1) & 1, bars, a.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + s * 128 + c * 32, sr[c]);
      tmem_wait_ld();
      // Columns [0, limit) of this tile are visible to this row.
      int limit = 128;
      if constexpr (M == Mode::kPhase1) {
        if (j == n_tiles - 1) limit = row + 1;                  // diagonal: causal
        else if (j == it.n_anchor - 1) limit = a.anchor_tail;  // partial last anchor tile
      } else {
        if (it.cache) {
          const int64_t lim = it.tok0 + row / a.G - 128 * j + 1;  // token j sees cache rows <= j
          limit = lim < 0 ? 0 : (lim > 128 ? 128 : static_cast<int>(lim));
        } else {
          const int64_t lim = it.k1 - it.k0 - 128 * j;            // end of the chunk
          limit = lim > 128 ? 128 : static_cast<int>(lim);
        }
      }
      // Most tiles are fully visible: mask only when some row of the warp needs it.
      if (__any_sync(0xffffffffu, limit < 128)) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= limit) sr[c][e] = __float_as_uint(-INFINITY);
      }
      // Row max with four independent 3-input max chains.
      float mc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        mc[c] = fmaxf(__uint_as_float(sr[c][0]), __uint_as_float(sr[c][1]));
#pragma unroll
        for (int e = 2; e < 32; e += 2)
          mc[c] = fmax3(mc[c], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
      }
      const float mt = fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
      const bool need = (m_run == -INFINITY) || ((mt - m_run) * sl2 > kRescaleLog2);
      const float m_new = need ? mt : m_run;
      const float m_use = m_new == -INFINITY ? 0.f : m_new;  // a row with nothing visible yet
      const float alpha = need ? ex2_approx((m_run - m_use) * sl2) : 1.f;
      m_run = m_new;
      const float ms = m_use * sl2;
      // p = 2^(s * scale * log2(e) - m'), two lanes per packed fp32 FMA / add.
      const float2 sl2v = make_float2(sl2, sl2);
      const float2 nms = make_float2(-ms, -ms);
      float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
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
          pk[c >> 1][(c & 1) * 16 + e / 2] = pack_bf16x2(p0, p1);
        }
      const float psum = (ps[0].x + ps[0].y) + (ps[1].x + ps[1].y);
      l_run = l_run * alpha + psum;
      if (j >= 1) {
        // PV of the previous tile must be done before O is rescaled and P overwritten.
        ok = __all_sync(0xffffffffu, wait_or_abort(&bars->o_bar, (j - 1) & 1, bars, a.status));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ob[32];
            tmem_ld32(lane_addr + 256 + c * 32, ob);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * alpha);
            tmem_st32(lane_addr + 256 + c * 32, ob);
          }
        }
      }
      tmem_st32(lane_addr + s * 128, pk[0]);
      tmem_st32(lane_addr + s * 128 + 32, pk[1]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(&bars->o_bar, (n_tiles - 1) & 1, bars, a.status));
    tc_fence_after();
    if (ok) {
      const bool has = l_run > 0.f;
      const float inv = has ? 1.f / l_run : 0.f;
      const float lse2 = has ? m_run * sl2 + log2f(l_run) : -INFINITY;
      if constexpr (M == Mode::kPhase1) {
        const int64_t t = it.t0 + row;
        __nv_bfloat16* dst = a.o + ((static_cast<int64_t>(it.bb) * a.L + t) * a.hq + it.h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ob[32];
          tmem_ld32(lane_addr + 256 + c * 32, ob);
          tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(ob[2 * e]) * inv, __uint_as_float(ob[2 * e + 1]) * inv);
          if (row < it.rows_valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              d4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
        if (a.lse && row < it.rows_valid)
          a.lse[(static_cast<int64_t>(it.bb) * a.hq + it.h) * a.L + t] = lse2 * 0.69314718055994531f;
      } else {
        const int tok = it.tok0 + row / a.G;
        const int hq = it.kvh * a.G + row % a.G;
        const bool valid = tok < a.lq;
        const int64_t prow = static_cast<int64_t>(it.split) * a.b + it.bb;
        float* dst = a.o_parts + ((prow * a.lq + tok) * a.hq + hq) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ob[32];
          tmem_ld32(lane_addr + 256 + c * 32, ob);
          tmem_wait_ld();
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              d4[q] = make_float4(__uint_as_float(ob[4 * q]) * inv, __uint_as_float(ob[4 * q + 1]) * inv,
                                  __uint_as_float(ob[4 * q + 2]) * inv, __uint_as_float(ob[4 * q + 3]) * inv);
          }
        }
        if (valid) a.lse_parts[(prow * a.hq + hq) * a.lq + tok] = lse2 * 0.69314718055994531f;
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
cudaError_t launch(const AttnArgs& a, const CUtensorMap (&m)[5], int64_t items, cudaStream_t st) {
  constexpr uint32_t kTileBytes = (D / 64) * kChunkBytes;
  // 5 tiles (Q, 2 K, 2 V) + barriers + alignment slack; at least 120 KB so that
  // only one CTA (and one 512-column TMEM allocation) lives on an SM.
  size_t smem = 5 * kTileBytes + sizeof(Bars) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  auto kern = attention_kernel<D, M>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (items <= 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  kern<<<static_cast<unsigned>(items), kThreads, smem, st>>>(m[0], m[1], m[2], m[3], m[4], a);
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
  a.anchor_tail = static_cast<int32_t>(s.B - 128 * static_cast<int64_t>(a.n_anchor - 1));
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  const int64_t items = static_cast<int64_t>(s.b) * s.hkv * a.n_blocks * a.mt * a.G;
  return launch<D, Mode::kPhase1>(a, m, items, st);
}

template <int D>
cudaError_t launch_query_t(const Shape& s, const SplitPlan& p, const void* q, int64_t lq,
                           const void* kc, const void* vc, const void* k_cache,
                           const void* v_cache, int64_t cap, float* o_parts, float* lse_parts,
                           cudaStream_t st) {
  const int G = s.group();
  alignas(64) CUtensorMap m[5];
  if (!encode_tma_bf16_4d(&m[0], q, D, s.hq, lq, lq, s.b, 64, G, 128 / G, true) ||
      !encode_tma_bf16_4d(&m[1], kc, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[2], vc, D, s.hkv, s.L, s.L, s.b, 64, 1, 128, true) ||
      // only the Lq rows written by this call are in bounds: rows past them
      // (unwritten, any bytes) read as zeros, so P = 0 never meets a NaN there
      !encode_tma_bf16_4d(&m[3], k_cache, D, s.hkv, lq, cap, s.b, 64, 1, 128, true) ||
      !encode_tma_bf16_4d(&m[4], v_cache, D, s.hkv, lq, cap, s.b, 64, 1, 128, true))
    return cudaErrorInvalidValue;
  AttnArgs a = base_args(s);
  a.lq = lq;
  a.chunk = p.chunk;
  a.spb = p.spb;
  a.n_ctx = p.n_ctx;
  a.n_splits = p.n_splits;
  a.n_qt = static_cast<int32_t>((lq * G + 127) / 128);
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  const int64_t items = static_cast<int64_t>(s.b) * s.hkv * a.n_splits * a.n_qt;
  return launch<D, Mode::kQuery>(a, m, items, st);
}

}  // namespace

int64_t query_tiles(const Shape& s, int64_t lq) { return (lq * s.group() + 127) / 128; }

cudaError_t launch_phase1_sm100(const Shape& s, const void* q, const void* k, const void* v,
                                void* o, float* lse, cudaStream_t st) {
  if (s.d == 128) return launch_phase1_t<128>(s, q, k, v, o, lse, st);
  return launch_phase1_t<64>(s, q, k, v, o, lse, st);
}

cudaError_t launch_query_path(const Shape& s, const SplitPlan& p, const void* q, int64_t lq,
                              const void* kc, const void* vc, const void* k_cache,
                              const void* v_cache, int64_t cap, float* o_parts, float* lse_parts,
                              void* o, float* lse, cudaStream_t st) {
  cudaError_t e = s.d == 128 ? launch_query_t<128>(s, p, q, lq, kc, vc, k_cache, v_cache, cap,
                                                   o_parts, lse_parts, st)
                             : launch_query_t<64>(s, p, q, lq, kc, vc, k_cache, v_cache, cap,
                                                  o_parts, lse_parts, st);
  if (e != cudaSuccess) return e;
  return launch_merge(o_parts, lse_parts, p.n_splits, s.b, lq, s.hq, s.d, o, lse, st);
}

}  // namespace star
