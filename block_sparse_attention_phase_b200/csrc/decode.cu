// Phase-2 decode step, split-KV partials (Star Attention, hotaipapers.com page,
// Phase 2 paragraph: the new token is sent to every block, each block attends
// with its own keys and returns one vector and one scalar; the query host
// appends the token's KV to its cache).
//
// One CTA = (split, batch, kv-head). A split is a chunk of one context block, or
// the query-local cache (which, after the append this kernel does, ends with the
// new token). The CTA streams its chunk's K and V rows for that kv-head once and
// serves all G = Hq/Hkv q-heads from them, so every KV byte is read from HBM
// exactly once per step. That makes the step HBM-bound; to keep the SMs from
// becoming the limit, the G x d x tokens contractions run as warp-level bf16
// MMAs (m16n8k16, fp32 accumulate) with the G heads as the MMA rows, about five
// instructions per key instead of ~80 on the FMA pipes.
//
// Data movement: a producer warp streams 64-token K and V tiles of one kv-head
// into a 3-stage ring with TMA (64-column boxes, 128-byte swizzle, so that the
// ldmatrix reads below hit 8 different bank groups). Each of the 4 consumer warps
// takes 16 tokens of every tile: S = Q K^T (2 n-tiles x d/16 k-steps), an online
// softmax per head (running max shared by the 4 lanes of a row), then O += P V
// with P reused straight from the S accumulators as the A operand. The warps'
// (m, l, O) meet in shared memory and the CTA writes one fp32 partial per head.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

struct DecodeArgs {
  const __nv_bfloat16* q;      // [b, 1, Hq, D]
  const __nv_bfloat16* k_new;  // [b, 1, Hkv, D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;      // [b, cap, Hkv, D]
  __nv_bfloat16* v_cache;
  int64_t cache_len, cap;
  int64_t L, B, chunk;
  int32_t spb, n_ctx, b, hq, hkv;
  float scale_log2;
  float* o_parts;    // [S, b, 1, Hq, D]
  float* lse_parts;  // [S, b, Hq, 1]
  uint32_t* status;
  // paged query-local cache (page_table == null: contiguous [b, cap, Hkv, D])
  const int32_t* page_table;  // [b, max_pages]; pool [num_pages, page_size, Hkv, D]
  int32_t page_size, max_pages, num_pages;
  // fused merge (counters == null: partials only, a separate merge kernel follows)
  __nv_bfloat16* o;    // [b, 1, Hq, D]
  float* lse;          // [b, Hq, 1]
  uint32_t* counters;  // [b * Hkv], zero between calls
  int32_t merge_batch; // splits the fused merge stages in shared memory per pass (>= 1)
};

constexpr int kTile = 64;      // tokens per TMA tile
constexpr int kWarps = 4;      // consumer warps (16 tokens of each tile apiece)
// Ring depth: 3 stages (96 KB at d = 128, two CTAs per SM) keep enough bytes in
// flight for long splits. For short splits the whole step is only a few tiles
// per CTA and the gaps between consecutive steps dominate, so 2 stages are used:
// three CTAs then fit on an SM, and the next step's CTAs (launched early through
// programmatic launch) start streaming in the free slot while this step drains.
constexpr int64_t kShortChunk = 2048;  // keys per split at or below which 2 stages are used
constexpr float kRescaleLog2 = 8.f;

STAR_HD constexpr size_t ring_bytes(int d, int stages) {
  return size_t{2} * stages * (d / 64) * kTile * 128;
}
STAR_HD constexpr size_t fused_weights_bytes(int64_t n_splits, int g) {
  return (static_cast<size_t>(n_splits) * g * 4 + 15) & ~size_t(15);
}
// The fused merge stages the LSE weights and then the splits' partial blocks (G x d
// fp32 each) in the CTA's shared memory, reusing the ring. The region may grow past
// the ring up to a cap that keeps the same number of CTAs per SM (three with 2
// stages, two with 3 stages); splits that do not fit are staged in several passes.
STAR_HD constexpr size_t merge_cap_bytes(int stages) {
  return stages <= 2 ? size_t{72} * 1024 : size_t{108} * 1024;
}
STAR_HD constexpr size_t split_block_bytes(int g, int d) { return static_cast<size_t>(g) * d * 4; }
STAR_HD constexpr size_t merge_region_bytes(int64_t n_splits, int g, int d, int stages) {
  const size_t ring = ring_bytes(d, stages);
  const size_t need = fused_weights_bytes(n_splits, g) + static_cast<size_t>(n_splits) * split_block_bytes(g, d);
  const size_t want = need < merge_cap_bytes(stages) ? need : merge_cap_bytes(stages);
  return want > ring ? want : ring;
}
// The fused merge needs room for the weights and at least one split's block.
STAR_HD constexpr bool fused_merge_fits(int64_t n_splits, int g, int d, int stages) {
  return fused_weights_bytes(n_splits, g) + split_block_bytes(g, d) <=
         merge_region_bytes(n_splits, g, d, stages);
}
// Splits staged per pass of the fused merge (at least 1 when it fits).
STAR_HD constexpr int64_t merge_batch_splits(int64_t n_splits, int g, int d, int stages) {
  const int64_t nb = static_cast<int64_t>(
      (merge_region_bytes(n_splits, g, d, stages) - fused_weights_bytes(n_splits, g)) /
      split_block_bytes(g, d));
  return nb < n_splits ? nb : n_splits;
}
// A uniform batch takes the two-kernel path (partials, then the merge kernel) when
// its fused merge would need more passes than this.
constexpr int64_t kMaxFusedPasses = 4;

template <class VL>
constexpr bool kIsVarlen = sizeof(VL) == sizeof(DecVarlen);

// The split a CTA streams, for a uniform batch (grid = splits x (batch * Hkv)) or a
// varlen one (1-D grid; the sequence found by binary search in the CTA table).
struct Split {
  int bb, kvh, split, n_splits;
  bool is_cache;
  int32_t k0, k1;           // key range: context tokens of the sequence, or cache rows
  int32_t ctx_tok, ctx_c3;  // context-map coordinate offset (packed varlen) and outer coordinate
  int32_t cache_len;
};

// Partial row (in units of Hq rows) of split s of the CTA's sequence: [S, b] for a
// uniform batch, the sequence's own run of rows for a varlen one.
template <class VL>
__device__ __forceinline__ int64_t part_row(const DecodeArgs& a, const VL& dv, const Split& w,
                                            int s) {
  if constexpr (kIsVarlen<VL>) return static_cast<int64_t>(dv.split0[w.bb]) + s;
  else return static_cast<int64_t>(s) * a.b + w.bb;
}

// A uniform batch needs no table: its launches carry this instead of DecVarlen.
struct NoVarlen {
  int32_t n;
};

template <class VL>
__device__ __forceinline__ Split locate(const DecodeArgs& a, const VL& dv) {
  Split w;
  int64_t L = a.L, B = a.B, chunk = a.chunk;
  int spb = a.spb, n_ctx = a.n_ctx;
  if constexpr (!kIsVarlen<VL>) {
    w.split = blockIdx.x;
    w.bb = blockIdx.y / a.hkv;
    w.kvh = blockIdx.y % a.hkv;
    w.n_splits = gridDim.x;
    w.cache_len = static_cast<int32_t>(a.cache_len);
    w.ctx_tok = 0;
    w.ctx_c3 = w.bb;
  } else {
    const int r0 = blockIdx.x;
    int lo = 0, hi = dv.n;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (dv.cta0[mid] <= r0) lo = mid; else hi = mid;
    }
    const int r = r0 - dv.cta0[lo];
    w.n_splits = dv.split0[lo + 1] - dv.split0[lo];
    w.kvh = r / w.n_splits;
    w.split = r % w.n_splits;
    w.bb = lo;
    n_ctx = w.n_splits - 1;
    L = dv.ctx0[lo + 1] - dv.ctx0[lo];
    B = min(a.B, L);
    spb = dv.spb[lo];
    chunk = L > 0 ? (B + spb - 1) / spb : 1;
    w.cache_len = dv.cache_len[lo];
    w.ctx_tok = dv.ctx0[lo];
    w.ctx_c3 = 0;
  }
  w.is_cache = w.split == n_ctx;
  if (!w.is_cache) {
    const int64_t blk = w.split / spb;
    const int64_t sub = w.split % spb;
    const int64_t bstart = blk * B;
    const int64_t bend = min(L, bstart + B);
    const int64_t k0 = min(bend, bstart + sub * chunk);
    w.k0 = static_cast<int32_t>(k0);
    w.k1 = static_cast<int32_t>(min(bend, k0 + chunk));
  } else {
    w.k0 = 0;
    w.k1 = w.cache_len + 1;  // the cached rows and the new token, appended by the CTA
  }
  return w;
}

// Fused merge, run by the consumer threads of every CTA after it has stored its
// partial: the CTA that completes the count of its (sequence, kv-head) is the
// last one, all the other splits' partials are in memory, and it combines them
// (the query host's aggregation: M = max lse_s, W = sum exp(lse_s - M),
// o = sum exp(lse_s - M) o_s / W, lse = M + ln W) for its G heads. It also puts
// the counter back to zero for the next call.
//
// The combine is bound by L2 latency, so it takes as few round trips as possible:
// one gpu-scope fence and one atomic per CTA (the grid-barrier pattern: the CTA's
// stores, a CTA barrier, then one thread's fence and count); in the last CTA one
// thread copies each split's partial block (G x d fp32, contiguous) into shared
// memory with one 1-D bulk copy on an mbarrier, issued before the LSEs are read so
// that both are in flight together. Each thread then owns float4 columns of the
// G x d output and sums over the staged splits from shared memory.
template <int D, int G, class VL>
__device__ __forceinline__ void merge_if_last(const DecodeArgs& a, const VL& dv, const Split& w,
                                              uint8_t* smem) {
  constexpr int kThreads = kWarps * 32;
  constexpr int F = G * D / 4;  // float4 columns of one split's G x D block
  __shared__ int s_last;
  __shared__ float s_m[G], s_w[G];
  __shared__ alignas(8) uint64_t s_staged;  // the bulk copies of one staging pass landed
  const int tid = threadIdx.x;  // 0 .. 127 (the consumer warps)
  asm volatile("bar.sync 1, %0;" ::"r"(kThreads) : "memory");  // every partial store issued
  if (tid == 0) {
    __threadfence();  // orders the CTA's partial stores (ordered before it by the barrier)
    uint32_t* ctr = a.counters + (static_cast<int64_t>(w.bb) * a.hkv + w.kvh);
    const uint32_t prev = atomicAdd(ctr, 1u);
    const int last = prev == static_cast<uint32_t>(w.n_splits - 1);
    if (last) {
      atomicExch(ctr, 0u);  // every split of this launch has counted
      __threadfence();      // the other splits' partials are visible from here on
    }
    s_last = last;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kThreads) : "memory");
  if (!s_last) return;

  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int S = w.n_splits;
  const int nb = a.merge_batch;
  const int64_t row0 = part_row(a, dv, w, 0) * a.hq + w.kvh * G;  // split 0, first head
  const int64_t stride = (part_row(a, dv, w, 1) - part_row(a, dv, w, 0)) * a.hq;  // between splits
  const int64_t orow0 = static_cast<int64_t>(w.bb) * a.hq + w.kvh * G;  // output row
  float* wts = reinterpret_cast<float*>(smem);                                  // [S][G]
  float4* parts = reinterpret_cast<float4*>(smem + fused_weights_bytes(S, G));  // [nb][F]
  const uint32_t parts_s = smem_u32(parts);

  // Copies of splits sp0 .. sp0 + nb - 1 into the staging area, one bulk copy of
  // G x D floats per split, completing on s_staged (thread 0 issues them).
  constexpr uint32_t kBlockBytes = G * D * 4;
  if (tid == 0) {
    mbar_init(&s_staged, 1);
    fence_barrier_init();
    // The partials were written by other CTAs (generic stores, acquired through the
    // counter above); the bulk copies below read them through the async proxy.
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  auto stage = [&](int sp0) {
    if (tid != 0) return;
    const int cnt = min(nb, S - sp0);
    mbar_arrive_expect_tx(&s_staged, cnt * kBlockBytes);
    for (int j = 0; j < cnt; ++j) {
      const float* src = a.o_parts + (row0 + static_cast<int64_t>(sp0 + j) * stride) * D;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              parts_s + j * kBlockBytes),
          "l"(src), "r"(kBlockBytes), "r"(smem_u32(&s_staged))
          : "memory");
    }
  };
  int pass = 0;
  // 1. the LSEs -> shared memory (the first 4 per thread are loaded before the
  //    staging copies are issued, so that they do not queue behind them); per head
  //    (warp h % 4, lanes over the splits) the maximum M, the weights exp(lse_s - M)
  //    in place and their sum W
  auto lse_at = [&](int i) {
    return __ldcg(a.lse_parts + row0 + static_cast<int64_t>(i / G) * stride + i % G);
  };
  float first[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = tid + kThreads * k;
    first[k] = i < S * G ? lse_at(i) : 0.f;
  }
  stage(0);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = tid + kThreads * k;
    if (i < S * G) wts[i] = first[k];
  }
  for (int i = tid + 4 * kThreads; i < S * G; i += kThreads) wts[i] = lse_at(i);
  asm volatile("bar.sync 1, %0;" ::"r"(kThreads) : "memory");
  for (int h = warp; h < G; h += kWarps) {
    float m = -INFINITY;
    for (int sp = lane; sp < S; sp += 32) m = fmaxf(m, wts[sp * G + h]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float sum = 0.f;
    for (int sp = lane; sp < S; sp += 32) {
      const float wv = m == -INFINITY ? 0.f : expf(wts[sp * G + h] - m);  // 0: empty split or head
      wts[sp * G + h] = wv;
      sum += wv;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) {
      s_m[h] = m;
      s_w[h] = sum;
    }
  }

  // 2. weighted sums of the staged partial blocks
  constexpr int KPT = (F + kThreads - 1) / kThreads;  // float4 columns per thread
  float4 acc[KPT];
#pragma unroll
  for (int k = 0; k < KPT; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp0 = 0; sp0 < S; sp0 += nb, ++pass) {
    // staged blocks landed (a second bounded wait after a timeout: no copy may
    // still be in flight when the CTA moves on)
    if (!mbar_wait(&s_staged, pass & 1, a.status)) mbar_wait(&s_staged, pass & 1, a.status);
    asm volatile("bar.sync 1, %0;" ::"r"(kThreads) : "memory");  // and the weights are ready
    const int cnt = min(nb, S - sp0);
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      const int f = tid + kThreads * k;
      if (F % kThreads == 0 || f < F) {
        const int h = f / (D / 4);
        for (int j = 0; j < cnt; ++j) {
          const float wv = wts[(sp0 + j) * G + h];
          const float4 x = parts[j * F + f];
          acc[k].x += wv * x.x;
          acc[k].y += wv * x.y;
          acc[k].z += wv * x.z;
          acc[k].w += wv * x.w;
        }
      }
    }
    if (sp0 + nb < S) {
      asm volatile("bar.sync 1, %0;" ::"r"(kThreads) : "memory");  // staging area free again
      if (tid == 0) fence_proxy_async_smem();  // the reads above precede the copies that overwrite it
      stage(sp0 + nb);
    }
  }
  // outputs [b, 1, Hq, D] and [b, Hq, 1]
  const int64_t out_rows = static_cast<int64_t>(kIsVarlen<VL> ? dv.n : a.b) * a.hq;
  if (!STAR_IN_BOUNDS(a.status, orow0 + G - 1, out_rows)) return;
  if (tid < G && a.lse) a.lse[orow0 + tid] = s_w[tid] > 0.f ? s_m[tid] + logf(s_w[tid]) : -INFINITY;
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    const int f = tid + kThreads * k;
    if (F % kThreads == 0 || f < F) {
      const float W = s_w[f / (D / 4)];
      const float inv = W > 0.f ? 1.f / W : 0.f;
      uint2 packed;
      packed.x = pack_bf16x2(acc[k].x * inv, acc[k].y * inv);
      packed.y = pack_bf16x2(acc[k].z * inv, acc[k].w * inv);
      *reinterpret_cast<uint2*>(a.o + orow0 * D + 4 * f) = packed;  // G heads are contiguous
    }
  }
}

template <int D, int G, int kStages, class VL>
__global__ void __launch_bounds__((kWarps + 1) * 32, kStages <= 2 ? 3 : 2) decode_partials_kernel(
    const __grid_constant__ CUtensorMap mk_ctx, const __grid_constant__ CUtensorMap mv_ctx,
    const __grid_constant__ CUtensorMap mk_cache, const __grid_constant__ CUtensorMap mv_cache,
    const DecodeArgs a, const __grid_constant__ VL dv) {
  constexpr int CH = D / 64;                        // 64-column chunks of a row
  constexpr uint32_t kChunk = kTile * 128;          // one chunk of a tile: 64 rows x 128 B
  constexpr uint32_t kTileBytes = CH * kChunk;
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "GQA group must be 1, 2, 4 or 8");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* kbuf = base;                          // [kStages][kTileBytes]
  uint8_t* vbuf = base + kStages * kTileBytes;   // [kStages][kTileBytes]
  // The barriers live outside the dynamic region, which the fused merge reuses whole.
  __shared__ alignas(8) uint64_t full[kStages];
  __shared__ alignas(8) uint64_t empty[kStages];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == kWarps && lane == 0) {  // descriptor fetches overlap the prologue
    tma_prefetch_desc(&mk_ctx);
    tma_prefetch_desc(&mv_ctx);
    tma_prefetch_desc(&mk_cache);
    tma_prefetch_desc(&mv_cache);
  }
  const Split w = locate(a, dv);
  const int bb = w.bb;
  const int kvh = w.kvh;
  const bool is_cache = w.is_cache;
  const int64_t k0 = w.k0, k1 = w.k1;
  const int64_t cache_len = w.cache_len;
  const int ntiles = static_cast<int>((k1 - k0 + kTile - 1) / kTile);
  // Varlen batches with a contiguous cache cannot end each sequence's cache map at
  // its own length, so rows past k1 in the cache's last tile are zeroed in shared
  // memory instead (those rows may hold any bytes; P = 0 times NaN would be NaN).
  const bool zero_tail = kIsVarlen<VL> && is_cache && !a.page_table;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  // The merge that reads this launch's partials may be scheduled now; it waits for
  // this grid to finish before reading anything. (This kernel itself may have
  // started while the previous step's merge was still reading the workspace: the
  // partials are written only after pdl_wait() below. Everything it reads — the
  // context, the cache rows and this step's inputs — was complete before that
  // merge could start.)
  pdl_launch_dependents();

  if (warp == kWarps) {
    // ---------------- producer warp: the cache append, then TMA loads ----------------
    // With the fused merge the previous decode step is a kernel of this same kind,
    // which may still be appending its own row: the cache split waits for it to
    // finish before it writes or reads any cache row. (Context splits read only
    // the context, written long before.)
    if (is_cache && a.counters) pdl_wait();
    if (is_cache && lane < D / 8) {
      // Cache row of (this sequence, row r): contiguous [b, cap, Hkv, D], or row
      // r % P of page table[b][r / P] in the pool [num_pages, P, Hkv, D]. A page id
      // outside the pool is refused (bounds flag, no write).
      int64_t page = 0;
      if (a.page_table) {
        page = a.page_table[static_cast<int64_t>(bb) * a.max_pages + cache_len / a.page_size];
        if (page < 0 || page >= a.num_pages) {
          if (lane == 0) atomicOr(a.status, kBoundsFlag);
          page = -1;
        }
      }
      auto row_off = [&](int64_t r) -> int64_t {
        const int64_t prow = a.page_table ? page * a.page_size + r % a.page_size
                                          : static_cast<int64_t>(bb) * a.cap + r;
        return (prow * a.hkv + kvh) * D + lane * 8;
      };
      // cache elements: the pool [num_pages, P, Hkv, D] or [b, cap, Hkv, D]
      const int64_t cache_elems =
          (a.page_table ? static_cast<int64_t>(a.num_pages) * a.page_size : static_cast<int64_t>(a.b) * a.cap) *
          a.hkv * D;
      if (page >= 0 && STAR_IN_BOUNDS(a.status, row_off(cache_len) + 7, cache_elems)) {
        const int64_t src = (static_cast<int64_t>(bb) * a.hkv + kvh) * D + lane * 8;
        const int64_t dst = row_off(cache_len);
        *reinterpret_cast<uint4*>(a.k_cache + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
        *reinterpret_cast<uint4*>(a.v_cache + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
        if (a.page_table && cache_len % a.page_size == 0) {
          // The append opens a new page: zero its other rows (for this kv-head), so
          // that tiles reaching past the last valid row read zeros, never stale bytes.
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          for (int64_t r = cache_len + 1; r < cache_len + a.page_size; ++r) {
            const int64_t off = row_off(r);
            if (!STAR_IN_BOUNDS(a.status, off + 7, cache_elems)) break;
            *reinterpret_cast<uint4*>(a.k_cache + off) = z;
            *reinterpret_cast<uint4*>(a.v_cache + off) = z;
          }
        }
      }
      fence_proxy_async_global();  // the TMA loads below read these rows
    }
    __syncwarp();
    if (lane == 0 && ntiles > 0) {
      const CUtensorMap* mk = is_cache ? &mk_cache : &mk_ctx;
      const CUtensorMap* mv = is_cache ? &mv_cache : &mv_ctx;
      for (int i = 0; i < ntiles; ++i) {
        const int stg = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (i >= kStages && !mbar_wait(&empty[stg], ph ^ 1, a.status)) break;
        mbar_arrive_expect_tx(&full[stg], 2 * kTileBytes);
        int32_t t0 = static_cast<int32_t>(k0 + static_cast<int64_t>(i) * kTile);
        // Outer coordinate: the sequence (a packed varlen context: 0, with the
        // sequence's first token added to t0), or for a paged cache the page.
        int32_t c3 = bb;
        if (!is_cache) {
          t0 += w.ctx_tok;
          c3 = w.ctx_c3;
        } else if (a.page_table) {
          c3 = a.page_table[static_cast<int64_t>(bb) * a.max_pages + t0 / a.page_size];
          t0 %= a.page_size;
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          tma_load_4d(kbuf + stg * kTileBytes + c * kChunk, mk, &full[stg], c * 64, kvh, t0, c3);
          tma_load_4d(vbuf + stg * kTileBytes + c * kChunk, mv, &full[stg], c * 64, kvh, t0, c3);
        }
      }
    }
  } else {
    // ---------------- consumer warps ----------------
    const int g = lane >> 2;        // MMA row: the q-head within the group (rows >= G are zero)
    const int q2 = (lane & 3) * 2;  // MMA column pair
    // Q as the A operand (rows = heads, k = d): a0 = row g, cols q2..q2+1; a2 = cols +8.
    uint32_t qa[D / 16][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      if (g < G) {
        const __nv_bfloat16* qrow = a.q + (static_cast<int64_t>(bb) * a.hq + kvh * G + g) * D + ks * 16;
        qa[ks][0] = *reinterpret_cast<const uint32_t*>(qrow + q2);
        qa[ks][1] = *reinterpret_cast<const uint32_t*>(qrow + q2 + 8);
      } else {
        qa[ks][0] = 0u;
        qa[ks][1] = 0u;
      }
    }
    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    float m_run = -INFINITY;  // running max of row g (raw score units); equal on its 4 lanes
    float l_run = 0.f;        // this lane's share of row g's running sum
    const float sl2 = a.scale_log2;

    // ldmatrix row addresses inside one stage tile, swizzled the way the TMA wrote them.
    // QK (B = K rows): lane -> matrix mi = lane/8 (d offset 8*mi), row ri = lane%8 (token).
    // PV (B = V rows, transposed): matrix mi -> tokens +8*(mi&1), d offset 8*(mi>>1).
    const int mi = lane >> 3, ri = lane & 7;
    const int tw0 = warp * 16;

    for (int i = 0; i < ntiles; ++i) {
      const int stg = i % kStages;
      const bool ok = mbar_wait(&full[stg], (i / kStages) & 1, a.status);
      if (ok) {
        const uint32_t kt = smem_u32(kbuf + stg * kTileBytes);
        const uint32_t vt = smem_u32(vbuf + stg * kTileBytes);
        if (zero_tail && i == ntiles - 1) {
          // this warp's 16 rows at or past k1: zero their K and V (whole 128-byte
          // swizzle rows of every 64-column chunk)
          const int64_t first = k1 - (k0 + static_cast<int64_t>(i) * kTile);  // first row to zero
          for (int u = lane; u < 16 * CH * 8; u += 32) {
            const int rr = tw0 + u / (CH * 8);
            const int c = (u / 8) % CH;
            if (rr >= first) {
              const uint32_t off = stg * kTileBytes + c * kChunk + rr * 128 + (u % 8) * 16;
              *reinterpret_cast<uint4*>(kbuf + off) = make_uint4(0u, 0u, 0u, 0u);
              *reinterpret_cast<uint4*>(vbuf + off) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          __syncwarp();
        }
        // ---- S = Q K^T for this warp's 16 tokens (two n-tiles of 8)
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
          const int tok = tw0 + nt * 8 + ri;
#pragma unroll
          for (int ks = 0; ks < D / 16; ks += 2) {
            const int d0 = ks * 16 + mi * 8;  // this lane's matrix covers d0..d0+7
            const uint32_t addr = kt + (d0 >> 6) * kChunk + tok * 128 +
                                  ((((d0 & 63) >> 3) ^ (tok & 7)) << 4);
            uint32_t b[4];
            ldsm_x4(addr, b);
            mma_16816(s[nt], qa[ks][0], 0u, qa[ks][1], 0u, b[0], b[1]);
            mma_16816(s[nt], qa[ks + 1][0], 0u, qa[ks + 1][1], 0u, b[2], b[3]);
          }
        }
        // ---- mask keys past the end of the split
        const int64_t tbase = k0 + static_cast<int64_t>(i) * kTile + tw0;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (tbase + nt * 8 + q2 + e >= k1) s[nt][e] = -INFINITY;
        // ---- online softmax for row g (values s[nt][0..1]; rows g+8 are padding)
        float mt = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const bool need = (m_run == -INFINITY) || ((mt - m_run) * sl2 > kRescaleLog2);
        const float m_new = need ? mt : m_run;
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        if (need) {
          const float alpha = ex2_approx((m_run - m_use) * sl2);
          l_run *= alpha;
#pragma unroll
          for (int nt = 0; nt < D / 8; ++nt) {
            o[nt][0] *= alpha;
            o[nt][1] *= alpha;
          }
        }
        m_run = m_new;
        const float ms = m_use * sl2;
        float p[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            p[nt][e] = ex2_approx(fmaf(s[nt][e], sl2, -ms));
            l_run += p[nt][e];
          }
        // P as the A operand (16 tokens): a0 = tokens q2.. of n-tile 0, a2 = of n-tile 1.
        const uint32_t pa0 = pack_bf16x2(p[0][0], p[0][1]);
        const uint32_t pa2 = pack_bf16x2(p[1][0], p[1][1]);
        // ---- O += P V
        const int vtok = tw0 + ri + 8 * (mi & 1);
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
          const int d0 = dt * 16 + 8 * (mi >> 1);
          const uint32_t addr = vt + (d0 >> 6) * kChunk + vtok * 128 +
                                ((((d0 & 63) >> 3) ^ (vtok & 7)) << 4);
          uint32_t b[4];
          ldsm_x4_trans(addr, b);
          mma_16816(o[2 * dt], pa0, 0u, pa2, 0u, b[0], b[1]);
          mma_16816(o[2 * dt + 1], pa0, 0u, pa2, 0u, b[2], b[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stg]);
    }

    // ---- combine the 4 lanes of each row, then the warps
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    // Every stage has been consumed and no copy is in flight: reuse the ring.
    asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
    float* cm = reinterpret_cast<float*>(base);  // [kWarps][G]
    float* cl = cm + kWarps * G;                 // [kWarps][G]
    float* cacc = cl + kWarps * G;               // [kWarps][G][D]
    if (g < G) {
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        cacc[(warp * G + g) * D + nt * 8 + q2] = o[nt][0];
        cacc[(warp * G + g) * D + nt * 8 + q2 + 1] = o[nt][1];
      }
      if (q2 == 0) {
        cm[warp * G + g] = m_run;
        cl[warp * G + g] = l_run;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
    // Per head: the CTA's maximum over the warps, each warp's weight exp2(m_w - M)
    // divided by the CTA's sum, and the CTA's LSE; then every thread writes float4
    // columns of the G x D partial as the weighted sum of the warps' accumulators.
    __shared__ float s_sc[kWarps][G];
    __shared__ float s_plse[G];
    if (threadIdx.x < G) {
      const int h = threadIdx.x;
      float M = -INFINITY;
#pragma unroll
      for (int wi = 0; wi < kWarps; ++wi) M = fmaxf(M, cm[wi * G + h]);
      float sc[kWarps];
      float lsum = 0.f;
#pragma unroll
      for (int wi = 0; wi < kWarps; ++wi) {
        sc[wi] = M == -INFINITY ? 0.f : ex2_approx((cm[wi * G + h] - M) * sl2);
        lsum += cl[wi * G + h] * sc[wi];
      }
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
      for (int wi = 0; wi < kWarps; ++wi) s_sc[wi][h] = sc[wi] * inv;
      s_plse[h] = lsum > 0.f ? (M * sl2 + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
    pdl_wait();  // the previous kernel (which may still read the workspace) has finished
    const int64_t prow = part_row(a, dv, w, w.split) * a.hq + kvh * G;  // first head's row
    const float4* cacc4 = reinterpret_cast<const float4*>(cacc);
    float4* dst = reinterpret_cast<float4*>(a.o_parts + prow * D);
    // partial rows of the launch: [S, b] (uniform) or the varlen splits; Hq rows of D each
    int64_t part_rows;
    if constexpr (kIsVarlen<VL>) part_rows = dv.split0[dv.n];
    else part_rows = static_cast<int64_t>(gridDim.x) * a.b;
    const bool part_ok = STAR_IN_BOUNDS(a.status, (prow + G) * D - 1, part_rows * a.hq * D);
    for (int f = threadIdx.x; part_ok && f < G * D / 4; f += kWarps * 32) {
      const int h = f / (D / 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int wi = 0; wi < kWarps; ++wi) {
        const float4 x = cacc4[wi * (G * D / 4) + f];
        const float sc = s_sc[wi][h];
        acc.x += sc * x.x;
        acc.y += sc * x.y;
        acc.z += sc * x.z;
        acc.w += sc * x.w;
      }
      dst[f] = acc;
    }
    if (threadIdx.x < G && part_ok) a.lse_parts[prow + threadIdx.x] = s_plse[threadIdx.x];
    if (a.counters) merge_if_last<D, G>(a, dv, w, base);
  }
}

// Context maps: uniform [b, L, Hkv, D], or a packed varlen context [total, Hkv, D]
// (ctx_batch = 1). Cache maps: the page pool; a contiguous uniform cache whose
// extent ends after the new row (rows past it read as zeros); or a contiguous varlen
// cache, all rows in bounds (the kernel zeroes the tail rows in shared memory).
template <int D, int G, int kStages, class VL>
cudaError_t launch_decode_t(const Shape& s, const DecodeArgs& a, const VL& dv, dim3 grid,
                            int64_t max_splits, uint64_t ctx_tokens, uint64_t ctx_batch,
                            int32_t num_pages, const void* kc, const void* vc, cudaStream_t st) {
  alignas(64) CUtensorMap m[4];
  bool ok = encode_tma_bf16_4d(&m[0], kc, D, s.hkv, ctx_tokens, ctx_tokens, ctx_batch, 64, 1, kTile, true) &&
            encode_tma_bf16_4d(&m[1], vc, D, s.hkv, ctx_tokens, ctx_tokens, ctx_batch, 64, 1, kTile, true);
  if (a.page_table) {
    ok = ok &&
         encode_tma_bf16_4d(&m[2], a.k_cache, D, s.hkv, a.page_size, a.page_size, num_pages, 64, 1, kTile, true) &&
         encode_tma_bf16_4d(&m[3], a.v_cache, D, s.hkv, a.page_size, a.page_size, num_pages, 64, 1, kTile, true);
  } else {
    const uint64_t cache_rows = kIsVarlen<VL> ? static_cast<uint64_t>(a.cap) : static_cast<uint64_t>(a.cache_len + 1);
    ok = ok &&
         encode_tma_bf16_4d(&m[2], a.k_cache, D, s.hkv, cache_rows, a.cap, s.b, 64, 1, kTile, true) &&
         encode_tma_bf16_4d(&m[3], a.v_cache, D, s.hkv, cache_rows, a.cap, s.b, 64, 1, kTile, true);
  }
  if (!ok) return cudaErrorInvalidValue;
  size_t region = ring_bytes(D, kStages);
  DecodeArgs args = a;
  if (a.counters) {
    if (!fused_merge_fits(max_splits, G, D, kStages)) return cudaErrorInvalidValue;
    region = merge_region_bytes(max_splits, G, D, kStages);
    args.merge_batch = static_cast<int32_t>(merge_batch_splits(max_splits, G, D, kStages));
  }
  const size_t smem = region + 1024;  // + alignment of the region to 1024 bytes
  auto kern = decode_partials_kernel<D, G, kStages, VL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_programmatic(kern, grid, dim3((kWarps + 1) * 32), smem, st, m[0], m[1], m[2], m[3], args,
                          dv);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

int decode_stages(int64_t chunk) { return chunk <= kShortChunk ? 2 : 3; }

DecodeArgs make_args(const Shape& s, const void* q, const void* k_new, const void* v_new,
                     const CacheRef& c, float* o_parts, float* lse_parts, const FusedMerge* fm) {
  DecodeArgs a{};
  a.o = fm ? static_cast<__nv_bfloat16*>(fm->o) : nullptr;
  a.lse = fm ? fm->lse : nullptr;
  a.counters = fm ? fm->counters : nullptr;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.k_cache = static_cast<__nv_bfloat16*>(c.k);
  a.v_cache = static_cast<__nv_bfloat16*>(c.v);
  a.cap = c.cap;
  a.page_table = c.page_table;
  a.page_size = c.page_size;
  a.max_pages = c.max_pages;
  a.num_pages = c.num_pages;
  a.L = s.L;
  a.B = s.B;
  a.b = s.b;
  a.hq = s.hq;
  a.hkv = s.hkv;
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  a.status = device_status_word();
  return a;
}

template <class VL>
cudaError_t dispatch(const Shape& s, const DecodeArgs& a, const VL& dv, dim3 grid,
                     int64_t max_splits, int64_t max_chunk, uint64_t ctx_tokens, uint64_t ctx_batch,
                     int32_t num_pages, const void* kc, const void* vc, cudaStream_t st) {
  const int G = s.group();
  const bool two = decode_stages(max_chunk) == 2;
#define STAR_DECODE_CASE(DD, GG)                                                                  \
  if (s.d == DD && G == GG)                                                                       \
    return two ? launch_decode_t<DD, GG, 2, VL>(s, a, dv, grid, max_splits, ctx_tokens,         \
                                                ctx_batch, num_pages, kc, vc, st)                 \
               : launch_decode_t<DD, GG, 3, VL>(s, a, dv, grid, max_splits, ctx_tokens,         \
                                                ctx_batch, num_pages, kc, vc, st);
  STAR_DECODE_CASE(128, 1) STAR_DECODE_CASE(128, 2) STAR_DECODE_CASE(128, 4)
  STAR_DECODE_CASE(128, 8) STAR_DECODE_CASE(64, 1) STAR_DECODE_CASE(64, 2)
  STAR_DECODE_CASE(64, 4) STAR_DECODE_CASE(64, 8)
#undef STAR_DECODE_CASE
  return cudaErrorNotSupported;
}

}  // namespace

bool decode_fused_fits(const Shape& s, const SplitPlan& p) {
  const int st = decode_stages(p.chunk);
  return fused_merge_fits(p.n_splits, s.group(), s.d, st) &&
         merge_batch_splits(p.n_splits, s.group(), s.d, st) * kMaxFusedPasses >= p.n_splits;
}

cudaError_t launch_decode_partials(const Shape& s, const SplitPlan& p, const void* q,
                                   const void* k_new, const void* v_new, const void* kc,
                                   const void* vc, const CacheRef& c, int64_t cache_len,
                                   float* o_parts, float* lse_parts, const FusedMerge* fm,
                                   cudaStream_t st) {
  DecodeArgs a = make_args(s, q, k_new, v_new, c, o_parts, lse_parts, fm);
  a.cache_len = cache_len;
  a.chunk = p.chunk;
  a.spb = p.spb;
  a.n_ctx = p.n_ctx;
  NoVarlen dv;
  dv.n = 0;
  return dispatch(s, a, dv, dim3(p.n_splits, s.b * s.hkv), p.n_splits, p.chunk, s.L, s.b,
                  c.num_pages, kc, vc, st);
}

int64_t plan_decode_varlen(const Shape& s, const int64_t* cu_ctx, const int64_t* cache_lens,
                           int64_t target_ctas, DecVarlen* dv, int64_t* max_splits,
                           int64_t* max_chunk) {
  const int64_t total = cu_ctx[s.b];
  const int64_t ctx_ctas = target_ctas - static_cast<int64_t>(s.b) * s.hkv;
  int64_t C = ctx_ctas > 0 ? (total * s.hkv + ctx_ctas - 1) / ctx_ctas : total;
  if (C < kTile) C = kTile;  // at least one TMA tile of keys per split
  dv->n = s.b;
  int64_t splits = 0, ctas = 0;
  *max_splits = 1;
  *max_chunk = kTile;
  for (int i = 0; i < s.b; ++i) {
    const int64_t L = cu_ctx[i + 1] - cu_ctx[i];
    int64_t spb = 1, n_ctx = 0;
    if (L > 0) {
      const int64_t B = s.B < L ? s.B : L;
      spb = (B + C - 1) / C;
      n_ctx = (L + B - 1) / B * spb;
      const int64_t chunk = (B + spb - 1) / spb;
      if (chunk > *max_chunk) *max_chunk = chunk;
    }
    const int64_t ns = n_ctx + 1;
    if (ns > *max_splits) *max_splits = ns;
    dv->cta0[i] = static_cast<int32_t>(ctas);
    dv->split0[i] = static_cast<int32_t>(splits);
    dv->ctx0[i] = static_cast<int32_t>(cu_ctx[i]);
    dv->spb[i] = static_cast<int32_t>(spb);
    dv->cache_len[i] = static_cast<int32_t>(cache_lens[i]);
    splits += ns;
    ctas += ns * s.hkv;
    if (ctas > 0x7fffffffLL) return -1;
  }
  dv->cta0[s.b] = static_cast<int32_t>(ctas);
  dv->split0[s.b] = static_cast<int32_t>(splits);
  dv->ctx0[s.b] = static_cast<int32_t>(total);
  return splits;
}

cudaError_t launch_decode_varlen(const Shape& s, const DecVarlen& dv, int64_t max_splits,
                                 int64_t max_chunk, const void* q, const void* k_new,
                                 const void* v_new, const void* kc, const void* vc,
                                 const CacheRef& c, float* o_parts, float* lse_parts,
                                 const FusedMerge& fm, cudaStream_t st) {
  DecodeArgs a = make_args(s, q, k_new, v_new, c, o_parts, lse_parts, &fm);
  return dispatch(s, a, dv, dim3(dv.cta0[s.b]), max_splits, max_chunk, dv.ctx0[s.b], 1,
                  c.num_pages, kc, vc, st);
}

bool decode_varlen_fused_fits(const Shape& s, int64_t max_splits, int64_t max_chunk) {
  return fused_merge_fits(max_splits, s.group(), s.d, decode_stages(max_chunk));
}

}  // namespace star
