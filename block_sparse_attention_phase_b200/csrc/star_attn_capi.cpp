// C-ABI layer: argument validation, Phase-2 split planning, workspace sizing and
// launch sequencing. Nothing here computes attention; every step of the path
// runs in the kernels of the .cu files.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/star_attn.h"
#include "star_internal.h"

namespace star {
namespace {

#ifndef STAR_DECODE_CTAS_PER_SM
#define STAR_DECODE_CTAS_PER_SM 2
#endif
constexpr int kDecodeCtasPerSM = STAR_DECODE_CTAS_PER_SM;
constexpr int64_t kMinChunk = 64;      // one TMA tile of keys

// Streaming multiprocessors of the current device, read once per device; 148 (a
// B200) when no device can be queried, e.g. for workspace sizing on a host
// without a GPU.
constexpr int kMaxDevices = 64;
constexpr int kDefaultSMs = 148;
std::atomic<int> g_sm_count[kMaxDevices];

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();  // a failed query must not linger as the next call's error
    return kDefaultSMs;
  }
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return kDefaultSMs;
  }
  g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// LSE outputs are written one float at a time: 4-byte alignment is enough.
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

star_status_t resolve(const star_attn_shape_t* in, Shape* out) {
  if (!in) return STAR_ERR_INVALID_ARG;
  if (in->batch < 1 || in->num_q_heads < 1 || in->num_kv_heads < 1 || in->ctx_len < 1 ||
      in->block_size < 1)
    return STAR_ERR_INVALID_ARG;
  if (in->num_q_heads % in->num_kv_heads != 0) return STAR_ERR_INVALID_ARG;
  if (!(in->softmax_scale == in->softmax_scale)) return STAR_ERR_INVALID_ARG;  // NaN
  if (in->head_dim != 64 && in->head_dim != 128) return STAR_ERR_UNSUPPORTED;
  const int G = in->num_q_heads / in->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return STAR_ERR_UNSUPPORTED;
  if (in->ctx_len > (int64_t{1} << 31) - 1) return STAR_ERR_UNSUPPORTED;  // TMA coordinates
  out->b = in->batch;
  out->hq = in->num_q_heads;
  out->hkv = in->num_kv_heads;
  out->d = in->head_dim;
  out->L = in->ctx_len;
  out->B = in->block_size < in->ctx_len ? in->block_size : in->ctx_len;
  out->scale = in->softmax_scale > 0.f ? in->softmax_scale
                                       : static_cast<float>(1.0 / std::sqrt(double(in->head_dim)));
  return STAR_OK;
}

star_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? STAR_OK : STAR_ERR_CUDA; }

SplitPlan make_plan(const Shape& s, int64_t target_ctas) {
  SplitPlan p;
  const int64_t n = s.n_blocks();
  const int64_t units = static_cast<int64_t>(s.b) * s.hkv;
  int64_t per_unit = target_ctas / units - 1;  // context splits wanted per (batch, kv-head)
  int64_t spb = per_unit / n;
  if (spb < 1) spb = 1;
  int64_t chunk = (s.B + spb - 1) / spb;
  if (chunk < kMinChunk) {
    chunk = kMinChunk;
    spb = (s.B + chunk - 1) / chunk;
  }
  p.spb = static_cast<int32_t>(spb);
  p.chunk = chunk;
  p.n_ctx = static_cast<int32_t>(n * spb);
  p.n_splits = p.n_ctx + 1;
  return p;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Host offsets of a varlen batch: cu[0] = 0, non-decreasing, cu[n] = total.
bool valid_offsets(const int64_t* cu, int n, int64_t total) {
  if (cu[0] != 0 || cu[n] != total) return false;
  for (int i = 0; i < n; ++i)
    if (cu[i + 1] < cu[i]) return false;
  return true;
}

int64_t varlen_target_ctas() { return int64_t{sm_count()} * kDecodeCtasPerSM; }

// Varlen decode workspace = [o_parts][lse_parts][counters: b * Hkv uint32], each
// 256-B aligned; partial rows = the plan's splits.
size_t varlen_decode_bytes(const Shape& s, const int64_t* cu_ctx) {
  std::vector<int64_t> zeros(static_cast<size_t>(s.b), 0);
  DecVarlen dv;
  int64_t max_splits = 0, max_chunk = 0;
  const int64_t splits = plan_decode_varlen(s, cu_ctx, zeros.data(), varlen_target_ctas(), &dv,
                                            &max_splits, &max_chunk);
  if (splits < 0) return 0;
  const size_t per = static_cast<size_t>(splits) * s.hq;
  return align256(per * s.d * sizeof(float)) + align256(per * sizeof(float)) +
         align256(static_cast<size_t>(s.b) * s.hkv * 4);
}

// Page-pool arguments: a tile (128 query-pass rows, 64 decode rows) must never
// straddle two pages, and TMA coordinates of a page are 32-bit.
star_status_t check_pages(int32_t page_size, int32_t num_pages, const int32_t* page_table,
                          int32_t max_pages) {
  if (page_size < 128 || page_size % 128 != 0) return STAR_ERR_INVALID_ARG;
  if (num_pages < 1 || max_pages < 1 || !page_table) return STAR_ERR_INVALID_ARG;
  if (!aligned4(page_table)) return STAR_ERR_INVALID_ARG;
  return STAR_OK;
}

CacheRef paged_ref(void* k, void* v, int32_t page_size, int32_t num_pages,
                   const int32_t* page_table, int32_t max_pages) {
  CacheRef c;
  c.k = k;
  c.v = v;
  c.page_table = page_table;
  c.page_size = page_size;
  c.num_pages = num_pages;
  c.max_pages = max_pages;
  return c;
}

// Workspace = [o_parts (256-B aligned)][lse_parts].
float* lse_parts_of(void* workspace, const Shape& s, const SplitPlan& p, int64_t rows) {
  const size_t per = static_cast<size_t>(p.n_splits) * s.b * rows * s.hq;
  return reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                  align256(per * s.d * sizeof(float)));
}

// Phase-2 query pass on validated arguments: partials (whose kernel also appends the
// query K/V to the cache) + merge.
star_status_t run_query(const Shape& s, const void* q, const void* k, const void* v,
                        int64_t query_len, const void* k_ctx, const void* v_ctx,
                        const CacheRef& c, void* o, float* lse, void* workspace,
                        cudaStream_t cs) {
  const SplitPlan plan = query_plan(s, query_len);
  const cudaError_t e =
      launch_query_path(s, plan, q, k, v, query_len, k_ctx, v_ctx, c, static_cast<float*>(workspace),
                        lse_parts_of(workspace, s, plan, query_len), o, lse, cs, false, true);
  return e == cudaSuccess ? STAR_OK : STAR_ERR_CUDA;
}

// Phase-2 decode step on validated arguments: partials (with the append) + merge.
star_status_t run_decode(const Shape& s, const void* q, const void* k, const void* v,
                         const void* k_ctx, const void* v_ctx, const CacheRef& c,
                         int64_t cache_len, void* o, float* lse, void* workspace,
                         cudaStream_t cs) {
  const SplitPlan plan = decode_plan(s);
  float* o_parts = static_cast<float*>(workspace);
  float* lse_parts = lse_parts_of(workspace, s, plan, 1);
  cudaError_t e = launch_decode_partials(s, plan, q, k, v, k_ctx, v_ctx, c, cache_len, o_parts,
                                         lse_parts, nullptr, cs);
  if (e != cudaSuccess) return STAR_ERR_CUDA;
  e = launch_merge(o_parts, lse_parts, plan.n_splits, s.b, 1, s.hq, s.d, o, lse, cs);
  return e == cudaSuccess ? STAR_OK : STAR_ERR_CUDA;
}

// Fused decode workspace = [o_parts][lse_parts][counters: b * Hkv uint32].
size_t fused_decode_bytes(const Shape& s) {
  return partial_bytes(s, decode_plan(s), 1) + align256(static_cast<size_t>(s.b) * s.hkv * 4);
}

std::atomic<uint64_t> g_launches{0};

}  // namespace

void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

star_status_t check_shape(const star_attn_shape_t* shape) {
  Shape s;
  return resolve(shape, &s);
}

SplitPlan decode_plan(const Shape& s) { return make_plan(s, int64_t{sm_count()} * kDecodeCtasPerSM); }

SplitPlan query_plan(const Shape& s, int64_t lq) {
  // One tensor-core CTA per SM, each taking two q-tiles; aim at about one wave
  // over (splits x pairs of q-tiles): a CTA's time is set by its K/V tiles, so
  // longer chunks in one wave beat shorter ones in two, and the fp32 partials
  // (one per split) halve.
  const int64_t pairs = (query_tiles(s, lq) + 1) / 2;
  return make_plan(s, int64_t{sm_count()} / pairs);
}

size_t partial_bytes(const Shape& s, const SplitPlan& p, int64_t rows) {
  const size_t per = static_cast<size_t>(p.n_splits) * s.b * rows * s.hq;
  return align256(per * s.d * sizeof(float)) + align256(per * sizeof(float));
}

}  // namespace star

using star::Shape;

extern "C" {

STAR_ATTN_API uint64_t star_attn_launch_count(void) {
  return star::g_launches.load(std::memory_order_relaxed);
}

STAR_ATTN_API const char* star_attn_version(void) { return "star-attn-b200 0.1 (sm_100a)"; }

STAR_ATTN_API const char* star_attn_status_string(star_status_t st) {
  switch (st) {
    case STAR_OK: return "ok";
    case STAR_ERR_INVALID_ARG: return "invalid argument";
    case STAR_ERR_UNSUPPORTED: return "unsupported shape";
    case STAR_ERR_WORKSPACE: return "workspace missing or too small";
    case STAR_ERR_CACHE_FULL: return "query-local cache full";
    case STAR_ERR_CUDA: return "CUDA error";
    case STAR_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

STAR_ATTN_API size_t star_attn_workspace_bytes(const star_attn_shape_t* shape, int32_t phase,
                                               int64_t rows) {
  Shape s;
  if (star::resolve(shape, &s) != STAR_OK) return 0;
  switch (phase) {
    case STAR_PHASE1: return 0;
    case STAR_PHASE2_QUERY:
      if (rows < 1) return 0;
      return star::partial_bytes(s, star::query_plan(s, rows), rows);
    case STAR_PHASE2_DECODE: return star::partial_bytes(s, star::decode_plan(s), 1);
    case STAR_PHASE2_DECODE_FUSED: return star::fused_decode_bytes(s);
    default: return 0;
  }
}

STAR_ATTN_API star_status_t star_attn_phase1(const star_attn_shape_t* shape, const void* q,
                                             const void* k, const void* v, void* o, float* lse,
                                             star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (!q || !k || !v || !o) return STAR_ERR_INVALID_ARG;
  if (!star::aligned16(q) || !star::aligned16(k) || !star::aligned16(v) || !star::aligned16(o) ||
      !star::aligned4(lse))
    return STAR_ERR_INVALID_ARG;
  return star::cuda_status(
      star::launch_phase1_sm100(s, q, k, v, o, lse, reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_phase1_anchored(const star_attn_shape_t* shape,
                                                      const void* q, const void* k, const void* v,
                                                      const void* k_anchor, const void* v_anchor,
                                                      void* o, float* lse, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  s.B = shape->block_size;  // the global block size: also the anchor's length
  if (s.B > (int64_t{1} << 31) - 1) return STAR_ERR_UNSUPPORTED;
  if (!q || !k || !v || !k_anchor || !v_anchor || !o) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_anchor, v_anchor, o};
  for (const void* p : ptrs)
    if (!star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse)) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_phase1_anchored(s, q, k, v, k_anchor, v_anchor, o, lse,
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_rope(const star_attn_shape_t* shape,
                                           const float* inv_freq, int64_t pos0, const void* q_in,
                                           const void* k_in, void* q_out, void* k_out,
                                           void* q_anchor, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (!inv_freq || !q_in || !k_in || !q_out || !k_out || pos0 < 0) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q_in, k_in, q_out, k_out};
  for (const void* p : ptrs)
    if (!star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (q_anchor && !star::aligned16(q_anchor)) return STAR_ERR_INVALID_ARG;
  for (int f = 0; f < s.d / 2; ++f)
    if (!(inv_freq[f] >= 0.f) || inv_freq[f] > 1e30f) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_rope(s, inv_freq, pos0, q_in, k_in, q_out, k_out, q_anchor,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_phase1_anchor_q(const star_attn_shape_t* shape,
                                                      const void* q, const void* q_anchor,
                                                      const void* k, const void* v, void* o,
                                                      float* lse, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (!q || !q_anchor || !k || !v || !o) return STAR_ERR_INVALID_ARG;
  if (!star::aligned16(q) || !star::aligned16(q_anchor) || !star::aligned16(k) ||
      !star::aligned16(v) || !star::aligned16(o) || !star::aligned4(lse))
    return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_phase1_anchor_q(s, q, q_anchor, k, v, o, lse,
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_phase1_varlen(const star_attn_shape_t* shape,
                                                    const int64_t* cu_seqlens, const void* q,
                                                    const void* k, const void* v, void* o,
                                                    float* lse, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (!cu_seqlens || !q || !k || !v || !o) return STAR_ERR_INVALID_ARG;
  if (s.b > star::kMaxVarSeqs) return STAR_ERR_UNSUPPORTED;
  if (cu_seqlens[0] != 0 || cu_seqlens[s.b] != s.L) return STAR_ERR_INVALID_ARG;
  for (int i = 0; i < s.b; ++i)
    if (cu_seqlens[i + 1] < cu_seqlens[i]) return STAR_ERR_INVALID_ARG;
  if (!star::aligned16(q) || !star::aligned16(k) || !star::aligned16(v) || !star::aligned16(o) ||
      !star::aligned4(lse))
    return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_phase1_varlen(s, cu_seqlens, q, k, v, o, lse,
                                                      reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_phase2_query(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    int64_t query_len, const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache,
    int64_t cache_capacity, void* o, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (query_len < 1 || cache_capacity < 1) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_cache, v_cache, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  if (query_len > cache_capacity) return STAR_ERR_CACHE_FULL;
  const size_t need = star::partial_bytes(s, star::query_plan(s, query_len), query_len);
  if (!workspace || workspace_bytes < need) return STAR_ERR_WORKSPACE;
  star::CacheRef c;
  c.k = k_cache;
  c.v = v_cache;
  c.cap = cache_capacity;
  return star::run_query(s, q, k, v, query_len, k_ctx, v_ctx, c, o, lse, workspace,
                         reinterpret_cast<cudaStream_t>(stream));
}

STAR_ATTN_API star_status_t star_attn_phase2_decode(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, void* o, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (cache_len < 0 || cache_capacity < 1) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_cache, v_cache, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  if (cache_len + 1 > cache_capacity) return STAR_ERR_CACHE_FULL;
  if (!workspace || workspace_bytes < star::partial_bytes(s, star::decode_plan(s), 1))
    return STAR_ERR_WORKSPACE;
  star::CacheRef c;
  c.k = k_cache;
  c.v = v_cache;
  c.cap = cache_capacity;
  return star::run_decode(s, q, k, v, k_ctx, v_ctx, c, cache_len, o, lse, workspace,
                          reinterpret_cast<cudaStream_t>(stream));
}

STAR_ATTN_API star_status_t star_attn_phase2_decode_fused(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, void* o, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (cache_len < 0 || cache_capacity < 1) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_cache, v_cache, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  if (cache_len + 1 > cache_capacity) return STAR_ERR_CACHE_FULL;
  if (!workspace || workspace_bytes < star::fused_decode_bytes(s)) return STAR_ERR_WORKSPACE;
  const star::SplitPlan plan = star::decode_plan(s);
  star::CacheRef c;
  c.k = k_cache;
  c.v = v_cache;
  c.cap = cache_capacity;
  if (!star::decode_fused_fits(s, plan))  // very many splits: partials + merge kernel
    return star::run_decode(s, q, k, v, k_ctx, v_ctx, c, cache_len, o, lse, workspace,
                            reinterpret_cast<cudaStream_t>(stream));
  const size_t parts = star::partial_bytes(s, plan, 1);
  star::FusedMerge fm;
  fm.o = o;
  fm.lse = lse;
  fm.counters = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + parts);
  return star::cuda_status(star::launch_decode_partials(
      s, plan, q, k, v, k_ctx, v_ctx, c, cache_len, static_cast<float*>(workspace),
      star::lse_parts_of(workspace, s, plan, 1), &fm, reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API size_t star_attn_decode_varlen_workspace_bytes(const star_attn_shape_t* shape,
                                                             const int64_t* cu_ctx) {
  Shape s;
  if (star::resolve(shape, &s) != STAR_OK || !cu_ctx || s.b > star::kMaxVarSeqs) return 0;
  if (!star::valid_offsets(cu_ctx, s.b, s.L)) return 0;
  return star::varlen_decode_bytes(s, cu_ctx);
}

STAR_ATTN_API star_status_t star_attn_phase2_decode_varlen(
    const star_attn_shape_t* shape, const int64_t* cu_ctx, const int64_t* cache_lens,
    const void* q, const void* k, const void* v, const void* k_ctx, const void* v_ctx,
    void* k_cache, void* v_cache, int64_t cache_capacity, const int32_t* page_table,
    int32_t page_size, int32_t num_pages, int32_t max_pages, void* o, float* lse,
    void* workspace, size_t workspace_bytes, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (s.b > star::kMaxVarSeqs) return STAR_ERR_UNSUPPORTED;
  if (!cu_ctx || !cache_lens || !star::valid_offsets(cu_ctx, s.b, s.L)) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_cache, v_cache, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  star::CacheRef c;
  if (page_table) {
    st = star::check_pages(page_size, num_pages, page_table, max_pages);
    if (st != STAR_OK) return st;
    c = star::paged_ref(k_cache, v_cache, page_size, num_pages, page_table, max_pages);
  } else {
    if (cache_capacity < 1) return STAR_ERR_INVALID_ARG;
    c.k = k_cache;
    c.v = v_cache;
    c.cap = cache_capacity;
  }
  for (int i = 0; i < s.b; ++i) {
    if (cache_lens[i] < 0 || cache_lens[i] > (int64_t{1} << 30)) return STAR_ERR_INVALID_ARG;
    if (page_table ? cache_lens[i] / page_size + 1 > max_pages : cache_lens[i] + 1 > cache_capacity)
      return STAR_ERR_CACHE_FULL;
  }
  star::DecVarlen dv;
  int64_t max_splits = 0, max_chunk = 0;
  const int64_t splits = star::plan_decode_varlen(s, cu_ctx, cache_lens, star::varlen_target_ctas(),
                                                  &dv, &max_splits, &max_chunk);
  if (splits < 0 || !star::decode_varlen_fused_fits(s, max_splits, max_chunk))
    return STAR_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < star::varlen_decode_bytes(s, cu_ctx)) return STAR_ERR_WORKSPACE;
  const size_t per = static_cast<size_t>(splits) * s.hq;
  char* ws = static_cast<char*>(workspace);
  float* o_parts = reinterpret_cast<float*>(ws);
  float* lse_parts = reinterpret_cast<float*>(ws + star::align256(per * s.d * sizeof(float)));
  star::FusedMerge fm;
  fm.o = o;
  fm.lse = lse;
  fm.counters = reinterpret_cast<uint32_t*>(ws + star::align256(per * s.d * sizeof(float)) +
                                            star::align256(per * sizeof(float)));
  return star::cuda_status(star::launch_decode_varlen(s, dv, max_splits, max_chunk, q, k, v,
                                                      k_ctx, v_ctx, c, o_parts, lse_parts, fm,
                                                      reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API size_t star_attn_query_varlen_workspace_bytes(const star_attn_shape_t* shape,
                                                            const int64_t* cu_ctx,
                                                            const int64_t* cu_q) {
  Shape s;
  if (star::resolve(shape, &s) != STAR_OK || !cu_ctx || !cu_q || s.b > star::kMaxVarSeqs) return 0;
  if (!star::valid_offsets(cu_ctx, s.b, s.L) || !star::valid_offsets(cu_q, s.b, cu_q[s.b])) return 0;
  star::VarSeqs vs;
  const int64_t rows = star::plan_query_varlen(s, cu_ctx, cu_q, star::varlen_target_ctas(), &vs);
  if (rows < 0) return 0;
  const size_t per = static_cast<size_t>(rows) * s.hq;
  return star::align256(per * s.d * sizeof(float)) + star::align256(per * sizeof(float));
}

STAR_ATTN_API star_status_t star_attn_phase2_query_varlen(
    const star_attn_shape_t* shape, const int64_t* cu_ctx, const int64_t* cu_q, const void* q,
    const void* k, const void* v, const void* k_ctx, const void* v_ctx, void* k_cache,
    void* v_cache, int64_t cache_capacity, const int32_t* page_table, int32_t page_size,
    int32_t num_pages, int32_t max_pages, void* o, float* lse, void* workspace,
    size_t workspace_bytes, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (s.b > star::kMaxVarSeqs) return STAR_ERR_UNSUPPORTED;
  if (!cu_ctx || !cu_q || !star::valid_offsets(cu_ctx, s.b, s.L) ||
      !star::valid_offsets(cu_q, s.b, cu_q[s.b]))
    return STAR_ERR_INVALID_ARG;
  if (cu_q[s.b] > (int64_t{1} << 31) - 1) return STAR_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_cache, v_cache, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  star::CacheRef c;
  if (page_table) {
    st = star::check_pages(page_size, num_pages, page_table, max_pages);
    if (st != STAR_OK) return st;
    c = star::paged_ref(k_cache, v_cache, page_size, num_pages, page_table, max_pages);
  } else {
    if (cache_capacity < 1) return STAR_ERR_INVALID_ARG;
    c.k = k_cache;
    c.v = v_cache;
    c.cap = cache_capacity;
  }
  for (int i = 0; i < s.b; ++i) {
    const int64_t lq = cu_q[i + 1] - cu_q[i];
    if (page_table ? (lq + page_size - 1) / page_size > max_pages : lq > cache_capacity)
      return STAR_ERR_CACHE_FULL;
  }
  star::VarSeqs vs;
  const int64_t rows = star::plan_query_varlen(s, cu_ctx, cu_q, star::varlen_target_ctas(), &vs);
  if (rows < 0) return STAR_ERR_UNSUPPORTED;
  const size_t per = static_cast<size_t>(rows) * s.hq;
  if (!workspace || workspace_bytes < star::align256(per * s.d * sizeof(float)) +
                                          star::align256(per * sizeof(float)))
    return STAR_ERR_WORKSPACE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = star::launch_cache_write_varlen(s, cu_q, k, v, c, cs);
  if (e != cudaSuccess) return STAR_ERR_CUDA;
  float* o_parts = static_cast<float*>(workspace);
  float* lse_parts = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                              star::align256(per * s.d * sizeof(float)));
  return star::cuda_status(
      star::launch_query_varlen(s, vs, q, k_ctx, v_ctx, c, o_parts, lse_parts, o, lse, cs));
}

STAR_ATTN_API star_status_t star_attn_phase2_partial(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v, int64_t rows,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, float* o32, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream) {
  const bool has_ctx = k_ctx != nullptr;
  const bool has_cache = k_cache != nullptr;
  if (!shape || (!has_ctx && !has_cache) || rows < 1) return STAR_ERR_INVALID_ARG;
  star_attn_shape_t sh = *shape;
  if (!has_ctx) sh.ctx_len = 1;  // no context keys on this rank (the plan gets none)
  Shape s;
  star_status_t st = star::resolve(&sh, &s);
  if (st != STAR_OK) return st;
  if (!q || !o32 || !lse || !star::aligned16(q) || !star::aligned16(o32) || !star::aligned4(lse))
    return STAR_ERR_INVALID_ARG;
  if (has_ctx && (!v_ctx || !star::aligned16(k_ctx) || !star::aligned16(v_ctx)))
    return STAR_ERR_INVALID_ARG;
  if (has_cache) {
    const void* ptrs[] = {k, v, k_cache, v_cache};
    for (const void* p : ptrs)
      if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
    if (cache_capacity < 1 || cache_len < 0) return STAR_ERR_INVALID_ARG;
    if (rows == 1 ? cache_len + 1 > cache_capacity : rows > cache_capacity) return STAR_ERR_CACHE_FULL;
  }
  if (!star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  star::SplitPlan plan = rows == 1 ? star::decode_plan(s) : star::query_plan(s, rows);
  if (!has_ctx) {
    plan.spb = 1;
    plan.chunk = 1;
    plan.n_ctx = 0;
    plan.n_splits = 1;
  } else if (!has_cache) {
    plan.n_splits = plan.n_ctx;
  }
  const size_t need = star::partial_bytes(s, plan, rows);
  if (!workspace || workspace_bytes < need) return STAR_ERR_WORKSPACE;
  // Stand-ins for an absent context or cache: valid buffers whose maps no split uses.
  star::CacheRef c;
  c.k = has_cache ? k_cache : const_cast<void*>(k_ctx);
  c.v = has_cache ? v_cache : const_cast<void*>(v_ctx);
  c.cap = has_cache ? cache_capacity : s.L;
  const void* kc = has_ctx ? k_ctx : k_cache;
  const void* vc = has_ctx ? v_ctx : v_cache;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  float* o_parts = static_cast<float*>(workspace);
  float* lse_parts = star::lse_parts_of(workspace, s, plan, rows);
  cudaError_t e;
  if (rows == 1) {
    e = star::launch_decode_partials(s, plan, q, has_cache ? k : q, has_cache ? v : q, kc, vc, c,
                                     has_cache ? cache_len : 0, o_parts, lse_parts, nullptr, cs);
    if (e != cudaSuccess) return STAR_ERR_CUDA;
    e = star::launch_merge(o_parts, lse_parts, plan.n_splits, s.b, 1, s.hq, s.d, o32, lse, cs, true);
  } else {
    e = star::launch_query_path(s, plan, q, has_cache ? k : nullptr, has_cache ? v : nullptr, rows, kc,
                                vc, c, o_parts, lse_parts, o32, lse, cs, true, has_cache);
  }
  return star::cuda_status(e);
}

STAR_ATTN_API star_status_t star_attn_phase2_query_paged(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    int64_t query_len, const void* k_ctx, const void* v_ctx, void* k_pages, void* v_pages,
    int32_t page_size, int32_t num_pages, const int32_t* page_table, int32_t max_pages, void* o,
    float* lse, void* workspace, size_t workspace_bytes, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (query_len < 1) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_pages, v_pages, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  st = star::check_pages(page_size, num_pages, page_table, max_pages);
  if (st != STAR_OK) return st;
  if ((query_len + page_size - 1) / page_size > max_pages) return STAR_ERR_CACHE_FULL;
  const size_t need = star::partial_bytes(s, star::query_plan(s, query_len), query_len);
  if (!workspace || workspace_bytes < need) return STAR_ERR_WORKSPACE;
  const star::CacheRef c = star::paged_ref(k_pages, v_pages, page_size, num_pages, page_table,
                                           max_pages);
  return star::run_query(s, q, k, v, query_len, k_ctx, v_ctx, c, o, lse, workspace,
                         reinterpret_cast<cudaStream_t>(stream));
}

STAR_ATTN_API star_status_t star_attn_phase2_decode_paged(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_pages, void* v_pages, int32_t page_size,
    int32_t num_pages, const int32_t* page_table, int32_t max_pages, int64_t cache_len, void* o,
    float* lse, void* workspace, size_t workspace_bytes, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (cache_len < 0) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_pages, v_pages, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if (!star::aligned4(lse) || !star::aligned16(workspace)) return STAR_ERR_INVALID_ARG;
  st = star::check_pages(page_size, num_pages, page_table, max_pages);
  if (st != STAR_OK) return st;
  if (cache_len / page_size + 1 > max_pages) return STAR_ERR_CACHE_FULL;
  if (!workspace || workspace_bytes < star::partial_bytes(s, star::decode_plan(s), 1))
    return STAR_ERR_WORKSPACE;
  const star::CacheRef c = star::paged_ref(k_pages, v_pages, page_size, num_pages, page_table,
                                           max_pages);
  return star::run_decode(s, q, k, v, k_ctx, v_ctx, c, cache_len, o, lse, workspace,
                          reinterpret_cast<cudaStream_t>(stream));
}

STAR_ATTN_API star_status_t star_attn_lse_merge(const float* o_parts, const float* lse_parts,
                                                int32_t num_splits, int32_t batch,
                                                int64_t tokens, int32_t heads, int32_t head_dim,
                                                void* o, float* lse, star_stream_t stream) {
  if (!o_parts || !lse_parts || !o) return STAR_ERR_INVALID_ARG;
  if (num_splits < 1 || batch < 1 || tokens < 1 || heads < 1) return STAR_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return STAR_ERR_UNSUPPORTED;
  if (!star::aligned16(o_parts) || !star::aligned16(o)) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_merge(o_parts, lse_parts, num_splits, batch, tokens,
                                              heads, head_dim, o, lse,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_simple_phase1(const star_attn_shape_t* shape,
                                                    const void* q, const void* k, const void* v,
                                                    void* o, float* lse, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (!q || !k || !v || !o) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_simple_phase1(s, q, k, v, o, lse,
                                                      reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_simple_phase2(
    const star_attn_shape_t* shape, const void* q, int64_t rows, const void* k_ctx,
    const void* v_ctx, const void* k_cache, const void* v_cache, int64_t cache_capacity,
    int64_t cache_visible_base, int32_t causal, void* o, float* lse, star_stream_t stream) {
  Shape s;
  star_status_t st = star::resolve(shape, &s);
  if (st != STAR_OK) return st;
  if (!q || !k_ctx || !v_ctx || !k_cache || !v_cache || !o || rows < 1 || cache_capacity < 1 ||
      cache_visible_base < 0)
    return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_simple_phase2(
      s, q, rows, k_ctx, v_ctx, k_cache, v_cache, cache_capacity, cache_visible_base, causal, o,
      lse, reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_get_device_status(star_stream_t stream) {
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return STAR_ERR_CUDA;
  uint32_t* word = star::device_status_word();
  if (!word) return STAR_ERR_CUDA;
  uint32_t flags = 0;
  if (cudaMemcpy(&flags, word, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess)
    return STAR_ERR_CUDA;
  if (flags) {
    const uint32_t zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return STAR_ERR_CUDA;
  }
  if (flags & star::kTimeoutFlag) return STAR_ERR_TIMEOUT;
  if (flags) return STAR_ERR_CUDA;
  return STAR_OK;
}

STAR_ATTN_API int32_t star_attn_debug_build(void) { return star::debug_build() ? 1 : 0; }

STAR_ATTN_API star_status_t star_attn_debug_record(int64_t* out, star_stream_t stream) {
  if (!out) return STAR_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return STAR_ERR_CUDA;
  uint32_t* word = star::device_status_word();
  if (!word) return STAR_ERR_CUDA;
  uint32_t rec[star::kStatusWords] = {};
  if (cudaMemcpy(rec, word, sizeof(rec), cudaMemcpyDeviceToHost) != cudaSuccess) return STAR_ERR_CUDA;
  out[0] = rec[1];
  out[1] = rec[2];
  out[2] = static_cast<int64_t>(static_cast<uint64_t>(rec[4]) | (static_cast<uint64_t>(rec[5]) << 32));
  out[3] = static_cast<int64_t>(static_cast<uint64_t>(rec[6]) | (static_cast<uint64_t>(rec[7]) << 32));
  if (rec[1]) {  // clear the record (the flags word stays for star_attn_get_device_status)
    const uint32_t zero[star::kStatusWords - 1] = {};
    if (cudaMemcpy(word + 1, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return STAR_ERR_CUDA;
  }
  return STAR_OK;
}

STAR_ATTN_API star_status_t star_attn_selftest_bounds(void* out, int64_t n, star_stream_t stream) {
  if (!out || n < 0 || !star::aligned4(out)) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_selftest_bounds(static_cast<uint32_t*>(out), n,
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_selftest_exp2(const float* x, float* y, int64_t n,
                                                    star_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(
      star::launch_selftest_exp2(x, y, n, reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_selftest_read(const void* src, size_t bytes,
                                                    uint32_t* sink, int32_t ctas,
                                                    star_stream_t stream) {
  if (!src || !sink || bytes == 0 || bytes % 16 != 0 || ctas < 1 || ctas > (1 << 20))
    return STAR_ERR_INVALID_ARG;
  if (!star::aligned16(src) || !star::aligned4(sink)) return STAR_ERR_INVALID_ARG;
  if (bytes > (size_t{1} << 40)) return STAR_ERR_INVALID_ARG;
  return star::cuda_status(star::launch_selftest_read(src, static_cast<int64_t>(bytes), sink, ctas,
                                                      reinterpret_cast<cudaStream_t>(stream)));
}

STAR_ATTN_API star_status_t star_attn_selftest_wait_timeout(uint64_t wait_ns,
                                                            star_stream_t stream) {
  if (wait_ns < 1000000ull) wait_ns = 1000000ull;
  if (wait_ns > 2000000000ull) wait_ns = 2000000000ull;
  return star::cuda_status(
      star::launch_selftest_wait(wait_ns, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
