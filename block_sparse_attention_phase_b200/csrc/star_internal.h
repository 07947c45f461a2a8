// Internal interface between the C-ABI layer (star_attn_capi.cpp) and the
// kernel launchers in the .cu files. Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#if defined(__CUDACC__)
#define STAR_HD __host__ __device__
#else
#define STAR_HD
#endif

namespace star {

// Flags kernels OR into the device status word (they never trap).
constexpr uint32_t kTimeoutFlag = 1u;  // a bounded wait ran out
constexpr uint32_t kBoundsFlag = 2u;   // a bounds check refused an access

// The status "word" is the first of kStatusWords 32-bit words. The rest hold the
// record of the first index a debug build's checks refused (builds with
// -DSTAR_DEBUG): [1] violations so far, [2] source line of the check, [3] unused,
// [4..5] the index, [6..7] its limit (64-bit, low word first).
constexpr int kStatusWords = 8;

struct Shape {
  int32_t b, hq, hkv, d;
  int64_t L, B;
  float scale;  // resolved softmax scale (> 0)
  STAR_HD int64_t n_blocks() const { return (L + B - 1) / B; }
  STAR_HD int32_t group() const { return hq / hkv; }
};

// Split plan of a Phase-2 pass: every context block is cut into `spb` chunks of
// at most `chunk` keys (a chunk never straddles two blocks); one more split
// covers the query-local cache.
struct SplitPlan {
  int32_t spb = 1;
  int64_t chunk = 1;
  int32_t n_ctx = 0;    // n_blocks * spb
  int32_t n_splits = 0; // n_ctx + 1
};

SplitPlan decode_plan(const Shape& s);
SplitPlan query_plan(const Shape& s, int64_t lq);
size_t partial_bytes(const Shape& s, const SplitPlan& p, int64_t rows);

// Counts kernel launches (host side); every launcher calls it once per launch.
void count_launch(uint64_t n = 1);

#if defined(__CUDACC__)
// Launch with programmatic stream serialisation: the kernel may begin while the
// previous kernel in the stream is still running; it must call pdl_wait() before
// touching anything that kernel writes or reads.
template <typename... Params, typename... Args>
cudaError_t launch_programmatic(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}
#endif

// Where the query-local cache rows live: one contiguous [b, cap, Hkv, d] buffer
// (page_table == nullptr), or pages of a pool [num_pages, page_size, Hkv, d] with
// page_table [b, max_pages].
struct CacheRef {
  void* k = nullptr;
  void* v = nullptr;
  int64_t cap = 0;               // contiguous: rows per sequence
  const int32_t* page_table = nullptr;
  int32_t page_size = 0, num_pages = 0, max_pages = 0;
  bool paged() const { return page_table != nullptr; }
};

// A varlen batch as the kernels see it (passed by value as a kernel parameter):
// sequence i owns work items [item0[i], item0[i+1]) and tokens
// [start[i], start[i+1]) of the packed tensors. n = 0: a uniform batch.
// The Phase-2 query pass of a varlen batch also uses: ctx0 (first context token of
// each sequence in the packed context), rbase (first partial token-row of each
// sequence: its splits' partials are [S_i, lq_i] token rows from there) and spb
// (chunks per context block).
constexpr int kMaxVarSeqs = 128;
struct VarSeqs {
  int32_t n;
  int32_t item0[kMaxVarSeqs + 1];
  int32_t start[kMaxVarSeqs + 1];
  int32_t ctx0[kMaxVarSeqs + 1];
  int32_t rbase[kMaxVarSeqs + 1];
  int32_t spb[kMaxVarSeqs];
};

// A varlen decode batch (kernel parameter): sequence i owns CTAs [cta0[i], cta0[i+1])
// (its splits x Hkv), partial rows [split0[i], split0[i+1]) (one per split; the last
// is its query-local cache), context tokens [ctx0[i], ctx0[i+1]) of the packed
// context, spb[i] chunks per context block, and cache_len[i] cached rows.
// n = 0: a uniform batch.
struct DecVarlen {
  int32_t n;
  int32_t cta0[kMaxVarSeqs + 1];
  int32_t split0[kMaxVarSeqs + 1];
  int32_t ctx0[kMaxVarSeqs + 1];
  int32_t spb[kMaxVarSeqs];
  int32_t cache_len[kMaxVarSeqs];
};

// Device status word of the current device (address valid on that device).
uint32_t* device_status_word();

// ---- launchers (return the launch's cudaError_t) ----
cudaError_t launch_simple_phase1(const Shape& s, const void* q, const void* k, const void* v,
                                 void* o, float* lse, cudaStream_t st);
cudaError_t launch_simple_phase2(const Shape& s, const void* q, int64_t rows, const void* kc,
                                 const void* vc, const void* kk, const void* vk, int64_t cap,
                                 int64_t vis_base, int causal, void* o, float* lse,
                                 cudaStream_t st);
// o: bf16 [b, tokens, heads, d], or fp32 with o_fp32.
cudaError_t launch_merge(const float* o_parts, const float* lse_parts, int32_t n_splits,
                         int32_t b, int64_t tokens, int32_t heads, int32_t d, void* o,
                         float* lse, cudaStream_t st, bool o_fp32 = false);
// Outputs of a decode step whose partial kernel also merges (the last CTA of each
// (sequence, kv-head) combines the splits); counters [b * Hkv] must be zero before
// the launch and are zero again after it.
struct FusedMerge {
  void* o;
  float* lse;
  uint32_t* counters;
};
cudaError_t launch_decode_partials(const Shape& s, const SplitPlan& p, const void* q,
                                   const void* k_new, const void* v_new, const void* kc,
                                   const void* vc, const CacheRef& c, int64_t cache_len,
                                   float* o_parts, float* lse_parts, const FusedMerge* fm,
                                   cudaStream_t st);
// Whether the fused merge's weights and sums fit in the decode kernel's shared memory.
bool decode_fused_fits(const Shape& s, const SplitPlan& p);
// Varlen decode: split plan (s.b sequences, packed context offsets cu_ctx and cache
// lengths, both host arrays) aiming at about target_ctas CTAs. Returns the total
// split count (partial rows), or -1 if the grid would be too large.
int64_t plan_decode_varlen(const Shape& s, const int64_t* cu_ctx, const int64_t* cache_lens,
                           int64_t target_ctas, DecVarlen* dv, int64_t* max_splits,
                           int64_t* max_chunk);
bool decode_varlen_fused_fits(const Shape& s, int64_t max_splits, int64_t max_chunk);
// One fused decode step over a varlen batch (always with the last-CTA merge).
cudaError_t launch_decode_varlen(const Shape& s, const DecVarlen& dv, int64_t max_splits,
                                 int64_t max_chunk, const void* q, const void* k_new,
                                 const void* v_new, const void* kc, const void* vc,
                                 const CacheRef& c, float* o_parts, float* lse_parts,
                                 const FusedMerge& fm, cudaStream_t st);
cudaError_t launch_phase1_sm100(const Shape& s, const void* q, const void* k, const void* v,
                                void* o, float* lse, cudaStream_t st);
// A host's share of Phase 1: q/k/v [b, L, H, d] hold whole blocks b_i.. (i > 0) of a
// longer context, the anchor b_0's K/V [b, B, Hkv, d] is a separate buffer; every
// local block attends to the anchor and causally to itself. s.B is not clamped to s.L.
cudaError_t launch_phase1_anchored(const Shape& s, const void* q, const void* k, const void* v,
                                   const void* k_anchor, const void* v_anchor, void* o, float* lse,
                                   cudaStream_t st);
// Phase 1 over a varlen batch: s.b sequences packed along tokens, s.L = total tokens,
// cu_seqlens (host) [s.b + 1]; o [total, Hq, d], lse [Hq, total].
cudaError_t launch_phase1_varlen(const Shape& s, const int64_t* cu_seqlens, const void* q,
                                 const void* k, const void* v, void* o, float* lse,
                                 cudaStream_t st);
// Phase-2 query tokens: partials + merge into o/lse. The cache split reads the query
// tokens' K/V from k_new/v_new [b, lq, Hkv, d]; with write_cache the partial kernel
// also appends them to the cache c (rows [0, lq), zeros to the end of a paged
// cache's last page).
cudaError_t launch_query_path(const Shape& s, const SplitPlan& p, const void* q,
                              const void* k_new, const void* v_new, int64_t lq,
                              const void* kc, const void* vc, const CacheRef& c, float* o_parts,
                              float* lse_parts, void* o, float* lse, cudaStream_t st,
                              bool o_fp32, bool write_cache);
// RoPE on q [b, L, Hq, d] and k [b, L, Hkv, d] at positions pos0 + t (in place
// allowed); q_anchor (or null) gets q rotated at the anchor-variant positions.
cudaError_t launch_rope(const Shape& s, const float* inv_freq, int64_t pos0, const void* q_in,
                        const void* k_in, void* q_out, void* k_out, void* q_anchor,
                        cudaStream_t st);
// Phase 1 whose anchor tiles are scored with q_anchor instead of q.
cudaError_t launch_phase1_anchor_q(const Shape& s, const void* q, const void* q_anchor,
                                   const void* k, const void* v, void* o, float* lse,
                                   cudaStream_t st);
// Phase-2 query pass over a varlen batch: split plan (host offsets cu_ctx, cu_q),
// returning the partial token-rows needed (-1: too large) and filling vs.
int64_t plan_query_varlen(const Shape& s, const int64_t* cu_ctx, const int64_t* cu_q,
                          int64_t target_ctas, VarSeqs* vs);
cudaError_t launch_cache_write_varlen(const Shape& s, const int64_t* cu_q, const void* k,
                                      const void* v, const CacheRef& c, cudaStream_t st);
// Partials (after the cache write) and the varlen merge into o [total_q, Hq, d],
// lse [Hq, total_q].
cudaError_t launch_query_varlen(const Shape& s, const VarSeqs& vs, const void* q,
                                const void* kc, const void* vc, const CacheRef& c,
                                float* o_parts, float* lse_parts, void* o, float* lse,
                                cudaStream_t st);
cudaError_t launch_merge_varlen(const float* o_parts, const float* lse_parts, const VarSeqs& vs,
                                int64_t block_size, int32_t heads, int32_t d, void* o, float* lse,
                                cudaStream_t st);
cudaError_t launch_selftest_wait(uint64_t wait_ns, cudaStream_t st);
// Whether this library was built with -DSTAR_DEBUG (index checks on every store).
bool debug_build();
// Checks index n against limit n in a tiny kernel (out: device, n + 1 words).
cudaError_t launch_selftest_bounds(uint32_t* out, int64_t n, cudaStream_t st);
cudaError_t launch_selftest_exp2(const float* x, float* y, int64_t n, cudaStream_t st);
cudaError_t launch_selftest_read(const void* src, int64_t bytes, uint32_t* sink, int32_t ctas,
                                 cudaStream_t st);

// TMA descriptor encoding (host). Returns false if the driver entry point is
// unavailable or the encode call rejects the arguments.
// 4-D bf16 tensor [batch][token_rows][heads][d] viewed as (inner0 = d, dim1 =
// heads, dim2 = tokens, dim3 = batch), box (box0, box1, box2, 1). Only the first
// `tokens` of the `token_rows` rows per sequence are in bounds: a box reaching
// past them reads zeros.
bool encode_tma_bf16_4d(void* tmap_out, const void* base, uint64_t d, uint64_t heads,
                        uint64_t tokens, uint64_t token_rows, uint64_t batch, uint32_t box0,
                        uint32_t box1, uint32_t box2, bool swizzle128);

// 128-row query tiles of the Phase-2 query pass (rows = query tokens x GQA heads).
int64_t query_tiles(const Shape& s, int64_t lq);

}  // namespace star
