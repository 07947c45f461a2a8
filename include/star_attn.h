/*
 * star_attn.h — C ABI of the B200 (sm_100a) Star Attention two-phase attention library.
 *
 * The method is Star Attention ("Star Attention: Efficient LLM Inference over
 * Long Sequences", Acharya, Jia, Ginsburg; ICML 2025). On one GPU the pages'
 * "hosts" become context blocks resident in HBM:
 *
 *   Phase 1 (context prefill): the context of L tokens is cut into blocks
 *     b_0..b_{n-1} of B tokens (n = ceil(L/B), the last block may be short).
 *     Block b_0 runs plain causal attention; every block b_i, i > 0, runs causal
 *     attention over [anchor = b_0 ; b_i] and keeps only its own rows
 *     (hotaipapers.com page, Phase 1 paragraph; rebuttal to reviewer EMsM,
 *     "Size of Anchor Block"). The anchor is read in place from b_0's K/V.
 *   Phase 2 (query and decode): each query or decoded token attends to every
 *     cached token. Every context block returns a partial output and its
 *     log-sum-exp; the partials are merged exactly (hotaipapers.com page, Phase 2
 *     paragraph). The query tokens' K/V and each decoded token's K/V are
 *     appended to a query-local cache.
 *
 * Conventions for every call
 *   - Q/K/V/O are bf16, contiguous, token-major: [batch, tokens, heads, head_dim].
 *   - LSE outputs are fp32 [batch, num_q_heads, rows], natural log of the sum of
 *     exp(softmax_scale * q.k) over the row's visible keys.
 *   - GQA: q-head h reads kv-head h / (num_q_heads / num_kv_heads).
 *   - All pointers are device pointers owned by the caller and must be 16-byte
 *     aligned, except LSE outputs, which need 4-byte alignment. The library
 *     never allocates device memory and never frees a caller's buffer; any
 *     scratch it needs is the caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *     Arguments are checked on the host before anything is launched; an invalid
 *     call returns an error and launches nothing. No C++ exception crosses the ABI.
 *   - Kernels never trap. A device-side wait that runs out (about one second)
 *     records a flag that star_attn_get_device_status() reports.
 */
#ifndef STAR_ATTN_H_
#define STAR_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define STAR_ATTN_API __attribute__((visibility("default")))
#else
#define STAR_ATTN_API
#endif

/* Same type as cudaStream_t, declared here so that this header needs no CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st* star_stream_t;

typedef enum {
  STAR_OK = 0,
  STAR_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, inconsistent shape */
  STAR_ERR_UNSUPPORTED = 2,  /* a shape the library does not implement (head_dim not 64/128, GQA group not 1/2/4/8) */
  STAR_ERR_WORKSPACE = 3,    /* workspace missing or smaller than star_attn_workspace_bytes() */
  STAR_ERR_CACHE_FULL = 4,   /* the query-local cache has no room for the rows to append */
  STAR_ERR_CUDA = 5,         /* a CUDA runtime call or a kernel launch failed */
  STAR_ERR_TIMEOUT = 6       /* a bounded device-side wait ran out (see get_device_status) */
} star_status_t;

/* Problem shape shared by all calls. */
typedef struct {
  int32_t batch;          /* sequences, >= 1; every sequence has the same ctx_len */
  int32_t num_q_heads;    /* Hq >= 1 */
  int32_t num_kv_heads;   /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t head_dim;       /* d: 64 or 128 */
  int64_t ctx_len;        /* L >= 1 context tokens */
  int64_t block_size;     /* B >= 1; also the anchor size (rebuttal to EMsM) */
  float softmax_scale;    /* <= 0 selects 1/sqrt(head_dim) */
} star_attn_shape_t;

/* Phase selectors for star_attn_workspace_bytes(). */
enum { STAR_PHASE1 = 1, STAR_PHASE2_QUERY = 2, STAR_PHASE2_DECODE = 3,
       STAR_PHASE2_DECODE_FUSED = 4 };

/*
 * Workspace (device scratch) a call needs, in bytes; 0 if none.
 * phase: STAR_PHASE1, STAR_PHASE2_QUERY (rows = query_len), STAR_PHASE2_DECODE or
 * STAR_PHASE2_DECODE_FUSED (rows ignored). The workspace holds the per-split fp32
 * partial outputs and LSEs of Phase 2 before they are merged (and, for the fused
 * decode, one 32-bit counter per (sequence, kv-head)). Returns 0 for an invalid
 * shape.
 */
STAR_ATTN_API size_t star_attn_workspace_bytes(const star_attn_shape_t* shape, int32_t phase,
                                               int64_t rows);

/*
 * Phase 1: anchor-prefixed blockwise-local causal attention over the context
 * (hotaipapers.com page, Phase 1 paragraph; rebuttal to EMsM, "Size of Anchor
 * Block"; rebuttal to x5MA, "Anchor Block Content and Position").
 *
 * For token t of block b_i (i = t / B) the visible keys are b_0 (all of it,
 * if i > 0) and the tokens of b_i up to t:
 *   o[t]   = sum_j softmax_j(scale * q_t . k_j) v_j,   lse[t] = ln sum_j exp(scale * q_t . k_j)
 * q [batch, L, Hq, d]; k, v [batch, L, Hkv, d]  (inputs, read only; k and v of
 *   every block are kept by the caller as that block's KV cache)
 * o [batch, L, Hq, d] bf16 (output, round-to-nearest-even from fp32)
 * lse [batch, Hq, L] fp32 (output) or NULL.
 * Needs no workspace.
 */
STAR_ATTN_API star_status_t star_attn_phase1(const star_attn_shape_t* shape, const void* q,
                                             const void* k, const void* v, void* o, float* lse,
                                             star_stream_t stream);

/*
 * One host's share of Phase 1 in the multi-host form (hotaipapers.com page,
 * Phase 1 paragraph: every host runs its blocks with the anchor b_0 in front;
 * rebuttal to reviewer dnhh: no communication in Phase 1 beyond giving every
 * host the anchor). The caller's context is a run of whole blocks b_i .. b_k of
 * a longer context with i > 0 (the last may be short), and b_0's K/V arrive as
 * separate buffers. Every local block attends to the whole anchor and causally to
 * itself, exactly the rows star_attn_phase1() computes for those blocks over the
 * whole context; the anchor is read where it lies and never copied next to the
 * blocks, and no anchor row is computed.
 *   shape->ctx_len: this host's tokens L; shape->block_size: the global block size
 *     B, which is also the anchor's length (B may exceed L: one short block).
 *   q [batch, L, Hq, d]; k, v [batch, L, Hkv, d]: this host's blocks.
 *   k_anchor, v_anchor [batch, B, Hkv, d]: b_0's K and V (read only).
 *   o [batch, L, Hq, d] bf16; lse [batch, Hq, L] fp32 or NULL.
 * Needs no workspace. Errors as star_attn_phase1().
 */
STAR_ATTN_API star_status_t star_attn_phase1_anchored(const star_attn_shape_t* shape,
                                                      const void* q, const void* k, const void* v,
                                                      const void* k_anchor, const void* v_anchor,
                                                      void* o, float* lse, star_stream_t stream);

/*
 * Rotary position embedding of a layer's projected q [batch, L, Hq, d] and
 * k [batch, L, Hkv, d] (the model step before Phase 1 and Phase 2), at positions
 * pos0 + t for token t (Phase 1: pos0 = 0; the query tokens: pos0 = L; decode step
 * n: pos0 = L + Lq + n with L = 1 in the shape). Rotate-half pairs: frequency f <
 * d/2 rotates (x[f], x[f + d/2]) by the angle position * inv_freq[f].
 *   inv_freq: HOST float [d/2] (the model's frequencies, scaling included).
 *   q_out, k_out may equal q_in, k_in (in place).
 *   q_anchor (or NULL): q rotated at the positions of the anchor-position variant
 *     of Phase 1 (rebuttal to x5MA, "Anchor Block Content and Position"): the
 *     anchor tokens of block i >= 1 placed right before the block, at positions
 *     (i-1)B .. iB-1. RoPE scores depend only on position differences, so this is
 *     q of token t rotated at t - (i-1)B (block 0: at t); pass it to
 *     star_attn_phase1_anchor_q(). Uses shape->block_size.
 */
STAR_ATTN_API star_status_t star_attn_rope(const star_attn_shape_t* shape,
                                           const float* inv_freq, int64_t pos0, const void* q_in,
                                           const void* k_in, void* q_out, void* k_out,
                                           void* q_anchor, star_stream_t stream);

/*
 * Phase 1 with the anchor's position IDs moved next to each block: identical to
 * star_attn_phase1() except that every block i >= 1 scores the anchor's keys with
 * q_anchor (from star_attn_rope()) instead of q; its own block's keys use q.
 * The kept K/V (the blocks' caches) are unchanged: the keys stay rotated at
 * their own positions, as Phase 2 needs.
 */
STAR_ATTN_API star_status_t star_attn_phase1_anchor_q(const star_attn_shape_t* shape,
                                                      const void* q, const void* q_anchor,
                                                      const void* k, const void* v, void* o,
                                                      float* lse, star_stream_t stream);

/*
 * Phase 1 over a varlen batch: shape->batch sequences of different lengths,
 * packed back to back along the token axis; each sequence is its own context
 * with its own blocks and its own anchor (its first block), exactly as if it
 * were run alone through star_attn_phase1() with batch 1.
 *   cu_seqlens: HOST array of batch + 1 int64 offsets, cu_seqlens[0] = 0,
 *     non-decreasing, cu_seqlens[batch] = shape->ctx_len (the total token count).
 *     Sequence i is tokens [cu_seqlens[i], cu_seqlens[i+1]); empty sequences are
 *     allowed. Read during the call only.
 *   A sequence shorter than block_size is one block (plain causal attention).
 * q [total, Hq, d]; k, v [total, Hkv, d]; o [total, Hq, d]; lse [Hq, total] or NULL.
 * Errors: STAR_ERR_UNSUPPORTED for more than 128 sequences; STAR_ERR_INVALID_ARG
 * for offsets that are not as above.
 * No counterpart on the pages (serving-side batching of documents of different
 * lengths; the per-sequence computation is Phase 1's).
 */
STAR_ATTN_API star_status_t star_attn_phase1_varlen(const star_attn_shape_t* shape,
                                                    const int64_t* cu_seqlens, const void* q,
                                                    const void* k, const void* v, void* o,
                                                    float* lse, star_stream_t stream);

/*
 * Phase 2, query tokens (abstract: query tokens attend to all prior cached
 * tokens; hotaipapers.com page, Phase 2 paragraph).
 *
 * Writes the query tokens' k, v into cache rows [0, query_len) and computes,
 * for query token j, attention over all L context keys and cache rows 0..j.
 * Each context block contributes a partial (o_s, lse_s); the query-local cache
 * contributes a causal partial; they are merged as in star_attn_lse_merge().
 *   q [batch, Lq, Hq, d]; k, v [batch, Lq, Hkv, d]   query tokens (inputs)
 *   k_ctx, v_ctx [batch, L, Hkv, d]                   Phase-1 context KV (inputs)
 *   k_cache, v_cache [batch, cache_capacity, Hkv, d]  query-local cache (rows 0..Lq-1 written)
 *   o [batch, Lq, Hq, d] bf16, lse [batch, Hq, Lq] fp32 or NULL (outputs)
 *   workspace: at least star_attn_workspace_bytes(shape, STAR_PHASE2_QUERY, query_len) bytes.
 * Errors: STAR_ERR_CACHE_FULL if query_len > cache_capacity.
 */
STAR_ATTN_API star_status_t star_attn_phase2_query(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    int64_t query_len, const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache,
    int64_t cache_capacity, void* o, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream);

/*
 * Phase 2, one decode step (hotaipapers.com page, Phase 2 paragraph: the query
 * host appends the new token's KV to its cache and the token attends globally).
 *
 * Appends k, v at cache row cache_len, then computes attention of q over all L
 * context keys and cache rows 0..cache_len (its own new key included), as a
 * split-KV pass over every block plus the cache, merged exactly.
 *   q [batch, 1, Hq, d]; k, v [batch, 1, Hkv, d]      new token (inputs)
 *   k_ctx, v_ctx [batch, L, Hkv, d]                    context KV (inputs)
 *   k_cache, v_cache [batch, cache_capacity, Hkv, d]   rows 0..cache_len-1 valid; row cache_len written
 *   o [batch, 1, Hq, d] bf16, lse [batch, Hq, 1] fp32 or NULL (outputs)
 *   workspace: at least star_attn_workspace_bytes(shape, STAR_PHASE2_DECODE, 1) bytes.
 * Errors: STAR_ERR_CACHE_FULL if cache_len + 1 > cache_capacity.
 */
STAR_ATTN_API star_status_t star_attn_phase2_decode(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, void* o, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream);

/*
 * star_attn_phase2_decode() in ONE kernel launch: the split-KV partial kernel also
 * does the exact merge (hotaipapers.com page, Phase 2 paragraph: the query host
 * aggregates one vector and one scalar per block). Every CTA stores its partial
 * and counts itself on a per-(sequence, kv-head) counter; the CTA that completes
 * the count combines all splits of its GQA group and resets the counter.
 * Same arguments, results and errors as star_attn_phase2_decode(), except:
 *   workspace: at least star_attn_workspace_bytes(shape, STAR_PHASE2_DECODE_FUSED, 1)
 *     bytes, ALL ZERO before the first call that uses it (e.g. cudaMemsetAsync once
 *     after allocation). Each call leaves its counter words zero again, so steps
 *     can reuse the workspace without clearing it; a workspace that another call
 *     (query pass, unfused decode) has written must be zeroed again first.
 *   The result equals star_attn_phase2_decode()'s to fp32 rounding of the merge
 *     (summation order differs); it is deterministic.
 *   Shapes with so many splits that the merge would need more than four passes over
 *     the kernel's shared memory (hundreds of splits per sequence and kv-head, e.g.
 *     block sizes of a few tokens) run as partials + merge kernel, with the same
 *     results and without touching the counters.
 */
STAR_ATTN_API star_status_t star_attn_phase2_decode_fused(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, void* o, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream);

/*
 * One host's share of Phase 2 in the pages' multi-host form (hotaipapers.com page,
 * Phase 2 paragraph: the query goes to every host, each attends with its own keys
 * and sends back one vector and one scalar per query row; the query host also
 * holds the query-local cache). Computes, for `rows` query rows q [batch, rows, Hq, d],
 * softmax attention over this host's keys only and returns it ready for
 * star_attn_lse_merge() across hosts:
 *   o32 [batch, rows, Hq, d] fp32 (normalised over these keys), lse [batch, Hq, rows].
 * Keys: the context k_ctx, v_ctx [batch, shape->ctx_len, Hkv, d], all visible (NULL:
 * this host holds no context; shape->ctx_len is then ignored), and, on the query
 * host, the query-local cache k_cache, v_cache [batch, cache_capacity, Hkv, d] (NULL
 * elsewhere) with k, v [batch, rows, Hkv, d] the rows' own KV:
 *   rows == 1: a decode step, appended at cache_len, seeing cache rows 0..cache_len;
 *   rows > 1: the query tokens, written to cache rows [0, rows), row j seeing 0..j.
 *   workspace: star_attn_workspace_bytes(shape, rows == 1 ? STAR_PHASE2_DECODE :
 *     STAR_PHASE2_QUERY, rows) bytes (nothing needs to be zero).
 * Errors: STAR_ERR_INVALID_ARG if neither keys nor cache are given; CACHE_FULL as
 * for the single-host calls.
 */
STAR_ATTN_API star_status_t star_attn_phase2_partial(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v, int64_t rows,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, float* o32, float* lse, void* workspace, size_t workspace_bytes,
    star_stream_t stream);

/*
 * The Phase-2 query pass over a varlen batch: every sequence has its own context
 * length and its own number of query tokens. Same computation per sequence as
 * star_attn_phase2_query() with batch 1, in one cache write, one partial launch and
 * one merge launch.
 *   shape->batch = sequences (at most 128); shape->ctx_len = total context tokens.
 *   cu_ctx: HOST int64 [batch + 1] offsets of the packed context k_ctx, v_ctx
 *     [total_ctx, Hkv, d]; cu_q: HOST int64 [batch + 1] offsets of the packed query
 *     tokens q [total_q, Hq, d], k, v [total_q, Hkv, d] (both: first 0, non-decreasing).
 *   Cache: contiguous k_cache/v_cache [batch, cache_capacity, Hkv, d] (page_table
 *     NULL) or a page pool (page_table [batch, max_pages], page_size, num_pages), as
 *     in star_attn_phase2_decode_varlen(). Rows [0, lq_i) of sequence i's cache get
 *     its query tokens' KV; the rows after them up to the end of their 128-row tile
 *     (contiguous, within the capacity) or page (paged) are written with zeros.
 *   o [total_q, Hq, d] bf16; lse [Hq, total_q] or NULL.
 *   workspace: star_attn_query_varlen_workspace_bytes(shape, cu_ctx, cu_q) bytes.
 * Errors: STAR_ERR_CACHE_FULL if a sequence's query tokens do not fit its cache;
 * STAR_ERR_UNSUPPORTED for more than 128 sequences.
 */
STAR_ATTN_API size_t star_attn_query_varlen_workspace_bytes(const star_attn_shape_t* shape,
                                                            const int64_t* cu_ctx,
                                                            const int64_t* cu_q);

STAR_ATTN_API star_status_t star_attn_phase2_query_varlen(
    const star_attn_shape_t* shape, const int64_t* cu_ctx, const int64_t* cu_q, const void* q,
    const void* k, const void* v, const void* k_ctx, const void* v_ctx, void* k_cache,
    void* v_cache, int64_t cache_capacity, const int32_t* page_table, int32_t page_size,
    int32_t num_pages, int32_t max_pages, void* o, float* lse, void* workspace,
    size_t workspace_bytes, star_stream_t stream);

/*
 * One decode step over a varlen batch (continuous batching): every sequence has its
 * own context length and its own number of cached query-local rows. Same
 * computation per sequence as star_attn_phase2_decode() with batch 1, in one
 * launch, with the merge fused (last-CTA merge, as star_attn_phase2_decode_fused()).
 *   shape->batch = sequences (at most 128); shape->ctx_len = total context tokens.
 *   cu_ctx: HOST int64 [batch + 1] offsets of each sequence's context in the packed
 *     k_ctx, v_ctx [total, Hkv, d] (cu_ctx[0] = 0, non-decreasing, last = total;
 *     an empty context is allowed).
 *   cache_lens: HOST int64 [batch], rows already cached per sequence; the new
 *     token's KV is appended at row cache_lens[i] of sequence i.
 *   q [batch, 1, Hq, d]; k, v [batch, 1, Hkv, d]; o [batch, 1, Hq, d]; lse [batch, Hq, 1] or NULL.
 *   The query-local cache is either contiguous, k_cache/v_cache [batch, cache_capacity,
 *     Hkv, d] (page_table NULL; rows past a sequence's cached ones may hold any
 *     bytes), or a page pool as in star_attn_phase2_decode_paged() (page_table
 *     [batch, max_pages], page_size, num_pages; cache_capacity ignored).
 *   workspace: star_attn_decode_varlen_workspace_bytes(shape, cu_ctx) bytes, all zero
 *     before its first use; every call leaves it reusable for the same cu_ctx.
 * Errors: STAR_ERR_CACHE_FULL if a sequence has no room for its new row;
 * STAR_ERR_UNSUPPORTED for more than 128 sequences, or a plan whose merge does not
 * fit in shared memory (thousands of context blocks in one sequence).
 * No counterpart on the pages (a serving-side batch of sequences at different
 * lengths; the per-sequence computation is the Phase-2 decode step's).
 */
STAR_ATTN_API size_t star_attn_decode_varlen_workspace_bytes(const star_attn_shape_t* shape,
                                                             const int64_t* cu_ctx);

STAR_ATTN_API star_status_t star_attn_phase2_decode_varlen(
    const star_attn_shape_t* shape, const int64_t* cu_ctx, const int64_t* cache_lens,
    const void* q, const void* k, const void* v, const void* k_ctx, const void* v_ctx,
    void* k_cache, void* v_cache, int64_t cache_capacity, const int32_t* page_table,
    int32_t page_size, int32_t num_pages, int32_t max_pages, void* o, float* lse,
    void* workspace, size_t workspace_bytes, star_stream_t stream);

/*
 * Paged query-local cache (paperhub.cn page, the authors' response to Reviewer
 * dKGV, item 3 "Compatibility with Parallelism Methods and Serving Frameworks":
 * PagedAttention-style memory management applies within each host to its local
 * KV cache). Same computation as star_attn_phase2_query() /
 * star_attn_phase2_decode(); only where the cache rows live differs:
 *   k_pages, v_pages [num_pages, page_size, Hkv, d] bf16 — a pool shared by the batch;
 *   page_table [batch, max_pages] int32 (device) — cache row r of sequence b is row
 *     r % page_size of page page_table[b * max_pages + r / page_size].
 * page_size must be a positive multiple of 128 (a tile never straddles pages);
 * every page id a call touches must lie in [0, num_pages) and each sequence's pages
 * must be distinct. Rows past the valid ones in a sequence's last page are written
 * with zeros by these calls (the query call zero-fills the rest of the page holding
 * its last row; a decode step that starts a new page zero-fills that page), so the
 * pool needs no initialisation.
 * Errors: STAR_ERR_CACHE_FULL if the rows to append need more than max_pages pages;
 * STAR_ERR_INVALID_ARG for a bad page_size, num_pages or max_pages.
 * No counterpart on the pages beyond the reference to PagedAttention.
 */
STAR_ATTN_API star_status_t star_attn_phase2_query_paged(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    int64_t query_len, const void* k_ctx, const void* v_ctx, void* k_pages, void* v_pages,
    int32_t page_size, int32_t num_pages, const int32_t* page_table, int32_t max_pages, void* o,
    float* lse, void* workspace, size_t workspace_bytes, star_stream_t stream);

STAR_ATTN_API star_status_t star_attn_phase2_decode_paged(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_pages, void* v_pages, int32_t page_size,
    int32_t num_pages, const int32_t* page_table, int32_t max_pages, int64_t cache_len, void* o,
    float* lse, void* workspace, size_t workspace_bytes, star_stream_t stream);

/*
 * The decode step of star_attn_phase2_decode() for callers that cannot allocate
 * device memory where they decode (a serving runtime whose pooled allocator owns
 * all of the GPU's memory, code that must avoid the implicit synchronisation of
 * cudaMalloc/cudaFree, C callers with no allocator at hand). No counterpart on
 * the Star Attention pages: this is a deployment variant of the same step.
 *
 * Same arguments and results as star_attn_phase2_decode() minus the workspace:
 * the per-split partials go to a 4 MiB array compiled into the library (one per
 * GPU, held until the process exits). The call allocates nothing.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress) with that device current; make it before any
 *     stream capture.
 *   - Every call shares the array: calls that may overlap on one GPU (e.g. on
 *     two streams) race and must be ordered by the caller.
 *   - Returns STAR_ERR_WORKSPACE, launching nothing, when the shape's partials
 *     (star_attn_workspace_bytes(shape, STAR_PHASE2_DECODE, 1)) exceed 4 MiB.
 */
STAR_ATTN_API star_status_t star_attn_phase2_decode_noalloc(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, void* o, float* lse, star_stream_t stream);

/*
 * Exact merge of per-split attention partials (hotaipapers.com page, Phase 2
 * paragraph: every host sends one vector and one scalar to the query host).
 *   lse = M + ln sum_s exp(lse_s - M),  M = max_s lse_s
 *   o   = sum_s exp(lse_s - lse) o_s          (a split with lse_s = -inf weighs 0)
 * o_parts [num_splits, batch, tokens, heads, head_dim] fp32,
 * lse_parts [num_splits, batch, heads, tokens] fp32 (inputs);
 * o [batch, tokens, heads, head_dim] bf16, lse [batch, heads, tokens] fp32 or NULL (outputs).
 * head_dim: 64 or 128.
 */
STAR_ATTN_API star_status_t star_attn_lse_merge(const float* o_parts, const float* lse_parts,
                                                int32_t num_splits, int32_t batch,
                                                int64_t tokens, int32_t heads, int32_t head_dim,
                                                void* o, float* lse, star_stream_t stream);

/*
 * Straightforward CUDA kernels (one warp per output row, fp32) computing the
 * same three operations with final outputs directly. They are a second,
 * independent GPU implementation used to cross-check the fast kernels at sizes
 * the CPU oracle cannot cover; they are not the fast path.
 */
STAR_ATTN_API star_status_t star_attn_simple_phase1(const star_attn_shape_t* shape,
                                                    const void* q, const void* k, const void* v,
                                                    void* o, float* lse, star_stream_t stream);
STAR_ATTN_API star_status_t star_attn_simple_phase2(
    const star_attn_shape_t* shape, const void* q, int64_t rows, const void* k_ctx,
    const void* v_ctx, const void* k_cache, const void* v_cache, int64_t cache_capacity,
    int64_t cache_visible_base, int32_t causal, void* o, float* lse, star_stream_t stream);

/*
 * Synchronises `stream`, then returns STAR_ERR_TIMEOUT if any kernel on the
 * current device recorded an expired bounded wait since the previous call
 * (clearing the flag), STAR_ERR_CUDA if the stream reports a CUDA error, else
 * STAR_OK.
 */
STAR_ATTN_API star_status_t star_attn_get_device_status(star_stream_t stream);

/*
 * Debug builds. A library built with -DSTAR_DEBUG checks the index of every
 * global store its kernels compute against the size of the buffer it lands in
 * (outputs, partials, LSEs, cache rows). A refused index is not stored: the
 * kernel raises the bounds flag (star_attn_get_device_status() then returns
 * STAR_ERR_CUDA) and the first refusal is recorded. Nothing traps.
 *   star_attn_debug_build(): 1 for such a build, else 0.
 *   star_attn_debug_record(out, stream): synchronises `stream`, then returns the
 *     record of the current device and clears it: out[0] = refusals since the
 *     last call, out[1] = the source line of the check, out[2] = the index,
 *     out[3] = its limit (all 0 when nothing was refused, always so in other
 *     builds). out: HOST array of 4 int64.
 *   star_attn_selftest_bounds(out, n, stream): one thread checks index n against
 *     limit n (one past the end) with the kernels' check; a debug build records
 *     it and skips the store, another build stores out[n] = 1. out: device,
 *     n + 1 uint32 (4-byte aligned).
 * No counterpart on the Star Attention pages (the library's own test tooling).
 */
STAR_ATTN_API int32_t star_attn_debug_build(void);
STAR_ATTN_API star_status_t star_attn_debug_record(int64_t* out, star_stream_t stream);
STAR_ATTN_API star_status_t star_attn_selftest_bounds(void* out, int64_t n, star_stream_t stream);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a
 * shared-memory barrier nobody arrives at, with a limit of `wait_ns`
 * nanoseconds (clamped to [1 ms, 2 s]); the wait gives up, records the timeout
 * flag and the block exits normally. The caller then reads the flag with
 * star_attn_get_device_status(). Faults nothing and leaves the context usable.
 */
STAR_ATTN_API star_status_t star_attn_selftest_wait_timeout(uint64_t wait_ns,
                                                            star_stream_t stream);

/*
 * Self-test of the base-2 exponential the attention softmax evaluates on the FMA
 * pipe for part of its scores (range reduction to n + f, f in [-1/2, 1/2], and a
 * degree-3 polynomial for 2^f; relative error about 7.5e-5 where the result is a
 * normal float, x in (-125, 8]; below that the result is below 2^-124 and
 * inputs under -126 give a subnormal near 2^-126 rather than 0).
 * x, y: device arrays of n floats. No counterpart on the Star Attention pages.
 */
STAR_ATTN_API star_status_t star_attn_selftest_exp2(const float* x, float* y, int64_t n,
                                                    star_stream_t stream);

/*
 * Read-only streaming probe: reads every byte of `src` once with 1-D bulk
 * asynchronous copies (32 KB chunks, four in flight per block) into shared
 * memory, spread over `ctas` blocks of one warp (one block per SM is enough), and
 * writes one 32-bit XOR of the first word of each chunk a block received to
 * sink[block]. Timing it over a buffer much larger than L2 gives the rate at which
 * this GPU reads HBM when nothing is written back, the ceiling of a read-only
 * kernel such as the decode step (a copy-based bandwidth figure counts a read
 * and a write per byte). Measurement infrastructure; no counterpart on the Star
 * Attention pages.
 * src: device, 16-byte aligned; bytes: a positive multiple of 16 (<= 2^40);
 * sink: device array of `ctas` uint32 (4-byte aligned); ctas in [1, 2^20].
 * Returns STAR_ERR_INVALID_ARG (nothing launched) otherwise.
 */
STAR_ATTN_API star_status_t star_attn_selftest_read(const void* src, size_t bytes, uint32_t* sink,
                                                    int32_t ctas, star_stream_t stream);

/*
 * Number of kernels this library has launched in this process (all devices).
 * A host-side counter for accounting, incremented at every successful launch.
 */
STAR_ATTN_API uint64_t star_attn_launch_count(void);

STAR_ATTN_API const char* star_attn_status_string(star_status_t status);
STAR_ATTN_API const char* star_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STAR_ATTN_H_ */
