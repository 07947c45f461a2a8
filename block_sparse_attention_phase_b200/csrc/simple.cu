// Straightforward CUDA kernels for both phases, one warp per output row.
//
// Each lane owns D/32 consecutive elements of the row's query and output; for
// every visible key the warp forms the dot product with a shuffle reduction and
// applies a running-max softmax update in fp32. They compute final outputs
// directly (no split/merge), which makes them an independent GPU
// implementation to cross-check the fast kernels at sizes the CPU oracle cannot
// cover. Visibility follows the Star Attention pages: Phase 1 sees the anchor
// b_0 plus its own block up to itself (hotaipapers.com page, Phase 1
// paragraph); Phase 2 sees every context key plus the cached rows up to itself
// (same page, Phase 2 paragraph).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int kWarps = 8;

template <int D>
struct RowAcc {
  static constexpr int E = D / 32;
  float q[E];
  float acc[E];
  float m = -INFINITY;
  float l = 0.f;

  __device__ void load_q(const __nv_bfloat16* qrow, int lane, float scale_log2) {
#pragma unroll
    for (int e = 0; e < E; ++e) q[e] = __bfloat162float(qrow[lane * E + e]) * scale_log2;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
  }

  // One key: s = q.k in log2 units, running max m, running sum l.
  __device__ void add(const __nv_bfloat16* krow, const __nv_bfloat16* vrow, int lane) {
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) part += q[e] * __bfloat162float(krow[lane * E + e]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    const float m_new = fmaxf(m, part);
    const float alpha = exp2f(m - m_new);  // m = -inf on the first key gives 0
    const float p = exp2f(part - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] * alpha + p * __bfloat162float(vrow[lane * E + e]);
    m = m_new;
  }

  __device__ void store(__nv_bfloat16* orow, float* lse_out, int lane) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) orow[lane * E + e] = __float2bfloat16_rn(acc[e] * inv);
    if (lse_out && lane == 0) {
      *lse_out = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }
};

template <int D>
__global__ void __launch_bounds__(kWarps * 32) simple_phase1_kernel(
    Shape s, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t total = static_cast<int64_t>(s.b) * s.hq * s.L;
  if (row >= total) return;
  // row enumerates (b, h, t) with t fastest so that a block's warps share keys.
  const int64_t t = row % s.L;
  const int h = static_cast<int>((row / s.L) % s.hq);
  const int bb = static_cast<int>(row / (s.L * s.hq));
  const int kvh = h / s.group();
  const float scale_log2 = s.scale * 1.4426950408889634f;

  RowAcc<D> r;
  r.load_q(q + ((static_cast<int64_t>(bb) * s.L + t) * s.hq + h) * D, lane, scale_log2);
  const int64_t blk0 = (t / s.B) * s.B;
  auto kv_at = [&](int64_t j) { return ((static_cast<int64_t>(bb) * s.L + j) * s.hkv + kvh) * D; };
  if (blk0 > 0) {
    for (int64_t j = 0; j < s.B; ++j) r.add(k + kv_at(j), v + kv_at(j), lane);  // anchor b_0
  }
  for (int64_t j = blk0; j <= t; ++j) r.add(k + kv_at(j), v + kv_at(j), lane);  // own block, causal
  r.store(o + ((static_cast<int64_t>(bb) * s.L + t) * s.hq + h) * D,
          lse ? lse + (static_cast<int64_t>(bb) * s.hq + h) * s.L + t : nullptr, lane);
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) simple_phase2_kernel(
    Shape s, const __nv_bfloat16* __restrict__ q, int64_t rows,
    const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc,
    const __nv_bfloat16* __restrict__ kk, const __nv_bfloat16* __restrict__ vk, int64_t cap,
    int64_t vis_base, int causal, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t total = static_cast<int64_t>(s.b) * s.hq * rows;
  if (row >= total) return;
  const int64_t r_tok = row % rows;
  const int h = static_cast<int>((row / rows) % s.hq);
  const int bb = static_cast<int>(row / (rows * s.hq));
  const int kvh = h / s.group();
  const float scale_log2 = s.scale * 1.4426950408889634f;

  RowAcc<D> r;
  r.load_q(q + ((static_cast<int64_t>(bb) * rows + r_tok) * s.hq + h) * D, lane, scale_log2);
  for (int64_t j = 0; j < s.L; ++j) {
    const int64_t off = ((static_cast<int64_t>(bb) * s.L + j) * s.hkv + kvh) * D;
    r.add(kc + off, vc + off, lane);
  }
  const int64_t last = vis_base + (causal ? r_tok : 0);  // inclusive
  for (int64_t j = 0; j <= last && j < cap; ++j) {
    const int64_t off = ((static_cast<int64_t>(bb) * cap + j) * s.hkv + kvh) * D;
    r.add(kk + off, vk + off, lane);
  }
  r.store(o + ((static_cast<int64_t>(bb) * rows + r_tok) * s.hq + h) * D,
          lse ? lse + (static_cast<int64_t>(bb) * s.hq + h) * rows + r_tok : nullptr, lane);
}

// Varlen cache write (the uniform query pass appends its rows inside the partial
// kernel): sequence i's rows [0, e0[i+1] - e0[i]) of its cache (its query rows,
// then zeros up to the end of the tile or page) come from packed rows q0[i] .. of
// k, v [total, Hkv, d]; e0 is the prefix of those row counts. A contiguous cache is
// [seqs, cap, Hkv, d]; a paged one puts row r of sequence i in row r % P of page
// table[i * max_pages + r / P] of a [pages, P, Hkv, d] pool. A page id outside
// [0, num_pages) is refused: the bounds flag is set and nothing is written.
struct CacheRows {
  int32_t n;
  int32_t q0[kMaxVarSeqs + 1];
  int32_t e0[kMaxVarSeqs + 1];
};

__global__ void cache_write_varlen_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                          int32_t hkv, int32_t d, uint4* __restrict__ kc,
                                          uint4* __restrict__ vc, int64_t cap,
                                          const int32_t* __restrict__ table, int32_t P,
                                          int32_t max_pages, int32_t num_pages, uint32_t* status,
                                          const __grid_constant__ CacheRows cr) {
  const int64_t per_row = static_cast<int64_t>(hkv) * d / 8;
  const int64_t total = static_cast<int64_t>(cr.e0[cr.n]) * per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i % per_row;
    const int64_t gr = i / per_row;
    int lo = 0, hi = cr.n;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cr.e0[mid] <= gr) lo = mid; else hi = mid;
    }
    const int64_t r = gr - cr.e0[lo];
    const int64_t rows = cr.q0[lo + 1] - cr.q0[lo];
    int64_t drow = static_cast<int64_t>(lo) * cap + r;
    if (table) {
      const int64_t page = table[static_cast<int64_t>(lo) * max_pages + r / P];
      if (page < 0 || page >= num_pages) {
        atomicOr(status, kBoundsFlag);
        continue;
      }
      drow = page * P + r % P;
    }
    const int64_t dst = drow * per_row + e;
    if (r < rows) {
      const int64_t src = (cr.q0[lo] + r) * per_row + e;
      kc[dst] = k[src];
      vc[dst] = v[src];
    } else {
      kc[dst] = make_uint4(0u, 0u, 0u, 0u);
      vc[dst] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

}  // namespace

cudaError_t launch_cache_write_varlen(const Shape& s, const int64_t* cu_q, const void* k,
                                      const void* v, const CacheRef& c, cudaStream_t st) {
  CacheRows cr;
  cr.n = s.b;
  int64_t ext_total = 0;
  for (int i = 0; i < s.b; ++i) {
    cr.q0[i] = static_cast<int32_t>(cu_q[i]);
    cr.e0[i] = static_cast<int32_t>(ext_total);
    const int64_t rows = cu_q[i + 1] - cu_q[i];
    // zero-fill to the end of the page (paged) or of the 128-row tile (contiguous,
    // within the capacity), so the query pass's cache tiles read zeros past the rows
    int64_t ext = rows;
    if (c.paged()) {
      ext = (rows + c.page_size - 1) / c.page_size * c.page_size;
    } else {
      ext = (rows + 127) / 128 * 128;
      if (ext > c.cap) ext = c.cap;
    }
    ext_total += ext;
  }
  cr.q0[s.b] = static_cast<int32_t>(cu_q[s.b]);
  cr.e0[s.b] = static_cast<int32_t>(ext_total);
  const int64_t total = ext_total * s.hkv * s.d / 8;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks64 = (total + threads - 1) / threads;
  const unsigned blocks = static_cast<unsigned>(blocks64 < 4096 ? blocks64 : 4096);
  cache_write_varlen_kernel<<<blocks, threads, 0, st>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), s.hkv, s.d,
      static_cast<uint4*>(c.k), static_cast<uint4*>(c.v), c.cap, c.page_table, c.page_size,
      c.max_pages, c.num_pages, device_status_word(), cr);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_simple_phase1(const Shape& s, const void* q, const void* k, const void* v,
                                 void* o, float* lse, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(s.b) * s.hq * s.L;
  const dim3 grid(static_cast<unsigned>((rows + kWarps - 1) / kWarps));
  auto* qq = static_cast<const __nv_bfloat16*>(q);
  auto* kk = static_cast<const __nv_bfloat16*>(k);
  auto* vv = static_cast<const __nv_bfloat16*>(v);
  auto* oo = static_cast<__nv_bfloat16*>(o);
  if (s.d == 128)
    simple_phase1_kernel<128><<<grid, kWarps * 32, 0, st>>>(s, qq, kk, vv, oo, lse);
  else
    simple_phase1_kernel<64><<<grid, kWarps * 32, 0, st>>>(s, qq, kk, vv, oo, lse);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_simple_phase2(const Shape& s, const void* q, int64_t rows, const void* kc,
                                 const void* vc, const void* kk, const void* vk, int64_t cap,
                                 int64_t vis_base, int causal, void* o, float* lse,
                                 cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(s.b) * s.hq * rows;
  const dim3 grid(static_cast<unsigned>((n + kWarps - 1) / kWarps));
  auto* qq = static_cast<const __nv_bfloat16*>(q);
  auto* a = static_cast<const __nv_bfloat16*>(kc);
  auto* b = static_cast<const __nv_bfloat16*>(vc);
  auto* c = static_cast<const __nv_bfloat16*>(kk);
  auto* dd = static_cast<const __nv_bfloat16*>(vk);
  auto* oo = static_cast<__nv_bfloat16*>(o);
  if (s.d == 128)
    simple_phase2_kernel<128><<<grid, kWarps * 32, 0, st>>>(s, qq, rows, a, b, c, dd, cap,
                                                            vis_base, causal, oo, lse);
  else
    simple_phase2_kernel<64><<<grid, kWarps * 32, 0, st>>>(s, qq, rows, a, b, c, dd, cap,
                                                           vis_base, causal, oo, lse);
  count_launch();
  return cudaGetLastError();
}


}  // namespace star
