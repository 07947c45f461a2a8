// Exact merge of split-KV attention partials (the query host's aggregation in
// Star Attention's Phase 2: hotaipapers.com page, Phase 2 paragraph — every
// block returns one vector and one scalar).
//
// For one output row with partials (o_s, lse_s):
//   M = max_s lse_s,  W = sum_s exp(lse_s - M),  lse = M + ln W,
//   o = sum_s exp(lse_s - M) o_s / W
// A split whose lse_s is -inf (it saw no key) contributes nothing.
//
// One warp per output row (batch, token, head), eight rows per CTA. The lanes
// first take the splits' LSEs (32 at a time) for the maximum M and the weights
// exp(lse_s - M); each lane owns d/32 contiguous elements of the row and sums the
// splits' partial rows (coalesced 512- or 256-byte warp reads) in split order. The
// reads of the first eight splits go out with the LSE reads and each later group of
// eight while the one before is summed: the merge is bound by L2 latency, not
// bandwidth. Every partial is read once.
#include <cuda_bf16.h>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int kRowsPerCta = 8;
constexpr int kGroup = 8;  // partial rows of a warp in flight per group

// Varlen query pass: one row per (packed query token, head); the token's sequence
// (binary search in vs.start) gives its split count and partial rows: split s of
// sequence i holds token-rows rbase[i] + s * lq_i .. (o: [rows, H, D]; lse: H x lq_i
// per split). Outputs are packed: o [total, H, D], lse [H, total].
template <int D, bool kVarlen, class OutT>
__global__ void __launch_bounds__(kRowsPerCta * 32) merge_kernel(
    const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int32_t S, int32_t b,
    int64_t T, int32_t H, OutT* __restrict__ o, float* __restrict__ lse,
    const __grid_constant__ VarSeqs vs, int64_t block_size, int64_t rows, uint32_t* status) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  // Launched programmatically: wait until the kernel that wrote the partials has
  // finished, then let the next kernel in the stream start being scheduled (the
  // next decode step writes this workspace only after its own pdl_wait()).
  pdl_wait();
  pdl_launch_dependents();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + (threadIdx.x >> 5);
  if (row >= rows) return;
  // (bb, t, h) with h fastest; varlen: (packed token, h)
  const int h = static_cast<int>(row % H);
  int64_t lse_stride, lse_off, o_stride, o_off, out_o, out_lse;
  if constexpr (kVarlen) {
    const int64_t tg = row / H;
    int lo = 0, hi = vs.n;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (vs.start[mid] <= tg) lo = mid; else hi = mid;
    }
    const int64_t lq = vs.start[lo + 1] - vs.start[lo];
    const int64_t t = tg - vs.start[lo];
    const int64_t L = vs.ctx0[lo + 1] - vs.ctx0[lo];
    const int64_t B = block_size < L ? block_size : L;
    S = static_cast<int32_t>((L > 0 ? (L + B - 1) / B * vs.spb[lo] : 0) + 1);
    const int64_t r0 = vs.rbase[lo];
    lse_stride = lq * H;
    lse_off = r0 * H + static_cast<int64_t>(h) * lq + t;
    o_stride = lq * H * D;
    o_off = ((r0 + t) * H + h) * D + lane * E;
    out_o = (tg * H + h) * D + lane * E;
    out_lse = static_cast<int64_t>(h) * T + tg;  // T = total packed tokens
  } else {
    const int64_t t = (row / H) % T;
    const int bb = static_cast<int>(row / (static_cast<int64_t>(H) * T));
    // lse_parts[s][bb][h][t]; o_parts[s][bb][t][h][:]
    lse_stride = static_cast<int64_t>(b) * H * T;
    lse_off = (static_cast<int64_t>(bb) * H + h) * T + t;
    o_stride = static_cast<int64_t>(b) * T * H * D;
    o_off = ((static_cast<int64_t>(bb) * T + t) * H + h) * D + lane * E;
    out_o = o_off;
    out_lse = lse_off;
  }

  // Partial row of split sp: E contiguous floats per lane (one coalesced warp read).
  auto load_row = [&](int sp, float (&x)[E]) {
    const float* r = o_parts + static_cast<int64_t>(sp) * o_stride + o_off;
    if constexpr (E == 4) {
      const float4 v = *reinterpret_cast<const float4*>(r);
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(r);
      x[0] = v.x; x[1] = v.y;
    }
  };
  // The partial rows do not depend on the weights: the first kGroup of them are
  // requested together with the LSEs, and every later group while the previous one
  // is summed, so a row costs about one L2 round trip per kGroup splits.
  float xa[kGroup][E];
#pragma unroll
  for (int u = 0; u < kGroup; ++u)
    if (u < S) load_row(u, xa[u]);
  // M = max over splits (lanes over splits; lane k keeps the LSE of split k)
  const float lse0 = lane < S ? lse_parts[lane * lse_stride + lse_off] : -INFINITY;
  float M = lse0;
  for (int sp = lane + 32; sp < S; sp += 32) M = fmaxf(M, lse_parts[sp * lse_stride + lse_off]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

  float W = 0.f;  // this lane's share of sum_s exp(lse_s - M)
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < S; s0 += 32) {
      const int cnt = S - s0 < 32 ? S - s0 : 32;
      // lane k holds the weight of split s0 + k (0 for an empty split)
      const float lv = s0 == 0 ? lse0 : (lane < cnt ? lse_parts[(s0 + lane) * lse_stride + lse_off] : 0.f);
      const float w = lane < cnt ? expf(lv - M) : 0.f;
      W += w;
      for (int g = 0; g < cnt; g += kGroup) {
        float xb[kGroup][E];
        const int nx = s0 + g + kGroup;  // the next group (32 is a multiple of kGroup)
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
          if (nx + u < S) load_row(nx + u, xb[u]);
#pragma unroll
        for (int u = 0; u < kGroup; ++u) {
          if (g + u < cnt) {
            const float wu = __shfl_sync(0xffffffffu, w, g + u);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += wu * xa[u][e];
          }
        }
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
          if (nx + u < S) {
#pragma unroll
            for (int e = 0; e < E; ++e) xa[u][e] = xb[u][e];
          }
      }
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
  const float inv = W > 0.f ? 1.f / W : 0.f;
  // outputs: o [b, T, H, D] or [total, H, D]; lse [b, H, T] or [H, total]
  const int64_t out_tokens = kVarlen ? T : static_cast<int64_t>(b) * T;
  if (!STAR_IN_BOUNDS(status, out_o + E - 1, out_tokens * H * D)) return;
  OutT* dst = o + out_o;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if constexpr (sizeof(OutT) == 4) dst[e] = acc[e] * inv;
    else dst[e] = __float2bfloat16_rn(acc[e] * inv);
  }
  if (lse && lane == 0 && STAR_IN_BOUNDS(status, out_lse, out_tokens * H))
    lse[out_lse] = W > 0.f ? M + logf(W) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge(const float* o_parts, const float* lse_parts, int32_t n_splits,
                         int32_t b, int64_t tokens, int32_t heads, int32_t d, void* o,
                         float* lse, cudaStream_t st, bool o_fp32) {
  const int64_t rows = static_cast<int64_t>(b) * tokens * heads;
  if (rows == 0) return cudaSuccess;
  if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta));
  auto* oo = static_cast<__nv_bfloat16*>(o);
  auto* of = static_cast<float*>(o);
  VarSeqs vs;
  vs.n = 0;
  const dim3 blk(kRowsPerCta * 32);
  uint32_t* status = device_status_word();
  const int64_t none = 0;
  cudaError_t e;
  if (o_fp32)
    e = d == 128 ? launch_programmatic(merge_kernel<128, false, float>, grid, blk, 0, st, o_parts,
                                       lse_parts, n_splits, b, tokens, heads, of, lse, vs, none, rows, status)
                 : launch_programmatic(merge_kernel<64, false, float>, grid, blk, 0, st, o_parts,
                                       lse_parts, n_splits, b, tokens, heads, of, lse, vs, none, rows, status);
  else
    e = d == 128 ? launch_programmatic(merge_kernel<128, false, __nv_bfloat16>, grid, blk, 0, st,
                                       o_parts, lse_parts, n_splits, b, tokens, heads, oo, lse, vs,
                                       none, rows, status)
                 : launch_programmatic(merge_kernel<64, false, __nv_bfloat16>, grid, blk, 0, st,
                                       o_parts, lse_parts, n_splits, b, tokens, heads, oo, lse, vs,
                                       none, rows, status);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_merge_varlen(const float* o_parts, const float* lse_parts, const VarSeqs& vs,
                                int64_t block_size, int32_t heads, int32_t d, void* o, float* lse,
                                cudaStream_t st) {
  const int64_t total = vs.start[vs.n];
  const int64_t rows = total * heads;
  if (rows == 0) return cudaSuccess;
  if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta));
  auto* oo = static_cast<__nv_bfloat16*>(o);
  uint32_t* status = device_status_word();
  const cudaError_t e =
      d == 128 ? launch_programmatic(merge_kernel<128, true, __nv_bfloat16>, grid, dim3(kRowsPerCta * 32), 0,
                                     st, o_parts, lse_parts, 0, 1, total, heads, oo, lse, vs, block_size, rows, status)
               : launch_programmatic(merge_kernel<64, true, __nv_bfloat16>, grid, dim3(kRowsPerCta * 32), 0,
                                     st, o_parts, lse_parts, 0, 1, total, heads, oo, lse, vs, block_size, rows, status);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace star
