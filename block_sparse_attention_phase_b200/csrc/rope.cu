// Rotary position embedding (RoPE) for the projected Q and K of a layer, and the
// Q of the anchor-position variant of Phase 1 (rebuttal to x5MA, "Anchor Block
// Content and Position": the anchor's content is b_0, and the position IDs its
// tokens get during the local attention barely matter).
//
// Convention (rotate-half pairs): for frequency f < d/2, the pair
// (x[f], x[f + d/2]) at position p is rotated by the angle p * inv_freq[f]:
//   y[f]       = x[f] cos - x[f + d/2] sin
//   y[f + d/2] = x[f + d/2] cos + x[f] sin
// The angle is formed and reduced to [-pi, pi] in double precision, then sin and
// cos are taken in float, so positions in the millions keep full accuracy.
//
// Anchor positions. With RoPE a score depends only on the difference of the two
// positions. If the anchor tokens of block i (i >= 1) are placed right before the
// block, at positions (i-1)B + j, the score of query t (position t) with anchor
// key j (stored rotated at its own position j) equals the score of the query
// rotated at position t - (i-1)B with that stored key. So the variant needs no
// copy of the anchor: q_anchor holds every query rotated at t - (i-1)B (block 0:
// at t), and Phase 1 scores the anchor tiles with q_anchor, its own block's with q.
//
// One CTA per token: its threads first build the token's cos/sin table in shared
// memory (d/2 entries, twice for the anchor positions), then rotate every head
// of q and k with 16-byte loads and stores.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int kRopeThreads = 256;

__device__ __forceinline__ void angle_sincos(int64_t pos, float inv_freq, float* s, float* c) {
  const double a = static_cast<double>(pos) * static_cast<double>(inv_freq);
  const double two_pi = 6.283185307179586476925286766559;
  const double r = a - two_pi * rint(a / two_pi);
  sincosf(static_cast<float>(r), s, c);
}

// Rotates 8 frequencies (part * 8 ..) of one row: into dst with (cs0, sn0) and,
// if dst1 is set, also into dst1 with (cs1, sn1). Both read the input first, so
// dst may alias src.
template <int D>
__device__ __forceinline__ void rotate_row(const __nv_bfloat16* src, __nv_bfloat16* dst,
                                           const float* cs0, const float* sn0,
                                           __nv_bfloat16* dst1, const float* cs1,
                                           const float* sn1, int part) {
  const int f0 = part * 8;
  const uint4 lo = *reinterpret_cast<const uint4*>(src + f0);
  const uint4 hi = *reinterpret_cast<const uint4*>(src + D / 2 + f0);
  const __nv_bfloat16* xl = reinterpret_cast<const __nv_bfloat16*>(&lo);
  const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(&hi);
  uint4 olo, ohi, alo, ahi;
  __nv_bfloat16* yl = reinterpret_cast<__nv_bfloat16*>(&olo);
  __nv_bfloat16* yh = reinterpret_cast<__nv_bfloat16*>(&ohi);
  __nv_bfloat16* zl = reinterpret_cast<__nv_bfloat16*>(&alo);
  __nv_bfloat16* zh = reinterpret_cast<__nv_bfloat16*>(&ahi);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float a = __bfloat162float(xl[e]);
    const float b = __bfloat162float(xh[e]);
    yl[e] = __float2bfloat16_rn(a * cs0[f0 + e] - b * sn0[f0 + e]);
    yh[e] = __float2bfloat16_rn(b * cs0[f0 + e] + a * sn0[f0 + e]);
    if (dst1) {
      zl[e] = __float2bfloat16_rn(a * cs1[f0 + e] - b * sn1[f0 + e]);
      zh[e] = __float2bfloat16_rn(b * cs1[f0 + e] + a * sn1[f0 + e]);
    }
  }
  *reinterpret_cast<uint4*>(dst + f0) = olo;
  *reinterpret_cast<uint4*>(dst + D / 2 + f0) = ohi;
  if (dst1) {
    *reinterpret_cast<uint4*>(dst1 + f0) = alo;
    *reinterpret_cast<uint4*>(dst1 + D / 2 + f0) = ahi;
  }
}

struct RopeFreqs {
  float inv_freq[64];  // d/2 <= 64
};

template <int D>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(
    const __nv_bfloat16* q_in, const __nv_bfloat16* k_in, __nv_bfloat16* q_out,
    __nv_bfloat16* k_out, __nv_bfloat16* q_anchor, int64_t L, int32_t hq,
    int32_t hkv, int64_t pos0, int64_t B, const __grid_constant__ RopeFreqs fr) {
  __shared__ float cs[2][D / 2], sn[2][D / 2];
  const int64_t token = blockIdx.x;  // (batch, t) flattened
  const int64_t t = token % L;
  const int64_t blk = t / B;
  for (int f = threadIdx.x; f < D / 2; f += kRopeThreads) {
    angle_sincos(pos0 + t, fr.inv_freq[f], &sn[0][f], &cs[0][f]);
    if (q_anchor) angle_sincos(pos0 + t - (blk > 0 ? (blk - 1) * B : 0), fr.inv_freq[f], &sn[1][f], &cs[1][f]);
  }
  __syncthreads();
  constexpr int kParts = D / 16;
  const int heads = hq + hkv;
  for (int u = threadIdx.x; u < heads * kParts; u += kRopeThreads) {
    const int h = u / kParts, part = u % kParts;
    if (h < hq) {
      const int64_t off = (token * hq + h) * D;
      rotate_row<D>(q_in + off, q_out + off, cs[0], sn[0], q_anchor ? q_anchor + off : nullptr,
                    cs[1], sn[1], part);
    } else {
      const int64_t off = (token * hkv + (h - hq)) * D;
      rotate_row<D>(k_in + off, k_out + off, cs[0], sn[0], nullptr, cs[1], sn[1], part);
    }
  }
}

}  // namespace

cudaError_t launch_rope(const Shape& s, const float* inv_freq, int64_t pos0, const void* q_in,
                        const void* k_in, void* q_out, void* k_out, void* q_anchor,
                        cudaStream_t st) {
  RopeFreqs fr{};
  for (int f = 0; f < s.d / 2; ++f) fr.inv_freq[f] = inv_freq[f];
  const int64_t tokens = static_cast<int64_t>(s.b) * s.L;
  if (tokens == 0) return cudaSuccess;
  if (tokens > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto* qi = static_cast<const __nv_bfloat16*>(q_in);
  auto* ki = static_cast<const __nv_bfloat16*>(k_in);
  auto* qo = static_cast<__nv_bfloat16*>(q_out);
  auto* ko = static_cast<__nv_bfloat16*>(k_out);
  auto* qa = static_cast<__nv_bfloat16*>(q_anchor);
  const dim3 grid(static_cast<unsigned>(tokens));
  if (s.d == 128)
    rope_kernel<128><<<grid, kRopeThreads, 0, st>>>(qi, ki, qo, ko, qa, s.L, s.hq, s.hkv, pos0, s.B, fr);
  else
    rope_kernel<64><<<grid, kRopeThreads, 0, st>>>(qi, ki, qo, ko, qa, s.L, s.hq, s.hkv, pos0, s.B, fr);
  count_launch();
  return cudaGetLastError();
}

}  // namespace star
