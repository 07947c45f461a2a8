// Phase-2 decode step, split-KV partials (Star Attention, hotaipapers.com page,
// Phase 2 paragraph: the new token is sent to every block, each block attends
// with its own keys and returns one vector and one scalar; the query host
// appends the token's KV to its cache).
//
// One CTA = (split, batch, kv-head). A split is a chunk of one context block, or
// the query-local cache plus the new token. The CTA streams its chunk's K and V
// rows for that kv-head once (TMA tiles of 64 tokens into a shared-memory ring)
// and serves all G = Hq/Hkv q-heads of the group from each row, so every KV byte
// is read from HBM exactly once per step. The work is HBM-bound: per key the
// CTA does 2*G*d multiply-adds against 4*d bytes.
//
// Consumer lanes own one 16-byte slice (8 elements) of a token row: a row is
// LPT = d/8 lanes, a warp covers 32/LPT rows per step. The G partial dot
// products of a lane are folded into full dot products with a transpose-reduce
// (each xor-shuffle level also halves the number of heads a lane carries), so a
// lane ends with the logit of one (token, head) pair. A running max / sum per
// head gives each warp a partial softmax state; warps are combined through
// shared memory at the end, and the CTA writes (o_s, lse_s) in fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

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
};

constexpr int kTile = 64;

template <int D, int G>
struct Lanes {
  static constexpr int LPT = D / 8;     // lanes per token row
  static constexpr int TPW = 32 / LPT;  // token rows per warp step
  // Head a lane carries after the transpose-reduce.
  __device__ static int head_of(int lane) {
    int h = 0, nh = G;
#pragma unroll
    for (int o = LPT / 2; o >= 1; o >>= 1) {
      if (nh > 1) {
        nh >>= 1;
        if (lane & o) h += nh;
      }
    }
    return h;
  }
  // A lane of token group g that carries head h.
  __device__ static int src_of(int h, int g) {
    int src = g * LPT, nh = G;
#pragma unroll
    for (int o = LPT / 2; o >= 1; o >>= 1) {
      if (nh > 1) {
        nh >>= 1;
        if (h >= nh) {
          src |= o;
          h -= nh;
        }
      }
    }
    return src;
  }
};

template <int D, int G>
struct WarpState {
  float q[G][8];
  float acc[G][8];
  float m = -INFINITY;  // running max (log2 units) of the head this lane carries
  float l = 0.f;            // running sum over this lane's token group
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& r, float (&f)[8]) {
  f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x); f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
  f[4] = bf16_lo(r.z); f[5] = bf16_hi(r.z); f[6] = bf16_lo(r.w); f[7] = bf16_hi(r.w);
}

// Fold G partial dots across the LPT lanes of a token row into one full dot
// for the head `head_of(lane)`.
template <int D, int G>
__device__ __forceinline__ float transpose_reduce(float (&v)[G], int lane) {
  constexpr int LPT = D / 8;
  int nh = G;
#pragma unroll
  for (int o = LPT / 2; o >= 1; o >>= 1) {
    if (nh > 1) {
      const int half = nh >> 1;
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < G / 2; ++j) {
        if (j < half) {
          const float send = upper ? v[j] : v[j + half];
          const float keep = upper ? v[j + half] : v[j];
          v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      nh = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

// Consume U warp-steps of token rows. krow[u] / vrow[u] point at this lane's
// 16-byte slice of step u's K and V rows (shared or global memory); valid[u]
// says whether that row is a key of this split. Rows are loaded lazily to keep
// register pressure low.
template <int D, int G, int U>
__device__ __forceinline__ void consume(WarpState<D, G>& st, const uint8_t* const (&krow)[U],
                                        const uint8_t* const (&vrow)[U], const bool (&valid)[U],
                                        int lane) {
  using LN = Lanes<D, G>;
  const int g = lane / LN::LPT;
  float s[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    float kf[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(krow[u]), kf);
    float part[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(st.q[h][e], kf[e], a);
      part[h] = a;
    }
    const float dot = transpose_reduce<D, G>(part, lane);
    s[u] = valid[u] ? dot : -INFINITY;
  }
  float mt = s[0];
#pragma unroll
  for (int u = 1; u < U; ++u) mt = fmaxf(mt, s[u]);
#pragma unroll
  for (int o = LN::LPT; o < 32; o <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
  const float m_new = fmaxf(st.m, mt);
  const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
  const float alpha = exp2f(st.m - m_use);
  float p[U];
  float psum = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    p[u] = exp2f(s[u] - m_use);
    psum += p[u];
  }
  st.l = st.l * alpha + psum;
  st.m = m_new;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float ah = __shfl_sync(0xffffffffu, alpha, LN::src_of(h, 0));
#pragma unroll
    for (int e = 0; e < 8; ++e) st.acc[h][e] *= ah;
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    // Rows past the split end may hold stale cache bytes (even NaN patterns);
    // use zeros there so that p = 0 never meets a NaN.
    uint4 raw = *reinterpret_cast<const uint4*>(vrow[u]);
    if (!valid[u]) raw = make_uint4(0u, 0u, 0u, 0u);
    float vf[8];
    bf16x8_to_f32(raw, vf);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float ph = __shfl_sync(0xffffffffu, p[u], LN::src_of(h, g));
#pragma unroll
      for (int e = 0; e < 8; ++e) st.acc[h][e] = fmaf(ph, vf[e], st.acc[h][e]);
    }
  }
}

template <int D, int G, int W, int NST>
__global__ void __launch_bounds__((W + 1) * 32, (G <= 4 ? 2 : 1)) decode_partials_kernel(
    const __grid_constant__ CUtensorMap mk_ctx, const __grid_constant__ CUtensorMap mv_ctx,
    const __grid_constant__ CUtensorMap mk_cache, const __grid_constant__ CUtensorMap mv_cache,
    const DecodeArgs a) {
  using LN = Lanes<D, G>;
  constexpr int LPT = LN::LPT;
  constexpr int TPW = LN::TPW;
  constexpr int TOK_PER_WARP = kTile / W;
  constexpr int U = TOK_PER_WARP / TPW;
  static_assert(U >= 1 && TOK_PER_WARP % TPW == 0, "tile must split evenly over warps");
  constexpr uint32_t kTileBytes = kTile * D * 2;

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* kbuf = smem;
  uint8_t* vbuf = smem + NST * kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * NST * kTileBytes);
  uint64_t* empty = full + NST;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bb = blockIdx.y / a.hkv;
  const int kvh = blockIdx.y % a.hkv;
  const bool is_cache = split == a.n_ctx;

  int64_t k0, k1;
  if (!is_cache) {
    const int64_t blk = split / a.spb;
    const int64_t sub = split % a.spb;
    const int64_t bstart = blk * a.B;
    const int64_t bend = min(a.L, bstart + a.B);
    k0 = min(bend, bstart + sub * a.chunk);
    k1 = min(bend, k0 + a.chunk);
  } else {
    k0 = 0;
    k1 = a.cache_len;
  }
  const int ntiles = static_cast<int>((k1 - k0 + kTile - 1) / kTile);

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], W);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == W) {
    // ---------------- producer warp: TMA loads, and the cache append ----------------
    if (lane == 0 && ntiles > 0) {
      const CUtensorMap* mk = is_cache ? &mk_cache : &mk_ctx;
      const CUtensorMap* mv = is_cache ? &mv_cache : &mv_ctx;
      for (int i = 0; i < ntiles; ++i) {
        const int stg = i % NST;
        const uint32_t ph = (i / NST) & 1;
        if (i >= NST && !mbar_wait(&empty[stg], ph ^ 1, a.status)) break;
        mbar_arrive_expect_tx(&full[stg], 2 * kTileBytes);
        const int32_t t0 = static_cast<int32_t>(k0 + static_cast<int64_t>(i) * kTile);
        tma_load_4d(kbuf + stg * kTileBytes, mk, &full[stg], 0, kvh, t0, bb);
        tma_load_4d(vbuf + stg * kTileBytes, mv, &full[stg], 0, kvh, t0, bb);
      }
    }
    if (is_cache && lane < LPT) {
      // Append the new token's K/V at cache row cache_len. No CTA of this launch
      // reads that row as a cache key (the token is taken from k_new / v_new).
      const int64_t src = (static_cast<int64_t>(bb) * a.hkv + kvh) * D + lane * 8;
      const int64_t dst = ((static_cast<int64_t>(bb) * a.cap + a.cache_len) * a.hkv + kvh) * D + lane * 8;
      *reinterpret_cast<uint4*>(a.k_cache + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
      *reinterpret_cast<uint4*>(a.v_cache + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
    }
  } else {
    // ---------------- consumer warps ----------------
    const int g = lane / LPT;
    const int c = lane % LPT;
    WarpState<D, G> st;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const int hq = kvh * G + h;
      const uint4 r = *reinterpret_cast<const uint4*>(
          a.q + (static_cast<int64_t>(bb) * a.hq + hq) * D + c * 8);
      float f[8];
      bf16x8_to_f32(r, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        st.q[h][e] = f[e] * a.scale_log2;
        st.acc[h][e] = 0.f;
      }
    }
    for (int i = 0; i < ntiles; ++i) {
      const int stg = i % NST;
      const uint32_t ph = (i / NST) & 1;
      const bool ok = mbar_wait(&full[stg], ph, a.status);
      if (ok) {
        const uint8_t* kt = kbuf + stg * kTileBytes;
        const uint8_t* vt = vbuf + stg * kTileBytes;
        const uint8_t* krow[U];
        const uint8_t* vrow[U];
        bool valid[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int tok = warp * TOK_PER_WARP + u * TPW + g;
          valid[u] = k0 + static_cast<int64_t>(i) * kTile + tok < k1;
          krow[u] = kt + tok * (D * 2) + c * 16;
          vrow[u] = vt + tok * (D * 2) + c * 16;
        }
        consume<D, G, U>(st, krow, vrow, valid, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stg]);
    }
    if (is_cache && warp == 0) {
      // The new token: one more row, read straight from the input.
      const int64_t off = (static_cast<int64_t>(bb) * a.hkv + kvh) * D + c * 8;
      const uint8_t* krow[1] = {reinterpret_cast<const uint8_t*>(a.k_new + off)};
      const uint8_t* vrow[1] = {reinterpret_cast<const uint8_t*>(a.v_new + off)};
      const bool valid[1] = {g == 0};
      consume<D, G, 1>(st, krow, vrow, valid, lane);
    }

    // Fold the token groups of the warp together.
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
      st.l += __shfl_xor_sync(0xffffffffu, st.l, o);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) st.acc[h][e] += __shfl_xor_sync(0xffffffffu, st.acc[h][e], o);
    }
    // Every stage has been consumed and no copy is in flight: reuse the ring.
    asm volatile("bar.sync 1, %0;" ::"r"(W * 32) : "memory");
    float* cm = reinterpret_cast<float*>(smem);  // [W][G]
    float* cl = cm + W * G;                      // [W][G]
    float* cacc = cl + W * G;                    // [W][G][D]
    if (g == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) cacc[(warp * G + h) * D + c * 8 + e] = st.acc[h][e];
      const int h = LN::head_of(lane);
      if (LN::src_of(h, 0) == lane) {
        cm[warp * G + h] = st.m;
        cl[warp * G + h] = st.l;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(W * 32) : "memory");
    for (int idx = threadIdx.x; idx < G * D; idx += W * 32) {
      const int h = idx / D;
      const int e = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) M = fmaxf(M, cm[w * G + h]);
      float lsum = 0.f, o = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const float sc = exp2f(cm[w * G + h] - M);
          lsum += cl[w * G + h] * sc;
          o += cacc[(w * G + h) * D + e] * sc;
        }
      }
      const int hq = kvh * G + h;
      const int64_t row = static_cast<int64_t>(split) * a.b + bb;
      a.o_parts[(row * a.hq + hq) * D + e] = lsum > 0.f ? o / lsum : 0.f;
      if (e == 0) {
        a.lse_parts[row * a.hq + hq] =
            lsum > 0.f ? (M + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
}

template <int D, int G>
cudaError_t launch_decode_t(const Shape& s, const SplitPlan& p, const DecodeArgs& a,
                            const void* kc, const void* vc, cudaStream_t st) {
  constexpr int W = 8;
  constexpr int NST = 3;
  alignas(64) CUtensorMap m[4];
  const bool ok = encode_tma_bf16_4d(&m[0], kc, D, s.hkv, s.L, s.L, s.b, D, 1, kTile, false) &&
                  encode_tma_bf16_4d(&m[1], vc, D, s.hkv, s.L, s.L, s.b, D, 1, kTile, false) &&
                  encode_tma_bf16_4d(&m[2], a.k_cache, D, s.hkv, a.cap, a.cap, s.b, D, 1, kTile, false) &&
                  encode_tma_bf16_4d(&m[3], a.v_cache, D, s.hkv, a.cap, a.cap, s.b, D, 1, kTile, false);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = 2 * NST * kTile * D * 2 + 2 * NST * sizeof(uint64_t);
  auto kern = decode_partials_kernel<D, G, W, NST>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(p.n_splits, s.b * s.hkv);
  kern<<<grid, (W + 1) * 32, smem, st>>>(m[0], m[1], m[2], m[3], a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_partials(const Shape& s, const SplitPlan& p, const void* q,
                                   const void* k_new, const void* v_new, const void* kc,
                                   const void* vc, void* k_cache, void* v_cache, int64_t cache_len,
                                   int64_t cap, float* o_parts, float* lse_parts,
                                   cudaStream_t st) {
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  a.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  a.cache_len = cache_len;
  a.cap = cap;
  a.L = s.L;
  a.B = s.B;
  a.chunk = p.chunk;
  a.spb = p.spb;
  a.n_ctx = p.n_ctx;
  a.b = s.b;
  a.hq = s.hq;
  a.hkv = s.hkv;
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  a.status = device_status_word();
  const int G = s.group();
#define STAR_DECODE_CASE(DD, GG) \
  if (s.d == DD && G == GG) return launch_decode_t<DD, GG>(s, p, a, kc, vc, st);
  STAR_DECODE_CASE(128, 1) STAR_DECODE_CASE(128, 2) STAR_DECODE_CASE(128, 4)
  STAR_DECODE_CASE(128, 8) STAR_DECODE_CASE(64, 1) STAR_DECODE_CASE(64, 2)
  STAR_DECODE_CASE(64, 4) STAR_DECODE_CASE(64, 8)
#undef STAR_DECODE_CASE
  return cudaErrorNotSupported;
}

}  // namespace star
