// Device status word (one per device) and the bounded-wait self-test.
//
// Kernels OR flags (kTimeoutFlag, kBoundsFlag) into the
// word instead of trapping; star_attn_get_device_status() reads and clears it.
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "star_internal.h"

namespace star {
namespace {

__device__ uint32_t g_status_word;

constexpr int kMaxDevices = 64;
std::atomic<uint32_t*> g_status_addr[kMaxDevices];

// One warp waits on a barrier that no thread arrives at; the wait runs out
// after wait_ns, records the timeout and the block returns normally.
__global__ void selftest_wait_kernel(uint64_t wait_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_ns();
    bool done = false;
    while (!done) {
      if (mbar_try_wait(&bar, 0)) break;
      if (global_ns() - t0 > wait_ns) done = true;
    }
    if (done) report(status, kTimeoutFlag);
  }
  __syncthreads();
}

// y[i] = the FMA-pipe 2^x the attention softmax uses for part of its scores.
__global__ void selftest_exp2_kernel(const float* x, float* y, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], x[i])).x;
  }
}

// Reads every 16-byte word of src once (streaming loads that bypass L1) and
// writes one XOR per CTA to sink, so that no load can be optimised away. A
// measure of how fast this GPU streams bytes out of HBM when nothing is written
// back: the ceiling for a kernel that only reads, such as the decode step.
__global__ void __launch_bounds__(512) selftest_read_kernel(const uint4* src, int64_t n16,
                                                            uint32_t* sink) {
  constexpr int kUnroll = 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (kUnroll - 1) * stride < n16; i += kUnroll * stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w)
                   : "l"(src + i + u * stride));
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = src[i];
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  for (int o = 16; o >= 1; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t warp_acc[16];
  if ((threadIdx.x & 31) == 0) warp_acc[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t x = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) x ^= warp_acc[w];
    sink[blockIdx.x] = x;
  }
}

}  // namespace

cudaError_t launch_selftest_read(const void* src, int64_t bytes, uint32_t* sink, int32_t ctas,
                                 cudaStream_t st) {
  if (bytes <= 0 || ctas <= 0) return cudaSuccess;
  selftest_read_kernel<<<static_cast<unsigned>(ctas), 512, 0, st>>>(
      static_cast<const uint4*>(src), bytes / 16, sink);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_selftest_exp2(const float* x, float* y, int64_t n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  const unsigned blocks = static_cast<unsigned>((pairs + 255) / 256);
  selftest_exp2_kernel<<<blocks, 256, 0, st>>>(x, y, n);
  count_launch();
  return cudaGetLastError();
}

uint32_t* device_status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  uint32_t* p = g_status_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return nullptr;
  p = static_cast<uint32_t*>(addr);
  g_status_addr[dev].store(p, std::memory_order_release);
  return p;
}

cudaError_t launch_selftest_wait(uint64_t wait_ns, cudaStream_t st) {
  uint32_t* status = device_status_word();
  if (!status) return cudaErrorInvalidDevice;
  selftest_wait_kernel<<<1, 32, 0, st>>>(wait_ns, status);
  count_launch();
  return cudaGetLastError();
}

}  // namespace star
