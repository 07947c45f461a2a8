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

}  // namespace

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
