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

__device__ uint32_t g_status_word[kStatusWords];

constexpr int kMaxDevices = 64;
std::atomic<uint32_t*> g_status_addr[kMaxDevices];

// Debug-check self-test: one thread checks index n against limit n (one past the
// end) with the same check the kernels' stores use, so a debug build records it
// and skips the store (the store itself would be in bounds anyway: the buffer has
// n + 1 elements and the kernel writes element n only when the check lets it).
__global__ void selftest_bounds_kernel(uint32_t* out, int64_t n, uint32_t* status) {
  if (threadIdx.x == 0 && blockIdx.x == 0 && STAR_IN_BOUNDS(status, n, n)) out[n] = 1u;
}

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

// Reads every byte of src once with 1-D bulk asynchronous copies (the copy engine
// the attention kernels stream K/V with) into a ring of shared-memory buffers, and
// writes one XOR per CTA of the first word of every chunk it received to sink. A
// measure of how fast this GPU streams bytes out of HBM when nothing is written
// back: the ceiling for a kernel that only reads, such as the decode step.
constexpr int kReadStages = 4;
constexpr uint32_t kReadChunk = 32768;

__global__ void __launch_bounds__(32) selftest_read_kernel(const uint8_t* src, int64_t bytes,
                                                           uint32_t* sink, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                            ~uintptr_t(127));
  __shared__ alignas(8) uint64_t full[kReadStages];
  if (threadIdx.x != 0) return;
  for (int s = 0; s < kReadStages; ++s) mbar_init(&full[s], 1);
  fence_barrier_init();
  const int64_t n_chunks = (bytes + kReadChunk - 1) / kReadChunk;
  auto issue = [&](int64_t c, int s) {
    const int64_t off = c * kReadChunk;
    const uint32_t n = static_cast<uint32_t>(bytes - off < kReadChunk ? bytes - off : kReadChunk);
    mbar_arrive_expect_tx(&full[s], n);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(buf + s * kReadChunk)),
        "l"(src + off), "r"(n), "r"(smem_u32(&full[s]))
        : "memory");
  };
  // Chunk i of this CTA is blockIdx.x + i * gridDim.x, in stage i % kReadStages.
  const int64_t mine = blockIdx.x < n_chunks ? (n_chunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  for (int64_t i = 0; i < kReadStages && i < mine; ++i)
    issue(blockIdx.x + i * gridDim.x, static_cast<int>(i));
  uint32_t acc = 0;
  int64_t i = 0;
  for (; i < mine; ++i) {
    const int s = static_cast<int>(i % kReadStages);
    if (!mbar_wait(&full[s], static_cast<uint32_t>((i / kReadStages) & 1), status)) break;
    acc ^= *reinterpret_cast<const uint32_t*>(buf + s * kReadChunk);
    if (i + kReadStages < mine) {
      fence_proxy_async_smem();  // the read above precedes the copy that overwrites the buffer
      issue(blockIdx.x + (i + kReadStages) * gridDim.x, s);
    }
  }
  // After a wait gave up, the copies still in flight land before the CTA exits
  // (each wait bounded again).
  for (int64_t k = i; k < mine && k < i + kReadStages; ++k)
    mbar_wait(&full[k % kReadStages], static_cast<uint32_t>((k / kReadStages) & 1), status);
  sink[blockIdx.x] = acc;
}

}  // namespace

cudaError_t launch_selftest_read(const void* src, int64_t bytes, uint32_t* sink, int32_t ctas,
                                 cudaStream_t st) {
  if (bytes <= 0 || ctas <= 0) return cudaSuccess;
  uint32_t* status = device_status_word();
  if (!status) return cudaErrorInvalidDevice;
  const size_t smem = size_t{kReadStages} * kReadChunk + 128;
  cudaError_t e = cudaFuncSetAttribute(selftest_read_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  selftest_read_kernel<<<static_cast<unsigned>(ctas), 32, smem, st>>>(
      static_cast<const uint8_t*>(src), bytes, sink, status);
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

bool debug_build() {
#ifdef STAR_DEBUG
  return true;
#else
  return false;
#endif
}

cudaError_t launch_selftest_bounds(uint32_t* out, int64_t n, cudaStream_t st) {
  uint32_t* status = device_status_word();
  if (!status) return cudaErrorInvalidDevice;
  selftest_bounds_kernel<<<1, 32, 0, st>>>(out, n, status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint64_t wait_ns, cudaStream_t st) {
  uint32_t* status = device_status_word();
  if (!status) return cudaErrorInvalidDevice;
  selftest_wait_kernel<<<1, 32, 0, st>>>(wait_ns, status);
  count_launch();
  return cudaGetLastError();
}

}  // namespace star
