// Decode step that allocates nothing: the split-KV partials live in a
// fixed-size scratch array compiled into the library instead of a
// caller-provided workspace.
//
// Who needs this: callers that cannot obtain device memory at the point where
// they decode. Examples are serving runtimes whose pooled allocator already owns
// every byte of the GPU, so an extra cudaMalloc would fail or fragment the pool;
// code that must not pay the implicit device-wide synchronisation that
// cudaMalloc/cudaFree can cause; and plain C callers that have no allocator
// handle to hand a workspace in. They still pass every input and output buffer.
//
// Rules of the scratch array:
//   * It is a file-scope __device__ array of kNoAllocScratchBytes (4 MiB). Every
//     GPU that loads this library holds one copy until the process exits.
//   * Its host-side name is only a stand-in, not a device address. Its device
//     address is looked up with cudaGetSymbolAddress once per device, with that
//     device current, on the first call of the entry point on that device. Make
//     that first call before any stream capture.
//   * All calls share it and it keeps the previous call's contents. Nothing in it
//     needs to start at zero: every partial the merge reads is written by the
//     partial kernel of the same call first.
//   * Calls whose kernels may overlap on one GPU (for example, calls on two
//     streams) race on that GPU's array; keep them ordered, e.g. on one stream.
//     Each GPU has its own copy, so calls on different GPUs do not interfere.
//   * Shapes whose partials exceed the array are rejected with
//     STAR_ERR_WORKSPACE before anything is launched.
#include <cuda_runtime.h>

#include <atomic>

#include "../../include/star_attn.h"
#include "star_internal.h"

namespace star {

// The shape checks every entry point applies (STAR_OK, STAR_ERR_INVALID_ARG or
// STAR_ERR_UNSUPPORTED), from the C-ABI layer.
star_status_t check_shape(const star_attn_shape_t* shape);

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{4} << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of this device's scratch array (nullptr on failure).
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
    return nullptr;
  g_scratch_addr[dev].store(addr, std::memory_order_release);
  return addr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace star

extern "C" STAR_ATTN_API star_status_t star_attn_phase2_decode_noalloc(
    const star_attn_shape_t* shape, const void* q, const void* k, const void* v,
    const void* k_ctx, const void* v_ctx, void* k_cache, void* v_cache, int64_t cache_len,
    int64_t cache_capacity, void* o, float* lse, star_stream_t stream) {
  // An invalid or unsupported shape gets the same status as from star_attn_phase2_decode().
  const star_status_t shape_status = star::check_shape(shape);
  if (shape_status != STAR_OK) return shape_status;
  const size_t need = star_attn_workspace_bytes(shape, STAR_PHASE2_DECODE, 1);
  if (need == 0) return STAR_ERR_INVALID_ARG;
  if (need > star::kNoAllocScratchBytes) return STAR_ERR_WORKSPACE;
  if (cache_len < 0 || cache_capacity < 1) return STAR_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, k_ctx, v_ctx, k_cache, v_cache, o};
  for (const void* p : ptrs)
    if (!p || !star::aligned16(p)) return STAR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return STAR_ERR_INVALID_ARG;  // one float each
  if (cache_len + 1 > cache_capacity) return STAR_ERR_CACHE_FULL;
  void* scratch = star::scratch_address();
  if (!scratch) return STAR_ERR_CUDA;
  // The existing entry point does the rest, with the static array as its workspace.
  return star_attn_phase2_decode(shape, q, k, v, k_ctx, v_ctx, k_cache, v_cache, cache_len,
                                 cache_capacity, o, lse, scratch, star::kNoAllocScratchBytes,
                                 stream);
}
