// Phase 1 and Phase-2 query launchers (bring-up: routed to the simple kernels).
#include "star_internal.h"

namespace star {

cudaError_t launch_phase1_sm100(const Shape& s, const void* q, const void* k, const void* v,
                                void* o, float* lse, cudaStream_t st) {
  return launch_simple_phase1(s, q, k, v, o, lse, st);
}

cudaError_t launch_query_path(const Shape& s, const SplitPlan& p, const void* q, int64_t lq,
                              const void* kc, const void* vc, const void* k_cache,
                              const void* v_cache, int64_t cap, float* o_parts, float* lse_parts,
                              void* o, float* lse, cudaStream_t st) {
  (void)p; (void)o_parts; (void)lse_parts;
  return launch_simple_phase2(s, q, lq, kc, vc, k_cache, v_cache, cap, 0, 1, o, lse, st);
}

}  // namespace star
