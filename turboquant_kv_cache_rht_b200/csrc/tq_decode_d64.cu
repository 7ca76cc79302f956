// Decode-attention kernels of the Lloyd-Max codec for head_dim 64 (one
// translation unit per head_dim and codec so the build compiles them in parallel).
#include "tq_decode_impl.cuh"

namespace tq {

template <>
cudaError_t launch_decode_dim<64, false>(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                                  int q_heads, float scale_log2, int max_ctx,
                                  const DecodePlan& plan, float* ws, cudaStream_t stream) {
  return dispatch_decode_dim<64, false>(tb, cv, q, dtype, q_heads, scale_log2, max_ctx, plan, ws, stream);
}

template <>
cudaError_t decode_occupancy_dim<64, false>(const Tables& tb, int group, int* ctas_per_sm) {
  return dispatch_occupancy_dim<64, false>(tb, group, ctas_per_sm);
}

}  // namespace tq
