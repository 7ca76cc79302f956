// Decode attention for callers that cannot allocate device memory.
//
// tq_decode_attention needs a caller-provided workspace for its per-split
// partial results.  Some callers have no way to provide one: a runtime whose
// device memory is fixed up front and handed out by its own pool, a plugin
// that is only given input and output pointers by its host, or code that must
// not call cudaMalloc because an allocation can synchronize the device or fail
// at an unpredictable point.  For them this file keeps the scratch in a static
// device array that is part of the library image: it is reserved on every GPU
// that loads the library and lives until the process exits.  Nothing here
// calls cudaMalloc, cudaFree or any other allocating routine.
#include "../../include/tq.h"
#include "tq_internal.cuh"

#include <cstdio>

namespace {

// 8 MiB.  The split planner keeps the number of partials near
// (query heads per KV head) x 592 + (batch rows x query heads), so this covers
// for example 32 batch rows x 32 query heads at head_dim 128 (1.6 MB) or
// 16 query heads over a 512k-token context at head_dim 256 (2.4 MB).
constexpr size_t kScratchBytes = 8u << 20;
static __device__ __align__(256) float g_decode_scratch[kScratchBytes / sizeof(float)];

// Device address of g_decode_scratch in the current context.  On the host the
// array's name only stands in for the symbol, so the address is looked up on
// every call: the lookup allocates nothing and costs little once the module is
// loaded, and it stays right after the context is reset (the module, and with
// it the array, is loaded afresh into the new context).
tq_status scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || !p) {
    char msg[256];
    std::snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static decode scratch failed: %s",
                  cudaGetErrorString(e));
    return (tq_status)tq::record_error(TQ_ERR_CUDA, msg);
  }
  *out = p;
  return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_decode_attention_noalloc(const tq_codebook* cb, const tq_cache* cache,
                                                 const void* q, tq_dtype dtype, int q_heads,
                                                 float softmax_scale, int max_ctx, float* out,
                                                 void* stream) {
  if (!cb || !cache)
    return (tq_status)tq::record_error(TQ_ERR_INVALID, "codebook or cache is NULL");
  const size_t need =
      tq_decode_workspace_bytes(cb, cache->batch, q_heads, cache->kv_heads, max_ctx);
  if (need > kScratchBytes) {
    char msg[256];
    std::snprintf(msg, sizeof msg,
                  "this decode needs %zu bytes of scratch but the built-in scratch holds %zu; "
                  "use tq_decode_attention with a workspace of that size",
                  need, kScratchBytes);
    return (tq_status)tq::record_error(TQ_ERR_CAPACITY, msg);
  }
  void* scratch = nullptr;
  const tq_status st = scratch_address(&scratch);
  if (st != TQ_OK) return st;
  return tq_decode_attention(cb, cache, q, dtype, q_heads, softmax_scale, max_ctx, out, scratch,
                             kScratchBytes, stream);
}
