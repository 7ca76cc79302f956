// Internal interface between the C ABI (tq_api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace tq {

// Programmatic dependent launch.  Every kernel is launched with programmatic
// stream serialization, waits for the previous kernel in the stream (and its
// memory) before reading any buffer, and lets the next kernel start launching
// once its own results are written.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

constexpr unsigned kFlagCapacity = 1u;  // mirrors TQ_FLAG_CAPACITY
constexpr unsigned kFlagMaxCtx = 2u;    // mirrors TQ_FLAG_MAXCTX

// Codebooks and rotation signs, passed to every kernel by value (they live in
// the kernel parameter bank; no device allocation is needed).
struct Tables {
  float k_cent[16];
  float k_bnd[16];   // first 2^k_bits - 1 entries used
  float v_cent[16];
  float v_bnd[16];
  uint32_t s1[8];    // bit i set: channel i of D1 is -1
  uint32_t s2[8];    // same for D2 (QJL rotation)
  int d, k_bits, v_bits, qjl;
};

struct CacheView {
  uint8_t *k_codes, *v_codes, *k_signs;
  uint16_t *k_norm, *v_norm, *k_rnorm;
  int32_t *seq_lens, *status, *append_sync;
  int batch, kv_heads, capacity;
};

// Input element types of k, v and q.
enum DType : int { kF32 = 0, kBF16 = 1, kF16 = 2 };

cudaError_t launch_quantize_append(const Tables& tb, const CacheView& cv, const void* k,
                                   const void* v, int dtype, int n_new, cudaStream_t stream);

// Split of the context over CTAs for one decode call.
struct DecodePlan {
  int splits;  // CTAs per (batch row, KV head)
  int chunk;   // tokens per split (multiple of the token tile)
};
DecodePlan plan_decode(int batch, int kv_heads, int max_ctx, int head_dim);
size_t decode_workspace_bytes(const DecodePlan& plan, int batch, int q_heads, int head_dim);

// Returns cudaErrorNotSupported when no kernel is built for this shape.
cudaError_t launch_decode(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                          int q_heads, float scale, const DecodePlan& plan, float* out,
                          float* workspace, cudaStream_t stream);
bool decode_supported(int head_dim, int group, int k_bits, int v_bits, int qjl);

// Stores `message` as this thread's last error and returns `status`.
int record_error(int status, const char* message);

}  // namespace tq
