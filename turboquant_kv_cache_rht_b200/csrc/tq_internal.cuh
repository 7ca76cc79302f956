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
constexpr unsigned kFlagLayout = 4u;    // mirrors TQ_FLAG_LAYOUT

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
  int affine;        // 1: the affine group-64 codec (centroids are the integer levels)
  // Scales in [1, 2) of the decode kernel's fp16 code tables: they hold
  // fp16(k_lam * k_cent[j]) and fp16(v_lam * v_cent[j]), chosen so that these
  // roundings are nearly exact; the kernels divide the scale out in fp32
  // (1 for the affine codec, whose levels are small integers).
  float k_lam, v_lam;
};

// Channels per group of the affine codec; its per-vector metadata is one
// (scale, bias) fp16 pair, i.e. one 32-bit word, per group.
constexpr int kAffineGroup = 64;

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
// Weights [rows][k] -> codes [k/d][rows][k_bits*d/8] and fp16 norms [k/d][rows].
cudaError_t launch_weights_quantize(const Tables& tb, const void* w, int dtype, int rows, int k,
                                    uint8_t* codes, uint16_t* norms, cudaStream_t stream);
// Y [m][rows] = X [m][k] W_hat^T on the codes above; the workspace holds the
// rotated inputs (B-fragment order, with their scales) and, when the plan
// splits the blocks, the per-split partial sums.
struct MatmulPlan {
  int inputs_per_group;  // inputs per CTA column group (4, 8 or 16)
  int groups;            // column groups
  int splits;            // CTAs along the k blocks
  int blocks_per_split;
  size_t frag_words;     // rotated-input fragments in the workspace
  size_t scale_floats;   // and their scales
};
// At most target_ctas CTAs (never more than the bound the workspace is sized for).
MatmulPlan plan_lut_matmul(int rows, int k, int m, int d, long target_ctas);
constexpr long kLutMatmulMaxCtas = 148L * 4;
size_t lut_matmul_workspace_bytes(const MatmulPlan& plan, int rows, int m);
cudaError_t launch_lut_matmul(const Tables& tb, const uint8_t* codes, const uint16_t* norms, int rows,
                              int k, const void* x, int dtype, int m, float* y, float* workspace,
                              cudaStream_t stream);
// Dense cache (strides in elements) -> compressed cache, lengths[b] tokens per row.
cudaError_t launch_quantize_cache(const Tables& tb, const CacheView& cv, const void* k,
                                  const void* v, int dtype, long stride_b, long stride_h,
                                  long stride_t, const int32_t* lengths, int max_len,
                                  cudaStream_t stream);

// Work partition of one decode call.  Row b holds n_b = ceil(L_b / 64) token
// tiles per KV head, L_b being seq_lens[b] clamped to [0, min(capacity,
// max_ctx)].  The units u = b * kv_heads + h are laid end to end (unit (b, h)
// covers tiles [kv_heads * P_b + h * n_b, ... + n_b), P_b = sum of n over the
// rows before b), and CTA c of `ctas` takes tiles [c*T/ctas, (c+1)*T/ctas) of
// the T in total.  The kernels compute this on the device from the lengths
// they read there.  Each (CTA, unit) segment leaves one partial result in
// workspace slot c + u; segments move monotonically in both c and u, so the
// slots are distinct and `slots` = ctas + units - 1 bounds them.
struct DecodePlan {
  int ctas;
  int slots;
};
// At most `target_ctas` CTAs and no more than the tiles max_ctx allows.
DecodePlan plan_decode(int batch, int kv_heads, int max_ctx, long target_ctas);
// The most CTAs a launch uses (4 per SM of a 148-SM B200); the workspace for
// it bounds the workspace of every launch.
constexpr long kMaxTargetCtas = 148L * 4;
size_t decode_workspace_bytes(const DecodePlan& plan, int q_heads, int kv_heads, int head_dim);

// Sizes the grid for one wave of the decode kernel at its real occupancy on
// this device and launches decode + combine.  Returns cudaErrorNotSupported when no kernel is
// built for this shape.
cudaError_t launch_decode(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                          int q_heads, float scale, int max_ctx, float* out, float* workspace,
                          cudaStream_t stream);
bool decode_supported(int head_dim, int group, int k_bits, int v_bits, int qjl);

// Stores `message` as this thread's last error and returns `status`.
int record_error(int status, const char* message);

}  // namespace tq
