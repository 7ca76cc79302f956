// Quantize-and-append kernel of the TurboQuant KV-cache codec.
//
// Per d-vector (a key or a value of one token, one KV head):
//   norm -> sign flips -> Walsh-Hadamard -> scale -> bucket -> pack, and for
//   keys with QJL: residual -> its norm -> second rotation -> sign bits.
// ("TurboQuant Performance Benefits ...", "What Is TurboQuant?": random
// Hadamard rotation then MSE codebook quantization; "mlx-turboquant" README,
// "The 1-bit QJL residual": sign(RHT2(r)) and ||r||.)  The kernels are also
// instantiated for the affine group-64 comparison codec (rotated keys, fp16
// scale and bias per group of 64 channels: encode_affine_store).
//
// Bulk layout: a group of d/32 adjacent lanes encodes one vector, each lane
// holding 32 consecutive channels, so a warp encodes 32*32/d vectors at once.
// Five of the transform's butterfly stages and five levels of the norm's
// pairwise tree run inside a lane; the rest are shuffles within the group.  A
// lane's 32 codes fill whole 32-bit words of the packed row, so packing needs
// no cross-lane traffic.  (Eight channels per lane, measured as well, runs 1.7x
// the instructions at a higher issue rate and is 30% slower.)  Small appends
// give each vector a warp (d/32 channels per lane); their lanes' codes are
// assembled into words by shuffles.
//
// Every floating-point step is a single correctly rounded fp32 operation in
// one fixed order (__fadd_rn / __fsub_rn / __fmul_rn / __fsqrt_rn /
// __fdiv_rn; the cross-lane butterfly is an FMA by +-1, which rounds exactly
// like the addition or subtraction), so codes, sign bits and fp16 norms are
// reproducible bit for bit.
#include "tq_codec.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

namespace tq {
namespace {

using namespace codec;

constexpr int kAppendWarps = 8;
// Channels per lane of the bulk layout (appends of many vectors, conversion).
constexpr int kBulkE = 32;

// The codec of one vector at its code width: Lloyd-Max (norm, codes, sketch)
// or the affine group-64 comparison codec (scale/bias pairs in `norm`).  BITS
// fixes the width at compile time (a grid of one kind: a third less register
// pressure than the kernel that holds all three widths, so a third more warps
// per SM); 0 takes it from `bits`.
template <int D, int E, bool AFF, int BITS = 0>
__device__ __forceinline__ void encode_vector(int bits, float (&u)[E], const Tables& tb, bool is_v,
                                              int g, int lane, bool valid, uint8_t* codes,
                                              uint16_t* norm, uint8_t* signs, uint16_t* rnorm,
                                              const float* s_kcent) {
  if constexpr (BITS != 0) {
    if constexpr (AFF)
      encode_affine_store<D, E, BITS>(u, tb, is_v, g, lane, valid, codes,
                                      reinterpret_cast<uint32_t*>(norm), signs, rnorm);
    else
      encode_store<D, E, BITS>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent);
  } else if constexpr (AFF) {
    uint32_t* meta = reinterpret_cast<uint32_t*>(norm);
    if (bits == 2)
      encode_affine_store<D, E, 2>(u, tb, is_v, g, lane, valid, codes, meta, signs, rnorm);
    else if (bits == 3)
      encode_affine_store<D, E, 3>(u, tb, is_v, g, lane, valid, codes, meta, signs, rnorm);
    else
      encode_affine_store<D, E, 4>(u, tb, is_v, g, lane, valid, codes, meta, signs, rnorm);
  } else {
    if (bits == 2)
      encode_store<D, E, 2>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent);
    else if (bits == 3)
      encode_store<D, E, 3>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent);
    else
      encode_store<D, E, 4>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent);
  }
}
constexpr int kAppendThreads = 32 * kAppendWarps;

// Grid: (kinds * blocks_per_kind, batch).  Blocks encode kind `first_kind`
// (0 keys, 1 values), the next blocks_per_kind blocks the other kind when
// kinds is 2, so a block's code width is uniform.  A group of D / E lanes
// encodes one vector: E = 32 packs 32 * 32 / D vectors into a warp (throughput:
// bulk appends); E = D / 32 gives each vector its own warp and keeps the
// unrolled code short (latency: a few tokens per row, as in a decode step).
// `publish`: this grid's last block of a row sets the row's new length (a
// bulk append runs keys and values as two grids, so that each grid executes
// one code width and its unrolled code stays in the instruction cache; the
// second grid publishes).
template <int D, typename T, int E, bool AFF, bool BULK, int BITS = 0>
__global__ void __launch_bounds__(kAppendThreads)
    quantize_append_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                           const T* __restrict__ kin, const T* __restrict__ vin, int n_new,
                           int blocks_per_kind, int first_kind, int publish) {
  constexpr int GL = D / E;                     // lanes per vector
  constexpr int VPB = kAppendThreads / GL;      // vectors per block
  __shared__ float s_kcent[16];

  const int tid = threadIdx.x, lane = tid & 31, g = lane & (GL - 1);
  if (tid < 16) s_kcent[tid] = tb.k_cent[tid];
  const int b = blockIdx.y;
  const int kind_block = (int)blockIdx.x / blocks_per_kind;
  const bool is_v = first_kind + kind_block == 1;
  const long r = (long)((int)blockIdx.x - kind_block * blocks_per_kind) * VPB + tid / GL;
  const long per_kind = (long)cv.kv_heads * n_new;
  const bool valid = r < per_kind;
  const int h = valid ? (int)(r / n_new) : 0, j = valid ? (int)(r % n_new) : 0;

  pdl_wait();
  // A small append (this layout) is a grid that is resident at once: let the
  // next kernel launch now, so that its set-up overlaps this one (it still waits
  // for this grid's completion before reading anything).  A bulk append keeps
  // the trigger at its end, so that waiting CTAs do not take its blocks' slots.
  if constexpr (!BULK) pdl_trigger();
  const int base = cv.seq_lens[b];
  const bool fits = base >= 0 && base <= cv.capacity - n_new;
  if (!fits && tid == 0 && blockIdx.x == 0) atomicOr(cv.status, (int)kFlagCapacity);
  __syncthreads();  // s_kcent

  if (fits && __any_sync(kFull, valid)) {
    float u[E];
    const T* src = (is_v ? vin : kin) + (((long)b * cv.kv_heads + h) * n_new + j) * D + g * E;
    if (valid) {
      load_elems<E>(src, u);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) u[e] = 0.f;
    }
    const long slot = ((long)b * cv.kv_heads + h) * cv.capacity + base + j;
    const int bits = is_v ? tb.v_bits : tb.k_bits;
    uint8_t* codes = (is_v ? cv.v_codes : cv.k_codes) + slot * (long)(bits * D / 8);
    // one fp16 norm per vector, or the affine codec's (scale, bias) per group
    constexpr int NH = AFF ? 2 * D / kAffineGroup : 1;
    uint16_t* norm = (is_v ? cv.v_norm : cv.k_norm) + slot * NH;
    uint8_t* signs = (!is_v && tb.qjl) ? cv.k_signs + slot * (long)(D / 8) : nullptr;
    uint16_t* rnorm = (!is_v && tb.qjl) ? cv.k_rnorm + slot : nullptr;
    encode_vector<D, E, AFF, BITS>(bits, u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent);
  }

  // The last block of this batch row to finish publishes the new length.  Every
  // block read seq_lens[b] before taking its ticket, so none can see the update.
  if (publish) {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const int ticket = atomicAdd(&cv.append_sync[b], 1);
      if (ticket == (int)gridDim.x - 1) {
        if (fits) cv.seq_lens[b] = base + n_new;
        cv.append_sync[b] = 0;
      }
    }
  }
  if constexpr (BULK) pdl_trigger();
}

// Conversion of a dense cache.  Grid: (kinds * blocks_per_kind, batch) as for
// the append (kinds = 1 encodes keys only: weight blocks); the vectors (h, t)
// of a row are numbered with t outermost when the input's head stride is the
// smaller one (a [batch][T][heads][d] cache) and with h outermost otherwise,
// so consecutive lanes read consecutive memory.  Without `lengths` every row
// holds max_len vectors and no length or flag is written.
template <int D, typename T, int E, bool AFF, int BITS = 0>
__global__ void __launch_bounds__(kAppendThreads)
    quantize_convert_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                            const T* __restrict__ kin, const T* __restrict__ vin, long stride_b,
                            long stride_h, long stride_t, const int32_t* __restrict__ lengths,
                            int max_len, int blocks_per_kind, int heads_inner, int first_kind) {
  constexpr int GL = D / E;
  constexpr int VPB = kAppendThreads / GL;
  __shared__ float s_kcent[16];

  const int tid = threadIdx.x, lane = tid & 31, g = lane & (GL - 1);
  if (tid < 16) s_kcent[tid] = tb.k_cent[tid];
  const int b = blockIdx.y, H = cv.kv_heads;
  const int kind_block = (int)blockIdx.x / blocks_per_kind;
  const bool is_v = first_kind + kind_block == 1;
  const long r = (long)((int)blockIdx.x - kind_block * blocks_per_kind) * VPB + tid / GL;
  const bool in_grid = r < (long)H * max_len;
  const int h = !in_grid ? 0 : heads_inner ? (int)(r % H) : (int)(r / max_len);
  const int t = !in_grid ? 0 : heads_inner ? (int)(r / H) : (int)(r % max_len);

  pdl_wait();
  const int asked = lengths ? max(lengths[b], 0) : max_len;
  const int len = min(asked, max_len);
  const bool fits = len <= cv.capacity;
  if (tid == 0 && blockIdx.x == 0 && lengths) {
    if (asked > max_len) atomicOr(cv.status, (int)kFlagMaxCtx);
    if (fits) cv.seq_lens[b] = len;  // no block of this grid reads seq_lens
    else atomicOr(cv.status, (int)kFlagCapacity);
  }
  const bool valid = fits && in_grid && t < len;
  __syncthreads();  // s_kcent

  if (__any_sync(kFull, valid)) {
    float u[E];
    const T* src = (is_v ? vin : kin) + b * stride_b + h * stride_h + t * stride_t + g * E;
    if (valid) {
      load_elems<E>(src, u);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) u[e] = 0.f;
    }
    const long slot = ((long)b * H + h) * cv.capacity + t;
    const int bits = is_v ? tb.v_bits : tb.k_bits;
    uint8_t* codes = (is_v ? cv.v_codes : cv.k_codes) + slot * (long)(bits * D / 8);
    // one fp16 norm per vector, or the affine codec's (scale, bias) per group
    constexpr int NH = AFF ? 2 * D / kAffineGroup : 1;
    uint16_t* norm = (is_v ? cv.v_norm : cv.k_norm) + slot * NH;
    uint8_t* signs = (!is_v && tb.qjl) ? cv.k_signs + slot * (long)(D / 8) : nullptr;
    uint16_t* rnorm = (!is_v && tb.qjl) ? cv.k_rnorm + slot : nullptr;
    encode_vector<D, E, AFF, BITS>(bits, u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent);
  }
  pdl_trigger();
}

// Appends of at most this many vectors in all (keys and values of every row)
// take the one-vector-per-warp layout: they are too few to fill the GPU, so
// latency rules; larger ones take the 32-channels-per-lane layout.
constexpr long kLatencyVectors = 4096;

// One grid over both kinds (small appends: one launch, latency) or, for the
// bulk layout, a grid of keys followed by a grid of values (each grid runs one
// code width, which keeps its unrolled encoder resident in the instruction
// cache); the grid that runs last publishes the lengths.
template <int D, typename T, int E, bool AFF, bool BULK>
cudaError_t launch_layout(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                          int n_new, cudaStream_t stream) {
  constexpr int VPB = kAppendThreads / (D / E);
  const long per_kind = (long)cv.kv_heads * n_new;
  const long blocks_per_kind = std::max<long>(1, (per_kind + VPB - 1) / VPB);
  if (2 * blocks_per_kind > 0x7fffffffL || cv.batch > 65535) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kAppendThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = quantize_append_kernel<D, T, E, AFF, BULK>;
  const T* kp = static_cast<const T*>(k);
  const T* vp = static_cast<const T*>(v);
  if constexpr (!BULK) {
    cfg.gridDim = dim3((unsigned)(2 * blocks_per_kind), (unsigned)cv.batch);
    return cudaLaunchKernelEx(&cfg, kern, tb, cv, kp, vp, n_new, (int)blocks_per_kind, 0, 1);
  } else {
    cfg.gridDim = dim3((unsigned)blocks_per_kind, (unsigned)cv.batch);
    auto of_width = [](int bits) {  // the kernel of one code width
      return bits == 2 ? quantize_append_kernel<D, T, E, AFF, BULK, 2>
           : bits == 3 ? quantize_append_kernel<D, T, E, AFF, BULK, 3>
                       : quantize_append_kernel<D, T, E, AFF, BULK, 4>;
    };
    const cudaError_t e =
        cudaLaunchKernelEx(&cfg, of_width(tb.k_bits), tb, cv, kp, vp, n_new, (int)blocks_per_kind, 0, 0);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, of_width(tb.v_bits), tb, cv, kp, vp, n_new, (int)blocks_per_kind, 1, 1);
  }
}

template <int D, typename T>
cudaError_t launch_typed(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                         int n_new, cudaStream_t stream) {
  const long vectors = 2L * cv.batch * cv.kv_heads * n_new;
  if (tb.affine) {
    if (vectors <= kLatencyVectors) return launch_layout<D, T, D / 32, true, false>(tb, cv, k, v, n_new, stream);
    return launch_layout<D, T, kBulkE, true, true>(tb, cv, k, v, n_new, stream);
  }
  if (vectors <= kLatencyVectors) return launch_layout<D, T, D / 32, false, false>(tb, cv, k, v, n_new, stream);
  return launch_layout<D, T, kBulkE, false, true>(tb, cv, k, v, n_new, stream);
}

template <int D, typename T, int E, bool AFF>
cudaError_t launch_convert_layout(const Tables& tb, const CacheView& cv, const void* k,
                                  const void* v, long sb, long sh, long st,
                                  const int32_t* lengths, int max_len, int kinds, bool small,
                                  cudaStream_t stream) {
  constexpr int VPB = kAppendThreads / (D / E);
  const long per_kind = (long)cv.kv_heads * max_len;
  const long blocks_per_kind = std::max<long>(1, (per_kind + VPB - 1) / VPB);
  if (kinds * blocks_per_kind > 0x7fffffffL || cv.batch > 65535) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kAppendThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = quantize_convert_kernel<D, T, E, AFF>;
  const T* kp = static_cast<const T*>(k);
  const T* vp = static_cast<const T*>(v);
  const int heads_inner = sh < st ? 1 : 0;
  // the bulk layout runs keys and values as two grids (one code width each,
  // as for the append)
  const bool split = !small && kinds == 2;
  cfg.gridDim = dim3((unsigned)((split ? 1 : kinds) * blocks_per_kind), (unsigned)cv.batch);
  if (!split) {
    return cudaLaunchKernelEx(&cfg, kern, tb, cv, kp, vp, sb, sh, st, lengths, max_len,
                              (int)blocks_per_kind, heads_inner, 0);
  }
  auto of_width = [](int bits) {  // the kernel of one code width
    return bits == 2 ? quantize_convert_kernel<D, T, E, AFF, 2>
         : bits == 3 ? quantize_convert_kernel<D, T, E, AFF, 3>
                     : quantize_convert_kernel<D, T, E, AFF, 4>;
  };
  cudaError_t e = cudaLaunchKernelEx(&cfg, of_width(tb.k_bits), tb, cv, kp, vp, sb, sh, st, lengths, max_len,
                                     (int)blocks_per_kind, heads_inner, 0);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, of_width(tb.v_bits), tb, cv, kp, vp, sb, sh, st, lengths, max_len,
                            (int)blocks_per_kind, heads_inner, 1);
}

template <int D, typename T>
cudaError_t launch_convert_typed(const Tables& tb, const CacheView& cv, const void* k,
                                 const void* v, long sb, long sh, long st, const int32_t* lengths,
                                 int max_len, int kinds, cudaStream_t stream) {
  const long vectors = (long)kinds * cv.batch * cv.kv_heads * max_len;
  const bool small = vectors <= kLatencyVectors;
  if (tb.affine)
    return small ? launch_convert_layout<D, T, D / 32, true>(tb, cv, k, v, sb, sh, st, lengths,
                                                             max_len, kinds, true, stream)
                 : launch_convert_layout<D, T, kBulkE, true>(tb, cv, k, v, sb, sh, st, lengths, max_len,
                                                             kinds, false, stream);
  return small ? launch_convert_layout<D, T, D / 32, false>(tb, cv, k, v, sb, sh, st, lengths,
                                                            max_len, kinds, true, stream)
               : launch_convert_layout<D, T, kBulkE, false>(tb, cv, k, v, sb, sh, st, lengths, max_len,
                                                            kinds, false, stream);
}

template <int D>
cudaError_t launch_convert_dim(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                               int dtype, long sb, long sh, long st, const int32_t* lengths,
                               int max_len, int kinds, cudaStream_t stream) {
  switch (dtype) {
    case kF32:
      return launch_convert_typed<D, float>(tb, cv, k, v, sb, sh, st, lengths, max_len, kinds, stream);
    case kBF16:
      return launch_convert_typed<D, __nv_bfloat16>(tb, cv, k, v, sb, sh, st, lengths, max_len, kinds,
                                                    stream);
    case kF16:
      return launch_convert_typed<D, __half>(tb, cv, k, v, sb, sh, st, lengths, max_len, kinds, stream);
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_dim(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                       int dtype, int n_new, cudaStream_t stream) {
  switch (dtype) {
    case kF32: return launch_typed<D, float>(tb, cv, k, v, n_new, stream);
    case kBF16: return launch_typed<D, __nv_bfloat16>(tb, cv, k, v, n_new, stream);
    case kF16: return launch_typed<D, __half>(tb, cv, k, v, n_new, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_quantize_append(const Tables& tb, const CacheView& cv, const void* k,
                                   const void* v, int dtype, int n_new, cudaStream_t stream) {
  switch (tb.d) {
    case 64: return launch_dim<64>(tb, cv, k, v, dtype, n_new, stream);
    case 128: return launch_dim<128>(tb, cv, k, v, dtype, n_new, stream);
    case 256: return launch_dim<256>(tb, cv, k, v, dtype, n_new, stream);
  }
  return cudaErrorNotSupported;
}

// Shared by the cache conversion (kinds = 2) and the weight encoding (kinds = 1).
cudaError_t launch_convert(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                           int dtype, long stride_b, long stride_h, long stride_t,
                           const int32_t* lengths, int max_len, int kinds, cudaStream_t stream) {
  switch (tb.d) {
    case 64:
      return launch_convert_dim<64>(tb, cv, k, v, dtype, stride_b, stride_h, stride_t, lengths,
                                    max_len, kinds, stream);
    case 128:
      return launch_convert_dim<128>(tb, cv, k, v, dtype, stride_b, stride_h, stride_t, lengths,
                                     max_len, kinds, stream);
    case 256:
      return launch_convert_dim<256>(tb, cv, k, v, dtype, stride_b, stride_h, stride_t, lengths,
                                     max_len, kinds, stream);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_quantize_cache(const Tables& tb, const CacheView& cv, const void* k,
                                  const void* v, int dtype, long stride_b, long stride_h,
                                  long stride_t, const int32_t* lengths, int max_len,
                                  cudaStream_t stream) {
  return launch_convert(tb, cv, k, v, dtype, stride_b, stride_h, stride_t, lengths, max_len, 2,
                        stream);
}

cudaError_t launch_weights_quantize(const Tables& tb, const void* w, int dtype, int rows, int k,
                                    uint8_t* codes, uint16_t* norms, cudaStream_t stream) {
  Tables t = tb;
  t.qjl = 0;  // weights carry only the MSE codes (the API rejects the affine codec)
  CacheView cv = {};
  cv.k_codes = codes;  // block j of row n is "token" n of "head" j
  cv.k_norm = norms;
  cv.batch = 1;
  cv.kv_heads = k / tb.d;
  cv.capacity = rows;
  return launch_convert(t, cv, w, w, dtype, 0, tb.d, k, nullptr, rows, 1, stream);
}

}  // namespace tq
