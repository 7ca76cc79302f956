// Quantize-and-append kernel of the TurboQuant KV-cache codec.
//
// One warp encodes one d-vector (a key or a value of one token, one KV head):
//   norm -> sign flips -> Walsh-Hadamard (warp shuffles) -> scale -> bucket
//   -> pack, and for keys with QJL: residual -> its norm -> second rotation ->
//   sign bits.  ("TurboQuant Performance Benefits ...", "What Is TurboQuant?":
//   random Hadamard rotation then MSE codebook quantization; "mlx-turboquant"
//   README, "The 1-bit QJL residual": sign(RHT2(r)) and ||r||.)
//
// Every floating-point step is a single correctly rounded fp32 operation
// (__fadd_rn / __fmul_rn / __fsqrt_rn / __fdiv_rn, never contracted into an
// FMA) in one fixed order, so codes, sign bits and fp16 norms are reproducible
// bit for bit.  Lane l holds the E = d/32 consecutive channels l*E .. l*E+E-1.
#include "tq_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tq {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr unsigned kFull = 0xffffffffu;

template <typename T>
__device__ __forceinline__ float load_f32(const T* p);
template <>
__device__ __forceinline__ float load_f32<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}
template <>
__device__ __forceinline__ float load_f32<__half>(const __half* p) { return __half2float(__ldg(p)); }

__device__ __forceinline__ bool sign_neg(const uint32_t* mask, int i) {
  return (mask[i >> 5] >> (i & 31)) & 1u;
}

// Balanced pairwise sum of the E in-lane values, then across lanes: the tree
// over channel order 0..d-1 (lanes hold aligned power-of-two blocks).
template <int E>
__device__ __forceinline__ float tree_sum(const float (&a)[E]) {
  float t[E];
#pragma unroll
  for (int e = 0; e < E; ++e) t[e] = a[e];
#pragma unroll
  for (int w = 1; w < E; w <<= 1)
#pragma unroll
    for (int e = 0; e < E; e += 2 * w) t[e] = __fadd_rn(t[e], t[e + w]);
  float s = t[0];
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, m));
  return s;
}

// Unnormalized Walsh-Hadamard transform in the canonical butterfly order:
// stage h pairs channels (j, j+h) with bit h of j clear -> (a+b, a-b).
template <int E>
__device__ __forceinline__ void fwht(float (&u)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1)
#pragma unroll
    for (int j = 0; j < E; ++j)
      if ((j & h) == 0) {
        const float a = u[j], b = u[j + h];
        u[j] = __fadd_rn(a, b);
        u[j + h] = __fsub_rn(a, b);
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float p = __shfl_xor_sync(kFull, u[e], m);
      u[e] = (lane & m) ? __fsub_rn(p, u[e]) : __fadd_rn(u[e], p);
    }
  }
}

// ORs the lane's `width`-bit chunk (at stream bit lane*width) into the warp's
// word buffer, then writes the `words` words to dst.
__device__ __forceinline__ void pack_store(uint32_t* buf, int words, uint32_t chunk, int width,
                                           int lane, uint32_t* dst) {
  if (lane < words) buf[lane] = 0u;
  __syncwarp();
  const int off = lane * width;
  const int w = off >> 5, sh = off & 31;
  atomicOr(&buf[w], chunk << sh);
  if (sh + width > 32) atomicOr(&buf[w + 1], chunk >> (32 - sh));
  __syncwarp();
  if (lane < words) dst[lane] = buf[lane];
  __syncwarp();
}

template <int D, typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    quantize_append_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                           const T* __restrict__ kin, const T* __restrict__ vin, int n_new) {
  constexpr int E = D / 32;
  __shared__ float s_cent[2][16];
  __shared__ float s_bnd[2][16];
  __shared__ uint32_t s_words[kWarpsPerBlock][D / 8 + 1];

  const int tid = threadIdx.x;
  if (tid < 16) {
    s_cent[0][tid] = tb.k_cent[tid];
    s_cent[1][tid] = tb.v_cent[tid];
    s_bnd[0][tid] = tb.k_bnd[tid];
    s_bnd[1][tid] = tb.v_bnd[tid];
  }
  const int b = blockIdx.y;
  pdl_wait();
  const int base = cv.seq_lens[b];
  const bool fits = base >= 0 && base <= cv.capacity - n_new;
  if (!fits && tid == 0 && blockIdx.x == 0) atomicOr(cv.status, (int)kFlagCapacity);
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const long per_kind = (long)cv.kv_heads * n_new;
  const long vb = (long)blockIdx.x * kWarpsPerBlock + warp;
  if (fits && vb < 2 * per_kind) {
    const int is_v = vb >= per_kind;
    const long r = is_v ? vb - per_kind : vb;
    const int h = (int)(r / n_new), j = (int)(r % n_new);
    const int bits = is_v ? tb.v_bits : tb.k_bits;
    const int levels = 1 << bits;
    const T* src = (is_v ? vin : kin) + (((long)b * cv.kv_heads + h) * n_new + j) * D + lane * E;

    float x[E];
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = load_f32<T>(src + e);

    // 1. norm, stored as fp16
    float sq[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(x[e], x[e]);
    const float n = __fsqrt_rn(tree_sum<E>(sq));
    const __half n16 = __float2half_rn(n);

    // 2. rotation (signs, then Walsh-Hadamard)
    float u[E];
#pragma unroll
    for (int e = 0; e < E; ++e) u[e] = sign_neg(tb.s1, lane * E + e) ? -x[e] : x[e];
    fwht<E>(u, lane);

    // 3.-4. normalize and bucket: code = #{boundaries strictly below z}
    const float inv = (n == 0.f) ? 0.f : __fdiv_rn(1.0f, n);
    const float* bnd = s_bnd[is_v];
    int code[E];
    uint32_t chunk = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float z = __fmul_rn(u[e], inv);
      int c = 0;
#pragma unroll
      for (int q = 0; q < 15; ++q)
        if (q < levels - 1) c += (bnd[q] < z) ? 1 : 0;
      code[e] = c;
      chunk |= (uint32_t)c << (bits * e);
    }

    // 5. pack and store
    const long slot = ((long)b * cv.kv_heads + h) * cv.capacity + base + j;
    const int code_words = bits * D / 32;
    uint8_t* codes = is_v ? cv.v_codes : cv.k_codes;
    pack_store(s_words[warp], code_words, chunk, bits * E, lane,
               reinterpret_cast<uint32_t*>(codes + slot * (long)(bits * D / 8)));
    if (lane == 0) (is_v ? cv.v_norm : cv.k_norm)[slot] = __half_as_ushort(n16);

    // 6.-8. QJL residual sketch of keys
    if (!is_v && tb.qjl) {
      const float n16f = __half2float(n16);
      const float* cent = s_cent[0];
      float res[E], rsq[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        res[e] = __fsub_rn(u[e], __fmul_rn(n16f, cent[code[e]]));
        rsq[e] = __fmul_rn(res[e], res[e]);
      }
      const float rho = __fdiv_rn(__fsqrt_rn(tree_sum<E>(rsq)), __fsqrt_rn((float)D));
#pragma unroll
      for (int e = 0; e < E; ++e) res[e] = sign_neg(tb.s2, lane * E + e) ? -res[e] : res[e];
      fwht<E>(res, lane);
      uint32_t sbits = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) sbits |= (res[e] >= 0.f ? 1u : 0u) << e;
      pack_store(s_words[warp], D / 32, sbits, E, lane,
                 reinterpret_cast<uint32_t*>(cv.k_signs + slot * (long)(D / 8)));
      if (lane == 0) cv.k_rnorm[slot] = __half_as_ushort(__float2half_rn(rho));
    }
  }

  // The last block of this batch row to finish publishes the new length.  Every
  // block read seq_lens[b] before taking its ticket, so none can see the update.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int ticket = atomicAdd(&cv.append_sync[b], 1);
    if (ticket == (int)gridDim.x - 1) {
      if (fits) cv.seq_lens[b] = base + n_new;
      cv.append_sync[b] = 0;
    }
  }
  pdl_trigger();
}

template <int D, typename T>
cudaError_t launch_typed(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                         int n_new, cudaStream_t stream) {
  const long vectors = 2L * cv.kv_heads * n_new;
  const long blocks = (vectors + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7fffffffL || cv.batch > 65535) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, (unsigned)cv.batch);
  cfg.blockDim = dim3(kWarpsPerBlock * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_append_kernel<D, T>, tb, cv, static_cast<const T*>(k),
                            static_cast<const T*>(v), n_new);
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
    case 128: return launch_dim<128>(tb, cv, k, v, dtype, n_new, stream);
    case 256: return launch_dim<256>(tb, cv, k, v, dtype, n_new, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace tq
