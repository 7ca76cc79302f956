// Quantize-and-append kernel of the TurboQuant KV-cache codec.
//
// Per d-vector (a key or a value of one token, one KV head):
//   norm -> sign flips -> Walsh-Hadamard -> scale -> bucket -> pack, and for
//   keys with QJL: residual -> its norm -> second rotation -> sign bits.
// ("TurboQuant Performance Benefits ...", "What Is TurboQuant?": random
// Hadamard rotation then MSE codebook quantization; "mlx-turboquant" README,
// "The 1-bit QJL residual": sign(RHT2(r)) and ||r||.)
//
// A group of d/32 adjacent lanes encodes one vector, each lane holding 32
// consecutive channels, so a warp encodes 32*32/d vectors at once.  Five of
// the transform's butterfly stages and five levels of the norm's pairwise tree
// run inside a lane; the rest are shuffles within the group.  A lane's 32
// codes fill whole 32-bit words of the packed row, so packing needs no
// cross-lane traffic.
//
// Every floating-point step is a single correctly rounded fp32 operation in
// one fixed order (__fadd_rn / __fsub_rn / __fmul_rn / __fsqrt_rn /
// __fdiv_rn; the cross-lane butterfly is an FMA by +-1, which rounds exactly
// like the addition or subtraction), so codes, sign bits and fp16 norms are
// reproducible bit for bit.
#include "tq_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

namespace tq {
namespace {

constexpr int kAppendWarps = 8;
constexpr int kAppendThreads = 32 * kAppendWarps;
constexpr unsigned kFull = 0xffffffffu;

// The lane's E consecutive input elements as fp32, read as 16-, 8- or 4-byte
// words (the row start is 16-byte aligned because k and v are, and the E
// elements of a lane span a multiple of that word).
template <int E, typename T>
__device__ __forceinline__ void load_elems(const T* p, float (&x)[E]) {
  constexpr int NB = E * (int)sizeof(T), NW = NB / 4;
  uint32_t w[NW];
  if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  } else if constexpr (NB == 8) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x;
    w[1] = v.y;
  } else {
    static_assert(NB == 4, "4, 8 or a multiple of 16 bytes per lane");
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
  }
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    if constexpr (sizeof(T) == 4) {
      x[i] = __uint_as_float(w[i]);
    } else if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      x[2 * i] = __uint_as_float(w[i] << 16);  // a bf16 is the top half of the fp32 of equal value
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
}

// Balanced pairwise sum over channel order 0..d-1: log2(E) levels over the
// lane's E channels, then one level per shuffle across the group of GL lanes
// (lanes hold aligned blocks of E channels, so the pairing is the tree's).
template <int E, int GL>
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
  for (int m = 1; m < GL; m <<= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, m));
  return s;
}

// Unnormalized Walsh-Hadamard transform in the canonical butterfly order:
// stage h pairs channels (j, j + h) with bit h of j clear -> (a + b, a - b).
// Stages h < E are inside the lane; stage E * m pairs lane l with lane l ^ m
// of the group: the lower lane computes own + partner, the upper partner - own.
template <int E, int GL>
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
  for (int m = 1; m < GL; m <<= 1) {
    const float sgn = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) u[e] = __fmaf_rn(u[e], sgn, __shfl_xor_sync(kFull, u[e], m));
  }
}

// Sign flips by the E bits of a +-1 vector (bit set: -1) for channels g*E ..
template <int E>
__device__ __forceinline__ void flip_signs(float (&u)[E], const uint32_t* mask, int g) {
  const uint32_t bits = mask[(g * E) >> 5] >> ((g * E) & 31);
#pragma unroll
  for (int e = 0; e < E; ++e) u[e] = __uint_as_float(__float_as_uint(u[e]) ^ (((bits >> e) & 1u) << 31));
}

// Stores a packed row whose lanes each hold `width` (< 32) consecutive bits at
// stream bit lane * width: the warp ORs the chunks into a shared word buffer
// and writes the `words` words (one vector per warp; every lane calls).
__device__ __forceinline__ void pack_store_shared(uint32_t* buf, int words, uint32_t chunk,
                                                  int width, int lane, bool store, uint32_t* dst) {
  if (lane < words) buf[lane] = 0u;
  __syncwarp();
  const int off = lane * width, w = off >> 5, sh = off & 31;
  atomicOr(&buf[w], chunk << sh);
  if (sh + width > 32) atomicOr(&buf[w + 1], chunk >> (32 - sh));
  __syncwarp();
  if (store && lane < words) dst[lane] = buf[lane];
  __syncwarp();
}

// #{q : p[q] < key} for the P = 2^(B-1) - 1 positive boundaries p (ascending),
// by a branch-free binary search.
template <int B>
__device__ __forceinline__ int count_below(float key, const float (&p)[8]) {
  if constexpr (B == 2) {
    return p[0] < key ? 1 : 0;
  } else if constexpr (B == 3) {
    int c = p[1] < key ? 2 : 0;
    c += (c ? p[2] : p[0]) < key ? 1 : 0;
    return c;
  } else {
    int c = p[3] < key ? 4 : 0;
    c += (c ? p[5] : p[1]) < key ? 2 : 0;
    const float piv = (c & 4) ? ((c & 2) ? p[6] : p[4]) : ((c & 2) ? p[2] : p[0]);
    c += piv < key ? 1 : 0;
    return c;
  }
}

// The code of z: #{j : bnd[j] < z} over all 2^B - 1 boundaries.  The codebook
// is odd-symmetric with bnd[L/2 - 1] = 0 and bnd[L/2 + q] = p[q] = -bnd[L/2 - 2 - q],
// so with a = |z|:  z > 0  ->  L/2 + #{p < a};  z <= 0  ->  L/2 - 1 - #{p <= a},
// and p <= a is p < nextup(a) (a non-negative, so nextup is one more in its bits).
template <int B>
__device__ __forceinline__ int bucket(float z, const float (&p)[8]) {
  constexpr int H = 1 << (B - 1);
  const bool pos = z > 0.f;
  const uint32_t abits = __float_as_uint(z) & 0x7fffffffu;
  const float key = __uint_as_float(abits + (pos ? 0u : 1u));
  const int c = count_below<B>(key, p);
  return pos ? H + c : H - 1 - c;
}

// Encodes the vector whose E-channel slice this lane holds in u (fp32) and
// stores codes, norm and, for QJL keys, the sketch.  g is the lane's index in
// its group of D / E lanes; `store` is false for lanes of a group past the
// end (they still take part in the group's shuffles).  `pack` is the warp's
// word buffer, used when a lane's bits do not fill whole words (E < 32, one
// vector per warp).
template <int D, int E, int B>
__device__ __forceinline__ void encode_store(float (&u)[E], const Tables& tb, bool is_v, int g,
                                             int lane, bool store, uint8_t* codes_row,
                                             uint16_t* norm, uint8_t* signs_row, uint16_t* rnorm,
                                             const float* s_kcent, uint32_t* pack) {
  constexpr int GL = D / E;
  constexpr int H = 1 << (B - 1);
  constexpr int LB = B * E;  // code bits per lane

  // 1. norm, stored as fp16
  float sq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(u[e], u[e]);
  const float n = __fsqrt_rn(tree_sum<E, GL>(sq));
  const __half n16 = __float2half_rn(n);

  // 2. rotation: sign flips, then the Walsh-Hadamard transform
  flip_signs<E>(u, tb.s1, g);
  fwht<E, GL>(u, lane);

  // 3.-5. scale, bucket, pack: code e at bit B*e of the lane's LB bits
  float p[8];
  const float* bnd = is_v ? tb.v_bnd : tb.k_bnd;
#pragma unroll
  for (int q = 0; q < H - 1; ++q) p[q] = bnd[H + q];
  const float inv = (n == 0.f) ? 0.f : __fdiv_rn(1.0f, n);
  const bool qjl = !is_v && tb.qjl;
  const float n16f = __half2float(n16);
  uint32_t words[(LB + 31) / 32];
#pragma unroll
  for (int w = 0; w < (LB + 31) / 32; ++w) words[w] = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = bucket<B>(__fmul_rn(u[e], inv), p);
    const int bit = B * e, w = bit >> 5, s = bit & 31;
    words[w] |= (uint32_t)c << s;
    if (s + B > 32) words[w + 1] |= (uint32_t)c >> (32 - s);
    // QJL keys: the residual r = u - fp16(n) * c[code] replaces u
    if (qjl) u[e] = __fsub_rn(u[e], __fmul_rn(n16f, s_kcent[c]));
  }
  if constexpr (LB % 32 == 0) {
    if (store) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(codes_row + g * (LB / 8));
#pragma unroll
      for (int w = 0; w < LB / 32; ++w) dst[w] = words[w];
    }
  } else {
    pack_store_shared(pack, B * D / 32, words[0], LB, lane, store,
                      reinterpret_cast<uint32_t*>(codes_row));
  }
  if (store && g == 0) *norm = __half_as_ushort(n16);

  // 6.-8. QJL sketch of keys: rho = ||r|| / sqrt(d); sign bits of H (s2 * r)
  if (qjl) {
#pragma unroll
    for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(u[e], u[e]);
    const float rho = __fdiv_rn(__fsqrt_rn(tree_sum<E, GL>(sq)), __fsqrt_rn((float)D));
    flip_signs<E>(u, tb.s2, g);
    fwht<E, GL>(u, lane);
    uint32_t sbits = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) sbits |= (u[e] >= 0.f ? 1u : 0u) << e;
    if constexpr (E % 32 == 0) {
      if (store) reinterpret_cast<uint32_t*>(signs_row)[g] = sbits;
    } else {
      pack_store_shared(pack, D / 32, sbits, E, lane, store, reinterpret_cast<uint32_t*>(signs_row));
    }
    if (store && g == 0) *rnorm = __half_as_ushort(__float2half_rn(rho));
  }
}

// Grid: (2 * blocks_per_kind, batch).  Blocks [0, blocks_per_kind) encode keys,
// the rest values, so a block's code width is uniform.  A group of D / E lanes
// encodes one vector: E = 32 packs 32 * 32 / D vectors into a warp (throughput:
// bulk appends); E = D / 32 gives each vector its own warp and keeps the
// unrolled code short (latency: a few tokens per row, as in a decode step).
template <int D, typename T, int E>
__global__ void __launch_bounds__(kAppendThreads)
    quantize_append_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                           const T* __restrict__ kin, const T* __restrict__ vin, int n_new,
                           int blocks_per_kind) {
  constexpr int GL = D / E;                     // lanes per vector
  constexpr int VPB = kAppendThreads / GL;      // vectors per block
  __shared__ float s_kcent[16];
  __shared__ uint32_t s_pack[kAppendWarps][E < 32 ? D / 8 + 1 : 1];

  const int tid = threadIdx.x, lane = tid & 31, g = lane & (GL - 1);
  if (tid < 16) s_kcent[tid] = tb.k_cent[tid];
  const int b = blockIdx.y;
  const bool is_v = (int)blockIdx.x >= blocks_per_kind;
  const long r = (long)(blockIdx.x - (is_v ? blocks_per_kind : 0)) * VPB + tid / GL;
  const long per_kind = (long)cv.kv_heads * n_new;
  const bool valid = r < per_kind;
  const int h = valid ? (int)(r / n_new) : 0, j = valid ? (int)(r % n_new) : 0;

  pdl_wait();
  // A small append (this layout) is a grid that is resident at once: let the
  // next kernel launch now, so that its set-up overlaps this one (it still waits
  // for this grid's completion before reading anything).  A bulk append keeps
  // the trigger at its end, so that waiting CTAs do not take its blocks' slots.
  if constexpr (E < 32) pdl_trigger();
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
    uint16_t* norm = (is_v ? cv.v_norm : cv.k_norm) + slot;
    uint8_t* signs = (!is_v && tb.qjl) ? cv.k_signs + slot * (long)(D / 8) : nullptr;
    uint16_t* rnorm = (!is_v && tb.qjl) ? cv.k_rnorm + slot : nullptr;
    uint32_t* pack = s_pack[tid >> 5];
    if (bits == 2)
      encode_store<D, E, 2>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent, pack);
    else if (bits == 3)
      encode_store<D, E, 3>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent, pack);
    else
      encode_store<D, E, 4>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent, pack);
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
  if constexpr (E == 32) pdl_trigger();
}

// Conversion of a dense cache.  Grid: (kinds * blocks_per_kind, batch) as for
// the append (kinds = 1 encodes keys only: weight blocks); the vectors (h, t)
// of a row are numbered with t outermost when the input's head stride is the
// smaller one (a [batch][T][heads][d] cache) and with h outermost otherwise,
// so consecutive lanes read consecutive memory.  Without `lengths` every row
// holds max_len vectors and no length or flag is written.
template <int D, typename T, int E>
__global__ void __launch_bounds__(kAppendThreads)
    quantize_convert_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                            const T* __restrict__ kin, const T* __restrict__ vin, long stride_b,
                            long stride_h, long stride_t, const int32_t* __restrict__ lengths,
                            int max_len, int blocks_per_kind, int heads_inner) {
  constexpr int GL = D / E;
  constexpr int VPB = kAppendThreads / GL;
  __shared__ float s_kcent[16];
  __shared__ uint32_t s_pack[kAppendWarps][E < 32 ? D / 8 + 1 : 1];

  const int tid = threadIdx.x, lane = tid & 31, g = lane & (GL - 1);
  if (tid < 16) s_kcent[tid] = tb.k_cent[tid];
  const int b = blockIdx.y, H = cv.kv_heads;
  const bool is_v = (int)blockIdx.x >= blocks_per_kind;
  const long r = (long)(blockIdx.x - (is_v ? blocks_per_kind : 0)) * VPB + tid / GL;
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
    uint16_t* norm = (is_v ? cv.v_norm : cv.k_norm) + slot;
    uint8_t* signs = (!is_v && tb.qjl) ? cv.k_signs + slot * (long)(D / 8) : nullptr;
    uint16_t* rnorm = (!is_v && tb.qjl) ? cv.k_rnorm + slot : nullptr;
    uint32_t* pack = s_pack[tid >> 5];
    if (bits == 2)
      encode_store<D, E, 2>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent, pack);
    else if (bits == 3)
      encode_store<D, E, 3>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent, pack);
    else
      encode_store<D, E, 4>(u, tb, is_v, g, lane, valid, codes, norm, signs, rnorm, s_kcent, pack);
  }
  pdl_trigger();
}

// Appends of at most this many vectors in all (keys and values of every row)
// take the one-vector-per-warp layout: they are too few to fill the GPU, so
// latency rules; larger ones take the 32-channels-per-lane layout.
constexpr long kLatencyVectors = 4096;

template <int D, typename T, int E>
cudaError_t launch_layout(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                          int n_new, cudaStream_t stream) {
  constexpr int VPB = kAppendThreads / (D / E);
  const long per_kind = (long)cv.kv_heads * n_new;
  const long blocks_per_kind = std::max<long>(1, (per_kind + VPB - 1) / VPB);
  if (2 * blocks_per_kind > 0x7fffffffL || cv.batch > 65535) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * blocks_per_kind), (unsigned)cv.batch);
  cfg.blockDim = dim3(kAppendThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_append_kernel<D, T, E>, tb, cv,
                            static_cast<const T*>(k), static_cast<const T*>(v), n_new,
                            (int)blocks_per_kind);
}

template <int D, typename T>
cudaError_t launch_typed(const Tables& tb, const CacheView& cv, const void* k, const void* v,
                         int n_new, cudaStream_t stream) {
  const long vectors = 2L * cv.batch * cv.kv_heads * n_new;
  if (vectors <= kLatencyVectors) return launch_layout<D, T, D / 32>(tb, cv, k, v, n_new, stream);
  return launch_layout<D, T, 32>(tb, cv, k, v, n_new, stream);
}

template <int D, typename T, int E>
cudaError_t launch_convert_layout(const Tables& tb, const CacheView& cv, const void* k,
                                  const void* v, long sb, long sh, long st,
                                  const int32_t* lengths, int max_len, int kinds,
                                  cudaStream_t stream) {
  constexpr int VPB = kAppendThreads / (D / E);
  const long per_kind = (long)cv.kv_heads * max_len;
  const long blocks_per_kind = std::max<long>(1, (per_kind + VPB - 1) / VPB);
  if (kinds * blocks_per_kind > 0x7fffffffL || cv.batch > 65535) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(kinds * blocks_per_kind), (unsigned)cv.batch);
  cfg.blockDim = dim3(kAppendThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_convert_kernel<D, T, E>, tb, cv,
                            static_cast<const T*>(k), static_cast<const T*>(v), sb, sh, st,
                            lengths, max_len, (int)blocks_per_kind, sh < st ? 1 : 0);
}

template <int D, typename T>
cudaError_t launch_convert_typed(const Tables& tb, const CacheView& cv, const void* k,
                                 const void* v, long sb, long sh, long st, const int32_t* lengths,
                                 int max_len, int kinds, cudaStream_t stream) {
  const long vectors = (long)kinds * cv.batch * cv.kv_heads * max_len;
  if (vectors <= kLatencyVectors)
    return launch_convert_layout<D, T, D / 32>(tb, cv, k, v, sb, sh, st, lengths, max_len, kinds,
                                               stream);
  return launch_convert_layout<D, T, 32>(tb, cv, k, v, sb, sh, st, lengths, max_len, kinds, stream);
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
  t.qjl = 0;  // weights carry only the MSE codes
  CacheView cv = {};
  cv.k_codes = codes;  // block j of row n is "token" n of "head" j
  cv.k_norm = norms;
  cv.batch = 1;
  cv.kv_heads = k / tb.d;
  cv.capacity = rows;
  return launch_convert(t, cv, w, w, dtype, 0, tb.d, k, nullptr, rows, 1, stream);
}

}  // namespace tq
