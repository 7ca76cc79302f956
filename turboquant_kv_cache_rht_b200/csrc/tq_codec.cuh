// Per-vector encoder of the TurboQuant KV-cache codec, shared by the append,
// conversion and weight-encoding kernels.
//
// Per d-vector (a key or a value of one token, one KV head):
//   norm -> sign flips -> Walsh-Hadamard -> scale -> bucket -> pack, and for
//   keys with QJL: residual -> its norm -> second rotation -> sign bits.
// ("TurboQuant Performance Benefits ...", "What Is TurboQuant?": random
// Hadamard rotation then MSE codebook quantization; "mlx-turboquant" README,
// "The 1-bit QJL residual": sign(RHT2(r)) and ||r||.)
//
// A group of d/E adjacent lanes encodes one vector, each lane holding E
// consecutive channels.  Every floating-point step is a single correctly
// rounded fp32 operation in one fixed order (__fadd_rn / __fsub_rn /
// __fmul_rn / __fsqrt_rn / __fdiv_rn; the cross-lane butterfly is an FMA by
// +-1, which rounds exactly like the addition or subtraction), so codes, sign
// bits and fp16 norms are reproducible bit for bit.
#pragma once

#include "tq_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

namespace tq {
namespace codec {

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
  for (int e = 0; e < E; ++e) u[e] = __uint_as_float(__float_as_uint(u[e]) ^ ((bits << (31 - e)) & 0x80000000u));
}

// Stores a packed row whose GL lanes (g = 0 .. GL-1 of the vector's group) each
// hold LB (< 32) consecutive bits at stream bit g * LB: lane g < W assembles
// word g of the row from the chunks of the lanes it spans (shuffles within
// the group, no shared memory) and stores it.  Every lane of the group calls.
template <int GL, int LB>
__device__ __forceinline__ void pack_store_shuffle(uint32_t chunk, int g, int lane, bool store,
                                                   uint32_t* dst) {
  static_assert(LB < 32 && (LB * GL) % 32 == 0, "sub-word chunks that fill whole words");
  constexpr int W = LB * GL / 32;          // words of the row
  constexpr int NS = (31 + LB - 1) / LB + 1;  // lanes one word can span
  const int base = lane - g, first = (32 * g) / LB, off = 32 * g - first * LB;
  uint32_t word = 0u;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const int src = first + i;
    const uint32_t c = __shfl_sync(kFull, chunk, base + (src < GL ? src : GL - 1), 32);
    const int pos = i * LB - off;  // where bit 0 of lane src's chunk lands in the word
    if (src < GL && pos < 32 && pos > -LB) word |= pos >= 0 ? (c << pos) : (c >> -pos);
  }
  if (store && g < W) dst[g] = word;
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

// Stores the lane's LB = B * E code bits (words[], code e at bit B * e) into
// the packed row at stream bit g * LB.
template <int D, int E, int B>
__device__ __forceinline__ void store_codes(const uint32_t (&words)[(B * E + 31) / 32], int g,
                                            int lane, bool store, uint8_t* codes_row) {
  constexpr int LB = B * E;
  if constexpr (LB % 32 == 0) {
    if (store) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(codes_row + g * (LB / 8));
#pragma unroll
      for (int w = 0; w < LB / 32; ++w) dst[w] = words[w];
    }
  } else {
    pack_store_shuffle<D / E, LB>(words[0], g, lane, store, reinterpret_cast<uint32_t*>(codes_row));
  }
}

// QJL sketch of the key residual r held in u: rnorm = fp16(||r|| / rdiv) and
// the sign bits of H (s2 * r) (bit set: >= 0).
template <int D, int E>
__device__ __forceinline__ void store_sketch(float (&u)[E], const Tables& tb, float rdiv, int g,
                                             int lane, bool store, uint8_t* signs_row,
                                             uint16_t* rnorm) {
  constexpr int GL = D / E;
  float sq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(u[e], u[e]);
  const float rho = __fdiv_rn(__fsqrt_rn(tree_sum<E, GL>(sq)), rdiv);
  flip_signs<E>(u, tb.s2, g);
  fwht<E, GL>(u, lane);
  uint32_t sbits = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) sbits |= (u[e] >= 0.f ? 1u : 0u) << e;
  if constexpr (E % 32 == 0) {
    if (store) reinterpret_cast<uint32_t*>(signs_row)[g] = sbits;
  } else {
    pack_store_shuffle<D / E, E>(sbits, g, lane, store, reinterpret_cast<uint32_t*>(signs_row));
  }
  if (store && g == 0) *rnorm = __half_as_ushort(__float2half_rn(rho));
}

// Encodes the vector whose E-channel slice this lane holds in u (fp32) and
// stores codes, norm and, for QJL keys, the sketch.  g is the lane's index in
// its group of D / E lanes; `store` is false for lanes of a group past the
// end (they still take part in the group's shuffles).  When a lane's bits do
// not fill whole words, the group assembles the words by shuffles.
template <int D, int E, int B>
__device__ __forceinline__ void encode_store(float (&u)[E], const Tables& tb, bool is_v, int g,
                                             int lane, bool store, uint8_t* codes_row,
                                             uint16_t* norm, uint8_t* signs_row, uint16_t* rnorm,
                                             const float* s_kcent) {
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
  store_codes<D, E, B>(words, g, lane, store, codes_row);
  if (store && g == 0) *norm = __half_as_ushort(n16);

  // 6.-8. QJL sketch of keys: rho = ||r|| / sqrt(d); sign bits of H (s2 * r)
  if (qjl) store_sketch<D, E>(u, tb, __fsqrt_rn((float)D), g, lane, store, signs_row, rnorm);
}

// The affine group-64 comparison codec ("mlx-turboquant" README, "Quantize
// the KV cache (long-context inference)" and "How it plugs in": an affine
// quantized cache with group size 64 whose keys are rotated).  Keys are coded
// in the rotated frame y = u * fp32(1/sqrt(d)), values as they are.  Per group
// of 64 channels (64 / E adjacent lanes): scale = fp16((max - min) / (2^B - 1)),
// bias = fp16(min), code = rint((y - bias) / scale) clamped to [0, 2^B - 1]
// (0 when scale is 0; fminf/fmaxf send a NaN quotient to 0).  meta receives
// the groups' (scale, bias) pairs, one 32-bit word each.  QJL keys then sketch
// r = y - (scale * code + bias) like the Lloyd-Max codec (||r||, undivided).
template <int D, int E, int B>
__device__ __forceinline__ void encode_affine_store(float (&u)[E], const Tables& tb, bool is_v,
                                                    int g, int lane, bool store,
                                                    uint8_t* codes_row, uint32_t* meta,
                                                    uint8_t* signs_row, uint16_t* rnorm) {
  constexpr int GL = D / E;
  constexpr int LB = B * E;
  constexpr int GG = kAffineGroup / E;  // lanes per channel group (2 .. 32)
  static_assert(E <= kAffineGroup && GG <= GL, "a lane's channels lie in one group");
  constexpr float kLevels = (float)((1 << B) - 1);

  if (!is_v) {
    flip_signs<E>(u, tb.s1, g);
    fwht<E, GL>(u, lane);
    const float rs = __fdiv_rn(1.0f, __fsqrt_rn((float)D));
#pragma unroll
    for (int e = 0; e < E; ++e) u[e] = __fmul_rn(u[e], rs);
  }
  // group minimum and maximum (exact: no rounding, so any order)
  float mn = u[0], mx = u[0];
#pragma unroll
  for (int e = 1; e < E; ++e) {
    mn = fminf(mn, u[e]);
    mx = fmaxf(mx, u[e]);
  }
#pragma unroll
  for (int m = 1; m < GG; m <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
  }
  // as values: -0 and +0 compare equal, so a zero extreme is taken as +0
  mn = __fadd_rn(mn, 0.0f);
  mx = __fadd_rn(mx, 0.0f);
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), kLevels));
  const __half b16 = __float2half_rn(mn);
  const float sf = __half2float(s16), bf = __half2float(b16);
  const bool qjl = !is_v && tb.qjl;
  uint32_t words[(LB + 31) / 32];
#pragma unroll
  for (int w = 0; w < (LB + 31) / 32; ++w) words[w] = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float t = sf == 0.f ? 0.f : rintf(__fdiv_rn(__fsub_rn(u[e], bf), sf));
    const int c = (int)fminf(fmaxf(t, 0.f), kLevels);
    const int bit = B * e, w = bit >> 5, s = bit & 31;
    words[w] |= (uint32_t)c << s;
    if (s + B > 32) words[w + 1] |= (uint32_t)c >> (32 - s);
    if (qjl) u[e] = __fsub_rn(u[e], __fadd_rn(__fmul_rn(sf, (float)c), bf));
  }
  store_codes<D, E, B>(words, g, lane, store, codes_row);
  if (store && g % GG == 0)
    meta[g / GG] = (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(b16) << 16);
  if (qjl) store_sketch<D, E>(u, tb, 1.0f, g, lane, store, signs_row, rnorm);
}

}  // namespace codec
}  // namespace tq
