// Fused decode attention on the packed TurboQuant cache (kernel template).
//
// One CTA handles one (split of the context, KV head, batch row) for all G
// query heads that share the KV head ("How to Use TurboQuant ...", "What is
// TurboQuant?": fused scoring kernels on packed low-bit data, GQA heads
// repeated over a shared KV head; "TurboQuant Performance Benefits ...",
// "Custom Metal Kernel Implementation": scores fused with value aggregation,
// no dequantization pass).  Per 128-token tile:
//   - cp.async stages the tile's key codes, value codes, norms (and QJL sign
//     words and residual norms) into shared memory, one tile ahead;
//   - key phase: thread t scores token t for the G heads directly on its code
//     bits: sum_i q_rot[g][i] * c_K[code_i] through a shared-memory codebook,
//     times the token's norm, plus the QJL sign-sketch term;
//   - online softmax (running max / sum, base-2 exponent);
//   - value phase: lane l accumulates channels l*d/32 .. for the G heads over
//     the tile's tokens, again straight from the packed codes.
// The rotated query and all constant factors (softmax scale, log2(e), the
// 1/sqrt(d) of the rotation and of the dequantization, sqrt(pi/(2d)) of QJL)
// are folded into the query once per CTA.  The partial (max, sum, output) of
// each head goes to the workspace; a combine kernel merges the splits in a
// fixed order and applies the inverse rotation.
#pragma once

#include "tq_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tq {

constexpr int kDecThreads = 128;
constexpr int kDecTile = 128;  // tokens per tile: one per thread in the key phase

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ float load_any(const void* p, long i, int dtype) {
  switch (dtype) {
    case kBF16: return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    case kF16: return __half2float(static_cast<const __half*>(p)[i]);
    default: return static_cast<const float*>(p)[i];
  }
}

template <int G>
__device__ __forceinline__ void load_group(const float* p, float (&o)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int g = 0; g < G; g += 4) {
      const float4 v = *reinterpret_cast<const float4*>(p + g);
      o[g] = v.x; o[g + 1] = v.y; o[g + 2] = v.z; o[g + 3] = v.w;
    }
  } else if constexpr (G == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x; o[1] = v.y;
  } else {
    o[0] = p[0];
  }
}

// code of channel i in a little-endian bit stream held in registers
template <int B>
__device__ __forceinline__ uint32_t code_at(const uint32_t* words, int i) {
  const int off = B * i, w = off >> 5, s = off & 31;
  if (s + B <= 32) return (words[w] >> s) & ((1u << B) - 1u);
  return __funnelshift_r(words[w], words[w + 1], s) & ((1u << B) - 1u);
}

template <int D, int G, int KB, int VB, bool QJL>
struct DecodeGeom {
  static constexpr int kBytes = KB * D / 8;
  static constexpr int vBytes = VB * D / 8;
  static constexpr int sBytes = QJL ? D / 8 : 0;
  static constexpr int kChunks = kBytes / 16;
  static constexpr int vChunks = vBytes / 16;
  static constexpr int sChunks = sBytes / 16;
  // Odd row strides (in 16-byte chunks) keep the key phase's row-per-thread
  // 128-bit reads free of bank conflicts.
  static constexpr int kStride = (kChunks & 1) ? kChunks : kChunks + 1;
  static constexpr int sStride = QJL ? ((sChunks & 1) ? sChunks : sChunks + 1) : 0;
  static constexpr int offK = 0;
  static constexpr int offV = offK + kDecTile * kStride * 16;
  static constexpr int offS = offV + kDecTile * vChunks * 16 + 16;
  static constexpr int offKN = offS + kDecTile * sStride * 16;
  static constexpr int offVN = offKN + kDecTile * 2;
  static constexpr int offRN = offVN + kDecTile * 2;
  static constexpr int stage = offRN + (QJL ? kDecTile * 2 : 0);
  static constexpr int stageAligned = (stage + 127) / 128 * 128;
  // shared-memory map after the two stages (bytes)
  static constexpr int offQK = 2 * stageAligned;               // float [D][G]
  static constexpr int offQQ = offQK + D * G * 4;               // float [D][G] (QJL)
  static constexpr int offQB = offQQ + (QJL ? D * G * 4 : 0);   // float [G][D] scratch
  static constexpr int offPW = offQB + D * G * 4;               // float [tile][G]
  static constexpr int offLUT = offPW + kDecTile * G * 4;       // float [2][16]
  static constexpr int offRED = offLUT + 32 * 4;                // float [4][G]
  static constexpr int total = offRED + 4 * G * 4;
  static_assert(4 * G * D * 4 <= 2 * stageAligned, "epilogue buffer must fit in the stages");
  static_assert(VB * (D / 32) <= 32, "value chunk per lane must fit a word");
};

template <int D, int G, int KB, int VB, bool QJL>
__global__ void __launch_bounds__(kDecThreads)
    decode_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                  const void* __restrict__ q, int q_dtype, int q_heads, float scale_log2,
                  int chunk, int splits, float* __restrict__ ws) {
  using Geo = DecodeGeom<D, G, KB, VB, QJL>;
  constexpr int EV = D / 32;  // value channels per lane
  extern __shared__ __align__(128) uint8_t smem[];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int T = min(max(cv.seq_lens[b], 0), cv.capacity);  // never read past a row
  const int t_begin = split * chunk;
  if (t_begin >= T) return;
  const int t_end = min(t_begin + chunk, T);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long row = (long)b * cv.kv_heads + kvh;
  const long row_slot = row * cv.capacity;

  float* qk = reinterpret_cast<float*>(smem + Geo::offQK);
  float* qq = reinterpret_cast<float*>(smem + Geo::offQQ);
  float* qb = reinterpret_cast<float*>(smem + Geo::offQB);
  float* pw = reinterpret_cast<float*>(smem + Geo::offPW);
  float* lutK = reinterpret_cast<float*>(smem + Geo::offLUT);
  float* lutV = lutK + 16;
  float* red = reinterpret_cast<float*>(smem + Geo::offRED);

  auto issue_tile = [&](int stage, int start) {
    uint8_t* st = smem + stage * Geo::stageAligned;
    const int n_valid = min(kDecTile, t_end - start);
    const int rows = (n_valid + 15) & ~15;  // within capacity (a multiple of 16)
    const uint8_t* kc = cv.k_codes + (row_slot + start) * Geo::kBytes;
    for (int c = tid; c < rows * Geo::kChunks; c += kDecThreads) {
      const int r = c / Geo::kChunks, col = c - r * Geo::kChunks;
      cp_async16(st + Geo::offK + (r * Geo::kStride + col) * 16, kc + r * Geo::kBytes + col * 16);
    }
    const uint8_t* vc = cv.v_codes + (row_slot + start) * Geo::vBytes;
    for (int c = tid; c < rows * Geo::vChunks; c += kDecThreads)
      cp_async16(st + Geo::offV + c * 16, vc + c * 16);
    if constexpr (QJL) {
      const uint8_t* sc = cv.k_signs + (row_slot + start) * Geo::sBytes;
      for (int c = tid; c < rows * Geo::sChunks; c += kDecThreads) {
        const int r = c / Geo::sChunks, col = c - r * Geo::sChunks;
        cp_async16(st + Geo::offS + (r * Geo::sStride + col) * 16, sc + r * Geo::sBytes + col * 16);
      }
    }
    const int nchunks = rows * 2 / 16;
    for (int c = tid; c < nchunks; c += kDecThreads) {
      cp_async16(st + Geo::offKN + c * 16, reinterpret_cast<const uint8_t*>(cv.k_norm + row_slot + start) + c * 16);
      cp_async16(st + Geo::offVN + c * 16, reinterpret_cast<const uint8_t*>(cv.v_norm + row_slot + start) + c * 16);
      if constexpr (QJL)
        cp_async16(st + Geo::offRN + c * 16, reinterpret_cast<const uint8_t*>(cv.k_rnorm + row_slot + start) + c * 16);
    }
  };

  issue_tile(0, t_begin);
  cp_async_commit();

  // ---- rotate the G queries once: qk = H (s1 * q) * scale*log2(e)/d,
  //      qq = H (s2 * H (s1 * q)) * scale*log2(e)*sqrt(pi/(2d))/d
  if (tid < 16) {
    lutK[tid] = tb.k_cent[tid];
    lutV[tid] = tb.v_cent[tid];
  }
  const long q_base = ((long)b * q_heads + (long)kvh * G) * D;
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int ch = i % D;
    const float x = load_any(q, q_base + i, q_dtype);
    qb[i] = ((tb.s1[ch >> 5] >> (ch & 31)) & 1u) ? -x : x;
  }
  auto fwht_rows = [&]() {
#pragma unroll 1
    for (int h = 1; h < D; h <<= 1) {
      __syncthreads();
      for (int p = tid; p < G * D / 2; p += kDecThreads) {
        const int g = p / (D / 2), k = p % (D / 2);
        const int j = (k / h) * 2 * h + (k % h);
        float* r = qb + g * D;
        const float a = r[j], c = r[j + h];
        r[j] = a + c;
        r[j + h] = a - c;
      }
    }
    __syncthreads();
  };
  fwht_rows();
  const float ck = scale_log2 / (float)D;
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, ch = i % D;
    qk[ch * G + g] = qb[i] * ck;
  }
  if constexpr (QJL) {
    __syncthreads();
    for (int i = tid; i < G * D; i += kDecThreads) {
      const int ch = i % D;
      if ((tb.s2[ch >> 5] >> (ch & 31)) & 1u) qb[i] = -qb[i];
    }
    fwht_rows();
    const float cq = scale_log2 * sqrtf(3.14159265358979f / (2.0f * D)) / (float)D;
    for (int i = tid; i < G * D; i += kDecThreads) {
      const int g = i / D, ch = i % D;
      qq[ch * G + g] = qb[i] * cq;
    }
  }

  float m_run[G], l_part[G], acc[G][EV];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_part[g] = 0.f;
#pragma unroll
    for (int c = 0; c < EV; ++c) acc[g][c] = 0.f;
  }

  int it = 0;
  for (int start = t_begin; start < t_end; start += kDecTile, ++it) {
    const int stage = it & 1;
    const bool has_next = start + kDecTile < t_end;
    if (has_next) {
      issue_tile(stage ^ 1, start + kDecTile);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint8_t* st = smem + stage * Geo::stageAligned;
    const int n_valid = min(kDecTile, t_end - start);

    // ---- key phase: thread tid scores token tid for the G heads
    float s[G];
    {
      uint32_t kw[Geo::kChunks * 4];
      const uint4* kr = reinterpret_cast<const uint4*>(st + Geo::offK + tid * Geo::kStride * 16);
#pragma unroll
      for (int c = 0; c < Geo::kChunks; ++c) {
        const uint4 v = kr[c];
        kw[4 * c] = v.x; kw[4 * c + 1] = v.y; kw[4 * c + 2] = v.z; kw[4 * c + 3] = v.w;
      }
      float ak[G];
#pragma unroll
      for (int g = 0; g < G; ++g) ak[g] = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const float val = lutK[code_at<KB>(kw, i)];
        float qv[G];
        load_group<G>(qk + i * G, qv);
#pragma unroll
        for (int g = 0; g < G; ++g) ak[g] = fmaf(qv[g], val, ak[g]);
      }
      const float kn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + Geo::offKN)[tid]));
#pragma unroll
      for (int g = 0; g < G; ++g) s[g] = ak[g] * kn;
      if constexpr (QJL) {
        uint32_t sw[Geo::sChunks * 4];
        const uint4* sr = reinterpret_cast<const uint4*>(st + Geo::offS + tid * Geo::sStride * 16);
#pragma unroll
        for (int c = 0; c < Geo::sChunks; ++c) {
          const uint4 v = sr[c];
          sw[4 * c] = v.x; sw[4 * c + 1] = v.y; sw[4 * c + 2] = v.z; sw[4 * c + 3] = v.w;
        }
        float aq[G];
#pragma unroll
        for (int g = 0; g < G; ++g) aq[g] = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) {
          // bit 1 -> +q, bit 0 -> -q: flip the float sign bit when the code bit is 0
          const uint32_t flip = ((~sw[i >> 5] >> (i & 31)) & 1u) << 31;
          float qv[G];
          load_group<G>(qq + i * G, qv);
#pragma unroll
          for (int g = 0; g < G; ++g) aq[g] += __uint_as_float(__float_as_uint(qv[g]) ^ flip);
        }
        const float rn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + Geo::offRN)[tid]));
#pragma unroll
        for (int g = 0; g < G; ++g) s[g] = fmaf(aq[g], rn, s[g]);
      }
      if (tid >= n_valid) {
#pragma unroll
        for (int g = 0; g < G; ++g) s[g] = -INFINITY;
      }
    }

    // ---- online softmax over the tile
    float tmax[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float m = s[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      tmax[g] = m;
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) red[warp * G + g] = tmax[g];
    }
    __syncthreads();
    const float vn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + Geo::offVN)[tid]));
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float tm = fmaxf(fmaxf(red[g], red[G + g]), fmaxf(red[2 * G + g], red[3 * G + g]));
      const float m_new = fmaxf(m_run[g], tm);
      alpha[g] = exp2f(m_run[g] - m_new);
      const float p = exp2f(s[g] - m_new);
      l_part[g] = fmaf(l_part[g], alpha[g], p);
      pw[tid * G + g] = (tid < n_valid) ? p * vn : 0.f;
      m_run[g] = m_new;
#pragma unroll
      for (int c = 0; c < EV; ++c) acc[g][c] *= alpha[g];
    }
    __syncthreads();

    // ---- value phase: warp w takes tokens w, w+4, ...; lane owns EV channels
    {
      constexpr int width = VB * EV;
      const int off = lane * width, w0 = off >> 5, sh = off & 31;
      const uint32_t* vrow = reinterpret_cast<const uint32_t*>(st + Geo::offV);
      for (int t = warp; t < n_valid; t += 4) {
        const uint32_t* r = vrow + t * (Geo::vBytes / 4);
        const uint32_t bits = __funnelshift_r(r[w0], r[w0 + 1], sh);
        float pv[G];
        load_group<G>(pw + t * G, pv);
#pragma unroll
        for (int c = 0; c < EV; ++c) {
          const float val = lutV[(bits >> (VB * c)) & ((1u << VB) - 1u)];
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g][c] = fmaf(pv[g], val, acc[g][c]);
        }
      }
    }
    __syncthreads();
  }

  // ---- epilogue: reduce the per-thread sums and the four warps' accumulators
  float l_tot[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float l = l_part[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    l_tot[g] = l;
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) red[warp * G + g] = l_tot[g];
  }
  float* obuf = reinterpret_cast<float*>(smem);  // [4][G][D], the stages are free now
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < EV; ++c) obuf[(warp * G + g) * D + lane * EV + c] = acc[g][c];
  __syncthreads();
  float* dst = ws + ((long)(b * q_heads + kvh * G) * splits + split) * (D + 2);
  const long head_stride = (long)splits * (D + 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, ch = i % D;
    const float o = ((obuf[(0 * G + g) * D + ch] + obuf[(1 * G + g) * D + ch]) +
                     obuf[(2 * G + g) * D + ch]) + obuf[(3 * G + g) * D + ch];
    dst[g * head_stride + 2 + ch] = o;
  }
  if (tid < G) {
    const int g = tid;
    dst[g * head_stride + 0] = m_run[g];
    dst[g * head_stride + 1] = ((red[g] + red[G + g]) + red[2 * G + g]) + red[3 * G + g];
  }
}

// Launches decode_kernel for one compile-time shape (grid: splits x kv_heads x batch).
template <int D, int G, int KB, int VB, bool QJL>
cudaError_t launch_decode_shape(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                                int q_heads, float scale_log2, const DecodePlan& plan,
                                float* ws, cudaStream_t stream) {
  using Geo = DecodeGeom<D, G, KB, VB, QJL>;
  auto kern = decode_kernel<D, G, KB, VB, QJL>;
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::total);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  dim3 grid(plan.splits, cv.kv_heads, cv.batch);
  kern<<<grid, kDecThreads, Geo::total, stream>>>(tb, cv, q, dtype, q_heads, scale_log2,
                                                  plan.chunk, plan.splits, ws);
  return cudaGetLastError();
}

// Per-head-dim dispatch over (group, k_bits, v_bits, qjl); defined in the
// tq_decode_d<D>.cu translation units.
template <int D>
cudaError_t launch_decode_dim(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                              int q_heads, float scale_log2, const DecodePlan& plan, float* ws,
                              cudaStream_t stream);

template <int D>
cudaError_t dispatch_decode_dim(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                                int q_heads, float scale_log2, const DecodePlan& plan, float* ws,
                                cudaStream_t stream) {
  const int G = q_heads / cv.kv_heads;
#define TQ_CASE(GG, KB, VB, QJ)                                                               \
  if (G == GG && tb.k_bits == KB && tb.v_bits == VB && (tb.qjl != 0) == QJ)                   \
    return launch_decode_shape<D, GG, KB, VB, QJ>(tb, cv, q, dtype, q_heads, scale_log2, plan, \
                                                  ws, stream);
#define TQ_BITS(GG, QJ) \
  TQ_CASE(GG, 2, 2, QJ) TQ_CASE(GG, 2, 3, QJ) TQ_CASE(GG, 3, 3, QJ) TQ_CASE(GG, 3, 4, QJ) TQ_CASE(GG, 4, 4, QJ)
#define TQ_GROUP(GG) TQ_BITS(GG, false) TQ_BITS(GG, true)
  TQ_GROUP(1)
  TQ_GROUP(2)
  TQ_GROUP(4)
  TQ_GROUP(8)
#undef TQ_GROUP
#undef TQ_BITS
#undef TQ_CASE
  return cudaErrorNotSupported;
}

}  // namespace tq
