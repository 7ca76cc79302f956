// Decode attention: split planning, dispatch, and the split-merge kernel.
#include "tq_decode_impl.cuh"

#include <algorithm>

namespace tq {

namespace {

constexpr int kCombineThreads = 128;
constexpr int kMaxSplits = 512;
// Split target: about four CTAs per SM of a 148-SM B200.  Fixed (not queried)
// so that the workspace size is a pure function of the call's sizes.
constexpr long kTargetCtas = 148L * 4;

// Merges the splits of one (query head, batch row) in split order and applies
// the inverse rotation: o = D1 H (sum_s w_s o_s) / (sum_s w_s l_s) / d with
// w_s = 2^(m_s - max m) ("How to Use TurboQuant ...", "What is TurboQuant?":
// _rht_inverse; the 1/d collects the rotation's and the dequantization's
// 1/sqrt(d)).
template <int D>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __grid_constant__ Tables tb, const int32_t* __restrict__ seq_lens,
                   int32_t* status, const float* __restrict__ ws, int q_heads, int splits,
                   int chunk, int capacity, float* __restrict__ out) {
  __shared__ float o[D];
  __shared__ float wgt[kMaxSplits];
  __shared__ float inv_l;
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int T = min(max(seq_lens[b], 0), capacity);
  if (tid == 0 && h == 0 && T > (long)splits * chunk) atomicOr(status, (int)kFlagMaxCtx);
  const int S = min(splits, (T + chunk - 1) / chunk);
  float* dst = out + ((long)b * q_heads + h) * D;
  if (S <= 0) {
    for (int i = tid; i < D; i += kCombineThreads) dst[i] = 0.f;
    return;
  }
  const float* src = ws + ((long)b * q_heads + h) * splits * (D + 2);
  if (tid == 0) {
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, src[(long)s * (D + 2)]);
    float l = 0.f;
    for (int s = 0; s < S; ++s) {
      const float w = exp2f(src[(long)s * (D + 2)] - m);
      wgt[s] = w;
      l = fmaf(src[(long)s * (D + 2) + 1], w, l);
    }
    inv_l = 1.0f / l;
  }
  __syncthreads();
  for (int i = tid; i < D; i += kCombineThreads) {
    float a = 0.f;
    for (int s = 0; s < S; ++s) a = fmaf(src[(long)s * (D + 2) + 2 + i], wgt[s], a);
    o[i] = a * inv_l;
  }
#pragma unroll 1
  for (int hh = 1; hh < D; hh <<= 1) {
    __syncthreads();
    for (int p = tid; p < D / 2; p += kCombineThreads) {
      const int j = (p / hh) * 2 * hh + (p % hh);
      const float a = o[j], c = o[j + hh];
      o[j] = a + c;
      o[j + hh] = a - c;
    }
  }
  __syncthreads();
  const float inv_d = 1.0f / (float)D;
  for (int i = tid; i < D; i += kCombineThreads) {
    const float v = o[i] * inv_d;
    dst[i] = ((tb.s1[i >> 5] >> (i & 31)) & 1u) ? -v : v;
  }
}

}  // namespace

DecodePlan plan_decode(int batch, int kv_heads, int max_ctx, int head_dim) {
  (void)head_dim;
  const long tiles = std::max<long>(1, (max_ctx + kDecTile - 1) / kDecTile);
  const long units = std::max<long>(1, (long)batch * kv_heads);
  long s = (kTargetCtas + units - 1) / units;
  s = std::max<long>(1, std::min<long>({s, tiles, (long)kMaxSplits}));
  const long per = (tiles + s - 1) / s;
  DecodePlan p;
  p.splits = (int)((tiles + per - 1) / per);
  p.chunk = (int)(per * kDecTile);
  return p;
}

size_t decode_workspace_bytes(const DecodePlan& plan, int batch, int q_heads, int head_dim) {
  return (size_t)batch * q_heads * plan.splits * (head_dim + 2) * sizeof(float);
}

bool decode_supported(int head_dim, int group, int k_bits, int v_bits, int qjl) {
  (void)qjl;
  if (head_dim != 128 && head_dim != 256) return false;
  if (group != 1 && group != 2 && group != 4 && group != 8) return false;
  if (k_bits < 2 || k_bits > 4) return false;
  return v_bits == k_bits || v_bits == k_bits + 1;
}

cudaError_t launch_decode(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                          int q_heads, float scale, const DecodePlan& plan, float* out,
                          float* workspace, cudaStream_t stream) {
  const float scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = cudaErrorNotSupported;
  if (tb.d == 128)
    e = launch_decode_dim<128>(tb, cv, q, dtype, q_heads, scale_log2, plan, workspace, stream);
  else if (tb.d == 256)
    e = launch_decode_dim<256>(tb, cv, q, dtype, q_heads, scale_log2, plan, workspace, stream);
  if (e != cudaSuccess) return e;
  dim3 grid(q_heads, cv.batch);
  if (tb.d == 128)
    combine_kernel<128><<<grid, kCombineThreads, 0, stream>>>(tb, cv.seq_lens, cv.status, workspace,
                                                             q_heads, plan.splits, plan.chunk, cv.capacity, out);
  else
    combine_kernel<256><<<grid, kCombineThreads, 0, stream>>>(tb, cv.seq_lens, cv.status, workspace,
                                                             q_heads, plan.splits, plan.chunk, cv.capacity, out);
  return cudaGetLastError();
}

}  // namespace tq
