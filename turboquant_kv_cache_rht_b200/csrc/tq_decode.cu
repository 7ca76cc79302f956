// Decode attention: split planning, dispatch, and the split-merge kernel.
#include "tq_decode_impl.cuh"

#include <algorithm>

namespace tq {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kMaxSplits = 512;
// Split target: about four CTAs per SM of a 148-SM B200.  Fixed (not queried)
// so that the workspace size is a pure function of the call's sizes.
constexpr long kTargetCtas = 148L * 4;

// Merges the splits of one (query head, batch row) and applies the inverse
// rotation: o = D1 H (sum_s w_s o_s) / (sum_s w_s l_s) / d with
// w_s = 2^(m_s - max m) ("How to Use TurboQuant ...", "What is TurboQuant?":
// _rht_inverse; the 1/d collects the rotation's and the dequantization's
// 1/sqrt(d)).  Every partial is loaded at once (warp w takes splits w, w+8,
// ..., lane l channels l*d/32 ..), so the merge costs one memory round trip;
// all reductions run in a fixed order.
template <int D>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __grid_constant__ Tables tb, const int32_t* __restrict__ seq_lens,
                   int32_t* status, const float* __restrict__ ws, int q_heads, int splits,
                   int chunk, int capacity, float* __restrict__ out) {
  constexpr int E = D / 32;
  constexpr int W = kCombineThreads / 32;
  constexpr int PER = 8;  // splits per warp per round, loaded together
  __shared__ float wgt[kMaxSplits];
  __shared__ __align__(16) float part[W][D];
  __shared__ float red[2][W];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  const long row = (long)b * q_heads + h;
  const float* po = ws + row * splits * D;
  const float* pml = ws + (long)gridDim.y * q_heads * splits * D + row * splits * 2;
  // issue the loads of the first round before anything depends on them
  float4 ov[PER][E / 4];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int s = warp + W * i;
    if (s < splits) {
#pragma unroll
      for (int v = 0; v < E / 4; ++v)
        ov[i][v] = reinterpret_cast<const float4*>(po + (long)s * D + lane * E)[v];
    }
  }
  float ms[kMaxSplits / kCombineThreads], ls[kMaxSplits / kCombineThreads];
#pragma unroll
  for (int i = 0; i < kMaxSplits / kCombineThreads; ++i) {
    const int s = tid + kCombineThreads * i;
    ms[i] = s < splits ? pml[2 * s] : -INFINITY;
    ls[i] = s < splits ? pml[2 * s + 1] : 0.f;
  }
  const int T = min(max(seq_lens[b], 0), capacity);
  if (tid == 0 && h == 0 && T > (long)splits * chunk) atomicOr(status, (int)kFlagMaxCtx);
  const int S = min(splits, (T + chunk - 1) / chunk);
  float* dst = out + row * D;
  if (S <= 0) {
    for (int i = tid; i < D; i += kCombineThreads) dst[i] = 0.f;
    pdl_trigger();
    return;
  }
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxSplits / kCombineThreads; ++i)
    if (tid + kCombineThreads * i < S) m = fmaxf(m, ms[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[0][warp] = m;
  __syncthreads();
  m = red[0][0];
#pragma unroll
  for (int w = 1; w < W; ++w) m = fmaxf(m, red[0][w]);
  float l = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxSplits / kCombineThreads; ++i) {
    const int s = tid + kCombineThreads * i;
    if (s < S) {
      const float w = exp2f(ms[i] - m);
      wgt[s] = w;
      l = fmaf(ls[i], w, l);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[1][warp] = l;
  __syncthreads();
  l = red[1][0];
#pragma unroll
  for (int w = 1; w < W; ++w) l += red[1][w];
  float a[E];
#pragma unroll
  for (int e = 0; e < E; ++e) a[e] = 0.f;
  for (int s0 = 0; s0 < S; s0 += W * PER) {
    if (s0 > 0) {
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int s = s0 + warp + W * i;
        if (s < S) {
#pragma unroll
          for (int v = 0; v < E / 4; ++v)
            ov[i][v] = reinterpret_cast<const float4*>(po + (long)s * D + lane * E)[v];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int s = s0 + warp + W * i;
      if (s < S) {
        const float w = wgt[s];
#pragma unroll
        for (int v = 0; v < E / 4; ++v) {
          a[4 * v] = fmaf(ov[i][v].x, w, a[4 * v]);
          a[4 * v + 1] = fmaf(ov[i][v].y, w, a[4 * v + 1]);
          a[4 * v + 2] = fmaf(ov[i][v].z, w, a[4 * v + 2]);
          a[4 * v + 3] = fmaf(ov[i][v].w, w, a[4 * v + 3]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) part[warp][lane * E + e] = a[e];
  __syncthreads();
  if (warp == 0) {
    const float inv = 1.0f / (l * (float)D);
    float u[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int ch = lane * E + e;
      float v = part[0][ch];
#pragma unroll
      for (int w = 1; w < W; ++w) v += part[w][ch];
      u[e] = v;
    }
    warp_fwht<E>(u, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int ch = lane * E + e;
      const float v = u[e] * inv;
      dst[ch] = ((tb.s1[ch >> 5] >> (ch & 31)) & 1u) ? -v : v;
    }
  }
  pdl_trigger();
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q_heads, cv.batch);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (tb.d == 128)
    e = cudaLaunchKernelEx(&cfg, combine_kernel<128>, tb, cv.seq_lens, cv.status,
                           (const float*)workspace, q_heads, plan.splits, plan.chunk, cv.capacity, out);
  else
    e = cudaLaunchKernelEx(&cfg, combine_kernel<256>, tb, cv.seq_lens, cv.status,
                           (const float*)workspace, q_heads, plan.splits, plan.chunk, cv.capacity, out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tq
