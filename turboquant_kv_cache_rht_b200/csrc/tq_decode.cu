// Decode attention: split planning, dispatch, and the split-merge kernel.
#include "tq_decode_impl.cuh"

#include <algorithm>
#include <type_traits>

namespace tq {

namespace {

// A lane's E = d/32 consecutive floats of a partial (16- or 8-byte loads).
template <int E>
__device__ __forceinline__ void load_lane(const float* p, float (&v)[E]) {
  if constexpr (E % 4 == 0) {
#pragma unroll
    for (int i = 0; i < E / 4; ++i) {
      const float4 x = reinterpret_cast<const float4*>(p)[i];
      v[4 * i] = x.x;
      v[4 * i + 1] = x.y;
      v[4 * i + 2] = x.z;
      v[4 * i + 3] = x.w;
    }
  } else {
    static_assert(E == 2, "d of 64, 128 or 256");
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x;
    v[1] = x.y;
  }
}

constexpr int kCombineThreads = 256;
constexpr int kMaxParts = 1024;  // partials one unit can have (at most one per CTA)
static_assert(kMaxTargetCtas <= kMaxParts, "a unit's partials must fit the merge");

// Merges the partial results of one (query head, batch row) and applies the
// inverse rotation: o = D1 H (sum_s w_s o_s) / (sum_s w_s l_s) / (d v_lam)
// with w_s = 2^(m_s - max m) ("How to Use TurboQuant ...", "What is
// TurboQuant?": _rht_inverse; the 1/d collects the rotation's and the
// dequantization's 1/sqrt(d), and v_lam is the value table's scale).  The affine codec's values are not rotated: o = sum / l.  The
// partials are those of the CTAs whose tile ranges meet the unit's (the
// partition of DecodePlan, recomputed here from the lengths).
// Every partial is loaded at once (warp w takes partials w, w+8, ..., lane l
// channels l*d/32 ..), so the merge costs one memory round trip; all
// reductions run in a fixed order.
template <int D>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                   const float* __restrict__ ws, int q_heads, int max_ctx, int nctas, int nslots,
                   float* __restrict__ out) {
  constexpr int E = D / 32;
  constexpr int W = kCombineThreads / 32;
  constexpr int PER = 8;  // partials per warp per round, loaded together
  __shared__ float wgt[kMaxParts];
  __shared__ __align__(16) float part[W][D];
  __shared__ float red[2][W];
  __shared__ long long tiles_red[2][W];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = cv.kv_heads, G = q_heads / H, kvh = h / G, hg = h - kvh * G;
  // The partition depends on the lengths alone, which the decode kernel does
  // not write and which were complete before it let this grid launch: it is
  // worked out before the wait, overlapping the decode's tail.
  // tiles per KV head of the rows before b, and of all rows
  long long before = 0, all = 0;
  for (int r = tid; r < cv.batch; r += kCombineThreads) {
    const long long x = row_tiles(cv, r, max_ctx);
    all += x;
    before += r < b ? x : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    all += __shfl_xor_sync(0xffffffffu, all, o);
    before += __shfl_xor_sync(0xffffffffu, before, o);
  }
  if (lane == 0) {
    tiles_red[0][warp] = all;
    tiles_red[1][warp] = before;
  }
  __syncthreads();
  all = before = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    all += tiles_red[0][w];
    before += tiles_red[1][w];
  }
  const int stored = min(max(cv.seq_lens[b], 0), cv.capacity);
  const int n = row_tiles(cv, b, max_ctx);
  float* dst = out + ((long)b * q_heads + h) * D;
  // the CTAs c_lo .. c_hi whose ranges [c*T/nctas, (c+1)*T/nctas) meet [su, eu)
  const long long T = all * H, su = before * H + (long long)kvh * n, eu = su + n;
  const int c_lo = n > 0 ? (int)(((su + 1) * nctas + T - 1) / T - 1) : 0;
  const int c_hi = n > 0 ? (int)((eu * nctas + T - 1) / T - 1) : -1;
  const int S = c_hi - c_lo + 1;
  pdl_wait();
  if (tid == 0 && h == 0 && stored > max_ctx) atomicOr(cv.status, (int)kFlagMaxCtx);
  if (n == 0) {
    for (int i = tid; i < D; i += kCombineThreads) dst[i] = 0.f;
    pdl_trigger();
    return;
  }

  const long first = (long)c_lo + (long)b * H + kvh;  // slot of partial 0
  const float* po = ws + (first * G + hg) * D;              // partial s at po + s * G * D
  const float* pml = ws + (long)nslots * G * D + (first * G + hg) * 2;  // at pml + s * G * 2
  // issue the loads of the first round before anything depends on them
  float ov[PER][E];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int s = warp + W * i;
    if (s < S) load_lane<E>(po + (long)s * G * D + lane * E, ov[i]);
  }
  float ms[kMaxParts / kCombineThreads], ls[kMaxParts / kCombineThreads];
#pragma unroll
  for (int i = 0; i < kMaxParts / kCombineThreads; ++i) {
    const int s = tid + kCombineThreads * i;
    bool valid = false;
    if (s < S) {  // a CTA with an empty range (T < nctas) left no partial
      const long long c = c_lo + s, f0 = tile_bound(c, T, nctas), f1 = tile_bound(c + 1, T, nctas);
      valid = max(f0, su) < min(f1, eu);
    }
    ms[i] = valid ? pml[(long)s * G * 2] : -INFINITY;
    ls[i] = valid ? pml[(long)s * G * 2 + 1] : 0.f;
  }
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxParts / kCombineThreads; ++i) m = fmaxf(m, ms[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[0][warp] = m;
  __syncthreads();
  m = red[0][0];
#pragma unroll
  for (int w = 1; w < W; ++w) m = fmaxf(m, red[0][w]);
  float l = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxParts / kCombineThreads; ++i) {
    const int s = tid + kCombineThreads * i;
    if (s < S) {
      const float w = ms[i] == -INFINITY ? 0.f : exp2f(ms[i] - m);
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
        if (s < S) load_lane<E>(po + (long)s * G * D + lane * E, ov[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int s = s0 + warp + W * i;
      if (s < S) {
        const float w = wgt[s];
        if (w > 0.f) {  // skips the slots no CTA wrote
#pragma unroll
          for (int e = 0; e < E; ++e) a[e] = fmaf(ov[i][e], w, a[e]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) part[warp][lane * E + e] = a[e];
  __syncthreads();
  if (warp == 0) {
    const float inv = 1.0f / (tb.affine ? l : l * (float)D * tb.v_lam);
    float u[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int ch = lane * E + e;
      float v = part[0][ch];
#pragma unroll
      for (int w = 1; w < W; ++w) v += part[w][ch];
      u[e] = v;
    }
    if (tb.affine) {
#pragma unroll
      for (int e = 0; e < E; ++e) dst[lane * E + e] = u[e] * inv;
    } else {
      warp_fwht<E>(u, lane);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int ch = lane * E + e;
        const float v = u[e] * inv;
        dst[ch] = ((tb.s1[ch >> 5] >> (ch & 31)) & 1u) ? -v : v;
      }
    }
  }
  pdl_trigger();
}

}  // namespace

DecodePlan plan_decode(int batch, int kv_heads, int max_ctx, long target_ctas) {
  const long tiles = std::max<long>(1, (max_ctx + kDecTile - 1) / kDecTile);
  const long units = std::max<long>(1, (long)batch * kv_heads);
  DecodePlan p;
  p.ctas = (int)std::max<long>(1, std::min(target_ctas, units * tiles));
  p.slots = (int)(p.ctas + units - 1);
  return p;
}

size_t decode_workspace_bytes(const DecodePlan& plan, int q_heads, int kv_heads, int head_dim) {
  return (size_t)plan.slots * (q_heads / kv_heads) * (head_dim + 2) * sizeof(float);
}

bool decode_supported(int head_dim, int group, int k_bits, int v_bits, int qjl) {
  (void)qjl;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return false;
  if (group != 1 && group != 2 && group != 4 && group != 8) return false;
  if (k_bits < 2 || k_bits > 4) return false;
  return v_bits == k_bits || v_bits == k_bits + 1;
}

cudaError_t launch_decode(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                          int q_heads, float scale, int max_ctx, float* out, float* workspace,
                          cudaStream_t stream) {
  const float scale_log2 = scale * 1.4426950408889634f;
  const int group = q_heads / cv.kv_heads;
  // one wave of CTAs at the kernel's occupancy (capped at the workspace bound)
  int ctas_per_sm = 0, sms = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (tb.affine)
    e = tb.d == 64    ? decode_occupancy_dim<64, true>(tb, group, &ctas_per_sm)
        : tb.d == 128 ? decode_occupancy_dim<128, true>(tb, group, &ctas_per_sm)
                      : decode_occupancy_dim<256, true>(tb, group, &ctas_per_sm);
  else
    e = tb.d == 64    ? decode_occupancy_dim<64, false>(tb, group, &ctas_per_sm)
        : tb.d == 128 ? decode_occupancy_dim<128, false>(tb, group, &ctas_per_sm)
                      : decode_occupancy_dim<256, false>(tb, group, &ctas_per_sm);
  if (e != cudaSuccess) return e;
  const long target = std::min<long>(kMaxTargetCtas, (long)std::max(ctas_per_sm, 1) * sms);
  const DecodePlan plan = plan_decode(cv.batch, cv.kv_heads, max_ctx, target);
  auto launch = [&](auto dim, auto aff) {
    return launch_decode_dim<decltype(dim)::value, decltype(aff)::value>(
        tb, cv, q, dtype, q_heads, scale_log2, max_ctx, plan, workspace, stream);
  };
  using T = std::true_type;
  using F = std::false_type;
  using D64 = std::integral_constant<int, 64>;
  using D128 = std::integral_constant<int, 128>;
  using D256 = std::integral_constant<int, 256>;
  if (tb.d == 64)
    e = tb.affine ? launch(D64{}, T{}) : launch(D64{}, F{});
  else if (tb.d == 128)
    e = tb.affine ? launch(D128{}, T{}) : launch(D128{}, F{});
  else if (tb.d == 256)
    e = tb.affine ? launch(D256{}, T{}) : launch(D256{}, F{});
  else
    e = cudaErrorNotSupported;
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
  if (tb.d == 64)
    e = cudaLaunchKernelEx(&cfg, combine_kernel<64>, tb, cv, (const float*)workspace, q_heads,
                           max_ctx, plan.ctas, plan.slots, out);
  else if (tb.d == 128)
    e = cudaLaunchKernelEx(&cfg, combine_kernel<128>, tb, cv, (const float*)workspace, q_heads,
                           max_ctx, plan.ctas, plan.slots, out);
  else
    e = cudaLaunchKernelEx(&cfg, combine_kernel<256>, tb, cv, (const float*)workspace, q_heads,
                           max_ctx, plan.ctas, plan.slots, out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tq
