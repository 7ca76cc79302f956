// LUT matmul on packed weight codes (the weights regime: "mlx-turboquant"
// README, introduction, "Weights (MSE regime)": rotate each weight matrix, then
// quantize; "The Metal kernels" item 1: non-uniform LUT dequant + matmul
// directly on packed indices).
//
// Each row of W [rows][k] is cut into k/d blocks of d input channels, and every
// block is encoded as a KV vector is: fp16 norm n and b-bit Lloyd-Max codes of
// its rotated, normalized coordinates.  For an input x,
//   y[n] = sum_j (n_{n,j} / sqrt(d)) <c[codes_{n,j}], R x_j>
//        = sum_j n_{n,j} <c[codes_{n,j}], H (s1 * x_j)> / d,
// the decode's key scoring without the softmax.
//
// Two kernels.  The first rotates every input block once (one warp per block,
// warp shuffles), scales it by a power of two that keeps its fp16 hi / lo
// parts normal, and writes it in the order of the tensor-core B fragments.
// The second takes 128 weight rows and 4, 8 or 16 inputs per CTA; per block it
// stages the rows' codes, their norms and the block's input fragments with
// one 3-stage cp.async pipeline, and each warp scores 2 slabs of 16 rows with
// a pair table as the decode's keys use (two codes -> an fp16 pair of
// lambda-scaled centroids, 32 copies), one MMA per 16 rows and k-block.  When rows x inputs give too few
// CTAs, the blocks are split across CTAs and the partial sums are merged in a
// fixed order.
#include "tq_decode_impl.cuh"

#include <algorithm>

namespace tq {
namespace {

constexpr int kMmThreads = 128;   // 4 warps
constexpr int kMmSlabs = 2;       // 16-row slabs per warp
constexpr int kMmRows = 4 * kMmSlabs * 16;  // weight rows per CTA
// pipeline stages: 3, or 2 with 16 inputs per CTA (their fragments double the
// stage; two stages keep three CTAs per SM)
template <int NT>
constexpr int mm_stages() { return NT == 4 ? 2 : 3; }
constexpr long kMmMaxCtas = kLutMatmulMaxCtas;  // bounds every plan (and so the workspace)

// fragments of one (block, column group): [nt][kb][lane] x 2 words
template <int D, int NT>
constexpr int frag_words() { return NT * (D / 16) * 32 * 2; }

template <int D, int KB, int NT>
struct MmGeom {
  static constexpr int KBLK = D / 16;
  static constexpr int kRowB = KB * D / 8;
  static constexpr int KS = k_stride_words(D, KB);
  static constexpr int CBK = (kRowB % 16 == 0) ? 16 : 8;
  static constexpr int QB = KB * D / 4;
  static constexpr int KW = (QB + 31) / 32;
  static constexpr int KNW = (QB % 32 == 0) ? QB / 32 : (QB + 16 + 31) / 32;
  static constexpr int LK = 1 << (2 * KB);
  static constexpr int RKL = 5;        // 32 copies: a warp's lookups never share a bank
  // 4-bit codes at head_dim <= 128, up to 4 inputs (BP): a pair is a whole byte, so with the
  // table's entries 256 bytes apart one byte permute forms the index (the code
  // byte above the lane's copy offset).  The other 128 bytes of every entry
  // form a logical space -- logical x at byte 128 + x + (x & ~127), which keeps
  // the bank of a plain layout -- holding the stages' code rows (64 or 32
  // bytes, so no row straddles two blocks); the rest of a stage follows the
  // 64 KB table region.  Otherwise entries are 128 bytes apart after the stages.
  // (measured: one input 31.3 -> 30.2 us; with 8 or 16 inputs the larger
  // stages cost a CTA per SM or more than the indices save, so not there)
  static constexpr bool BP = KB == 4 && D <= 128 && NT == 1;
  static constexpr int KSH = BP ? 8 : 2 + RKL;
  static constexpr int FW = frag_words<D, NT>();
  static constexpr int codeBytes = kMmRows * KS * 4;  // code rows of one stage
  // one stage: codes [kMmRows][KS] (BP: in the logical space), norms
  // [kMmRows], fragments [FW], scales [4 NT]
  static constexpr int offN = BP ? 0 : codeBytes;
  static constexpr int offF = offN + kMmRows * 2;
  static constexpr int offS = offF + FW * 4;
  static constexpr int stageA = (offS + 16 * NT + 127) / 128 * 128;
  static constexpr int STG = mm_stages<NT>();
  static constexpr int offLK = BP ? 0 : STG * stageA;
  static constexpr int pBase = BP ? (LK << KSH) : 0;  // stage parts outside the logical space
  static constexpr int total = BP ? pBase + STG * stageA : offLK + (LK << KSH);
  // byte of offset x into stage s's code rows
  __host__ __device__ static constexpr int code_off(int s, int x) {
    return BP ? 128 + (s * codeBytes + x) + ((s * codeBytes + x) & ~127) : s * stageA + x;
  }
  static_assert(!BP || ((KS * 4) % 32 == 0 && 128 % (KS * 4) == 0 && STG * codeBytes <= 32768 &&
                        codeBytes % 128 == 0),
                "code rows inside the logical space");
};

// Input rotation: one warp per (input, block).  frag[(j * groups + cg) * FW ..]
// holds, for lane l = 4 g + qd and k-block kb, the two B-fragment words of
// column g of n-tile nt: input cg * 4 NT + 4 nt + (g >> 1), part g & 1 (fp16
// hi or lo) of channels qd * d/4 + 4 kb + (0,1) and (2,3), scaled by 2^e;
// scale[(j * groups + cg) * 4 NT + input] = 1 / (d * 2^e).
template <int D, int NT>
__global__ void __launch_bounds__(128)
    lut_rotate_inputs_kernel(const __grid_constant__ Tables tb, const void* __restrict__ x, int x_dtype,
                             int m, int nblocks, int groups, uint32_t* __restrict__ frag,
                             float* __restrict__ scale) {
  constexpr int E = D / 32, KBLK = D / 16, CPG = 4 * NT;  // inputs per column group
  __shared__ __align__(16) float xs[4][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long pair = (long)blockIdx.x * 4 + warp;  // (block j, input i), i fastest
  const long total = (long)nblocks * groups * CPG;
  pdl_wait();
  if (pair < total) {
    const int i = (int)(pair % (groups * CPG)), j = (int)(pair / (groups * CPG));
    const long k = (long)nblocks * D;
    float u[E], amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int ch = lane * E + e;
      const float v = i < m ? load_any(x, (long)i * k + (long)j * D + ch, x_dtype) : 0.f;
      u[e] = ((tb.s1[ch >> 5] >> (ch & 31)) & 1u) ? -v : v;
    }
    warp_fwht<E>(u, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(u[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int ex = 0;
    frexpf(amax > 0.f ? amax : 1.f, &ex);
    const float sc = ldexpf(1.f, 8 - ex);
#pragma unroll
    for (int e = 0; e < E; ++e) xs[warp][lane * E + e] = u[e] * sc;
    __syncwarp();
    const int cg = i / CPG, ii = i % CPG, nt = ii / 4, in4 = ii % 4;
    uint32_t* f = frag + ((long)j * groups + cg) * frag_words<D, NT>();
    // lanes of this input's two columns: g = 2 in4 + part, qd = 0..3 -> 8 lanes x KBLK
    for (int t = lane; t < 8 * KBLK; t += 32) {
      const int part = t & 1, qd = (t >> 1) & 3, kb = t >> 3, g = 2 * in4 + part;
      const float* r = xs[warp] + qd * (D / 4) + 4 * kb;
      uint32_t h01, l01, h23, l23;
      split_pair(r[0], r[1], h01, l01);
      split_pair(r[2], r[3], h23, l23);
      uint32_t* dst = f + ((nt * KBLK + kb) * 32 + 4 * g + qd) * 2;
      dst[0] = part ? l01 : h01;
      dst[1] = part ? l23 : h23;
    }
    if (lane == 0) scale[((long)j * groups + cg) * CPG + ii] = 1.f / ((float)D * sc);
  }
  pdl_trigger();
}

template <int D, int KB, int NT>
__global__ void __launch_bounds__(kMmThreads)
    lut_matmul_kernel(const __grid_constant__ Tables tb, const uint8_t* __restrict__ codes,
                      const uint16_t* __restrict__ norms, int rows, int nblocks,
                      int blocks_per_split, int groups, const uint32_t* __restrict__ frag,
                      const float* __restrict__ scale, int m, float* __restrict__ out) {
  using Geo = MmGeom<D, KB, NT>;
  constexpr int CPG = 4 * NT;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, qd = lane & 3;
  const int row0 = blockIdx.x * kMmRows, cg = blockIdx.y, split = blockIdx.z;
  const int j0 = split * blocks_per_split, j1 = min(nblocks, j0 + blocks_per_split);

  // pair table of fp16(k_lam * c) (k_lam divided out with the scales); it
  // depends on the kernel parameters only, so it is built before the wait
  {
    constexpr int RK = 1 << Geo::RKL;
    for (int p = tid; p < Geo::LK; p += kMmThreads) {
      const uint32_t v = pack_half2(__float2half_rn(tb.k_cent[p & ((1 << KB) - 1)] * tb.k_lam),
                                    __float2half_rn(tb.k_cent[p >> KB] * tb.k_lam));
      uint4* dst = reinterpret_cast<uint4*>(smem + Geo::offLK + (p << Geo::KSH));
#pragma unroll
      for (int c = 0; c < RK / 4; ++c) dst[c] = make_uint4(v, v, v, v);
    }
  }
  pdl_wait();

  const int valid_rows = min(kMmRows, rows - row0);  // a multiple of 16
  constexpr int CK = Geo::kRowB / Geo::CBK;
  constexpr int NK = (kMmRows * CK + kMmThreads - 1) / kMmThreads;
  constexpr int NF = Geo::FW / 4;  // 16-byte chunks of the fragments
  auto issue_block = [&](int stage, int j) {
    uint8_t* st = smem + Geo::pBase + stage * Geo::stageA;
    const uint8_t* src = codes + ((size_t)j * rows + row0) * Geo::kRowB;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const int c = tid + kMmThreads * i, r = c / CK, col = c - r * CK;
      if (c < kMmRows * CK && r < valid_rows)
        cp_async_chunk<Geo::CBK>(smem + Geo::code_off(stage, r * Geo::KS * 4 + col * Geo::CBK),
                                 src + r * Geo::kRowB + col * Geo::CBK);
    }
    for (int c = tid; c < valid_rows / 8; c += kMmThreads)  // norms: 16 bytes per 8 rows
      cp_async16(st + Geo::offN + c * 16,
                 reinterpret_cast<const uint8_t*>(norms + (size_t)j * rows + row0) + c * 16);
    const uint32_t* fsrc = frag + ((size_t)j * groups + cg) * Geo::FW;
    for (int c = tid; c < NF; c += kMmThreads) cp_async16(st + Geo::offF + c * 16, fsrc + 4 * c);
    if (tid < NT) cp_async16(st + Geo::offS + tid * 16, scale + ((size_t)j * groups + cg) * CPG + 4 * tid);
  };

  const int nb = max(0, j1 - j0);
  constexpr int STG = Geo::STG;
  if (nb > 0) issue_block(0, j0);  // the first STG - 1 blocks, one commit group each
  cp_async_commit();
  if constexpr (STG == 3) {
    if (nb > 1) issue_block(1, j0 + 1);
    cp_async_commit();
  }

  const uint8_t* lutK = smem + Geo::offLK;
  const uint32_t k_lane = (uint32_t)lane << 2;
  const float inv_lam = 1.0f / tb.k_lam;
  float y[kMmSlabs][NT][2];  // rows (slab, g) and (slab, g + 8), input cg*CPG + 4 nt + qd
#pragma unroll
  for (int s = 0; s < kMmSlabs; ++s)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) y[s][nt][0] = y[s][nt][1] = 0.f;

  for (int it = 0; it < nb; ++it) {
    cp_async_wait<STG - 2>();  // block it has landed
    __syncthreads();           // and the stage refilled next is no longer read
    if (it + STG - 1 < nb) issue_block((it + STG - 1) % STG, j0 + it + STG - 1);
    cp_async_commit();
    const int sidx = it % STG;
    const uint8_t* st = smem + Geo::pBase + sidx * Geo::stageA;  // norms, fragments, scales

    uint32_t bk[NT][Geo::KBLK][2];
    float post[NT];
    {
      const uint2* f = reinterpret_cast<const uint2*>(st + Geo::offF);
      const float* sc = reinterpret_cast<const float*>(st + Geo::offS);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int kb = 0; kb < Geo::KBLK; ++kb) {
          const uint2 v = f[(nt * Geo::KBLK + kb) * 32 + lane];
          bk[nt][kb][0] = v.x;
          bk[nt][kb][1] = v.y;
        }
        post[nt] = sc[4 * nt + qd] * inv_lam;
      }
    }
#pragma unroll
    for (int s = 0; s < kMmSlabs; ++s) {
      const int r0 = 16 * (warp * kMmSlabs + s);
      if (r0 >= valid_rows) break;
      // MMA rows g and g + 8 are weight rows r0 + g and r0 + g + 8; columns
      // are (input, part): input qd's fp16 hi and lo parts at 2 qd, 2 qd + 1
      float sacc[2][NT][4];
#pragma unroll
      for (int par = 0; par < 2; ++par)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[par][nt][e] = 0.f;
      uint32_t kw0[Geo::KW], kw1[Geo::KW];
      // rows r0 + g and r0 + g + 8 (BP: 8 rows are whole 128-byte blocks apart)
      const uint32_t* k0 = reinterpret_cast<const uint32_t*>(smem + Geo::code_off(sidx, (r0 + g) * Geo::KS * 4));
      const uint32_t* k1 = Geo::BP ? k0 + 2 * 8 * Geo::KS : k0 + 8 * Geo::KS;
      static_assert(!Geo::BP || (8 * Geo::KS * 4) % 128 == 0, "rows g and g + 8 whole blocks apart");
      load_value_chunk<Geo::QB, Geo::KW, Geo::KNW>(k0, qd, kw0);
      load_value_chunk<Geo::QB, Geo::KW, Geo::KNW>(k1, qd, kw1);
#pragma unroll
      for (int kb = 0; kb < Geo::KBLK; ++kb) {
        const int o1 = KB * 4 * kb, o2 = o1 + 2 * KB;
        uint32_t i0, i1, i2, i3;
        if constexpr (Geo::BP) {  // whole code bytes
          i0 = quad_index<true, 8>(kw0[o1 >> 5], (o1 & 31) >> 3, k_lane);
          i1 = quad_index<true, 8>(kw1[o1 >> 5], (o1 & 31) >> 3, k_lane);
          i2 = quad_index<true, 8>(kw0[o2 >> 5], (o2 & 31) >> 3, k_lane);
          i3 = quad_index<true, 8>(kw1[o2 >> 5], (o2 & 31) >> 3, k_lane);
        } else {
          i0 = field_scaled(kw0, Geo::KW, o1, 2 * KB, Geo::KSH) | k_lane;
          i1 = field_scaled(kw1, Geo::KW, o1, 2 * KB, Geo::KSH) | k_lane;
          i2 = field_scaled(kw0, Geo::KW, o2, 2 * KB, Geo::KSH) | k_lane;
          i3 = field_scaled(kw1, Geo::KW, o2, 2 * KB, Geo::KSH) | k_lane;
        }
        const uint32_t a0 = *reinterpret_cast<const uint32_t*>(lutK + i0);
        const uint32_t a1 = *reinterpret_cast<const uint32_t*>(lutK + i1);
        const uint32_t a2 = *reinterpret_cast<const uint32_t*>(lutK + i2);
        const uint32_t a3 = *reinterpret_cast<const uint32_t*>(lutK + i3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma16816(sacc[kb & 1][nt], a0, a1, a2, a3, bk[nt][kb][0], bk[nt][kb][1]);
      }
      const uint16_t* nr = reinterpret_cast<const uint16_t*>(st + Geo::offN) + r0;
      const float n0 = __half2float(__ushort_as_half(nr[g]));
      const float n1 = __half2float(__ushort_as_half(nr[g + 8]));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        y[s][nt][0] = fmaf((sacc[0][nt][0] + sacc[1][nt][0]) + (sacc[0][nt][1] + sacc[1][nt][1]),
                           n0 * post[nt], y[s][nt][0]);
        y[s][nt][1] = fmaf((sacc[0][nt][2] + sacc[1][nt][2]) + (sacc[0][nt][3] + sacc[1][nt][3]),
                           n1 * post[nt], y[s][nt][1]);
      }
    }
  }
  // out: y [m][rows] (one split) or the partials [splits][m][rows]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int col = cg * CPG + 4 * nt + qd;
    if (col >= m) continue;
#pragma unroll
    for (int s = 0; s < kMmSlabs; ++s) {
      const int r0 = 16 * (warp * kMmSlabs + s);
      if (r0 >= valid_rows) break;
      float* o = out + ((size_t)split * m + col) * rows + row0 + r0;
      o[g] = y[s][nt][0];
      o[g + 8] = y[s][nt][1];
    }
  }
  pdl_trigger();
}

// y[i] = sum over splits s (ascending) of partials[s][i]
__global__ void __launch_bounds__(256)
    lut_matmul_merge_kernel(const float* __restrict__ partials, int splits, long n, float* __restrict__ y) {
  pdl_wait();
  for (long i = (long)blockIdx.x * 256 + threadIdx.x; i < n; i += (long)gridDim.x * 256) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += partials[(long)s * n + i];
    y[i] = acc;
  }
  pdl_trigger();
}

cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int D, int KB, int NT>
cudaError_t launch_mm_shape(const Tables& tb, const uint8_t* codes, const uint16_t* norms, int rows,
                            int k, const void* x, int dtype, int m, uint32_t* frag, float* scale,
                            float* partials, float* y, cudaStream_t stream) {
  using Geo = MmGeom<D, KB, NT>;
  auto kern = lut_matmul_kernel<D, KB, NT>;
  int ctas_per_sm = 1, sms = 0, dev = 0;
  static KernelConfig config;  // one per shape
  cudaError_t e = configure_kernel(config, kern, Geo::total, kMmThreads, &ctas_per_sm);
  if (e != cudaSuccess) return e;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // one wave at the kernel's occupancy (never more CTAs than the workspace bound)
  const MatmulPlan plan = plan_lut_matmul(rows, k, m, D, std::min<long>(kMmMaxCtas, (long)std::max(ctas_per_sm, 1) * sms));
  float* out = plan.splits > 1 ? partials : y;
  const int nblocks = k / D;
  cudaLaunchAttribute attr[1];
  const long pairs = (long)nblocks * plan.groups * 4 * NT;
  cudaLaunchConfig_t rc = pdl_config(dim3((unsigned)((pairs + 3) / 4)), dim3(128), 0, stream, attr);
  e = cudaLaunchKernelEx(&rc, lut_rotate_inputs_kernel<D, NT>, tb, x, dtype, m, nblocks, plan.groups,
                         frag, scale);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = pdl_config(dim3((rows + kMmRows - 1) / kMmRows, plan.groups, plan.splits),
                                      dim3(kMmThreads), Geo::total, stream, attr);
  e = cudaLaunchKernelEx(&cfg, kern, tb, codes, norms, rows, nblocks, plan.blocks_per_split,
                         plan.groups, (const uint32_t*)frag, (const float*)scale, m, out);
  if (e != cudaSuccess || plan.splits == 1) return e;
  const long n = (long)m * rows;
  cudaLaunchConfig_t mc = pdl_config(dim3((unsigned)std::min<long>((n + 255) / 256, 148L * 8)),
                                     dim3(256), 0, stream, attr);
  return cudaLaunchKernelEx(&mc, lut_matmul_merge_kernel, (const float*)partials, plan.splits, n, y);
}

template <int D, int NT>
cudaError_t launch_mm_bits(const Tables& tb, const uint8_t* codes, const uint16_t* norms, int rows,
                           int k, const void* x, int dtype, int m, uint32_t* frag, float* scale,
                           float* partials, float* y, cudaStream_t stream) {
  switch (tb.k_bits) {
    case 2: return launch_mm_shape<D, 2, NT>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
    case 3: return launch_mm_shape<D, 3, NT>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
    case 4: return launch_mm_shape<D, 4, NT>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
  }
  return cudaErrorNotSupported;
}

template <int D>
cudaError_t launch_mm_dim(const Tables& tb, const uint8_t* codes, const uint16_t* norms, int rows,
                          int k, const void* x, int dtype, int m, uint32_t* frag, float* scale,
                          float* partials, float* y, cudaStream_t stream) {
  if (m > 8) return launch_mm_bits<D, 4>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
  if (m > 4) return launch_mm_bits<D, 2>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
  return launch_mm_bits<D, 1>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
}

}  // namespace

MatmulPlan plan_lut_matmul(int rows, int k, int m, int d, long target_ctas) {
  MatmulPlan p;
  p.inputs_per_group = m > 8 ? 16 : m > 4 ? 8 : 4;
  p.groups = (m + p.inputs_per_group - 1) / p.inputs_per_group;
  const long tiles = std::max<long>(1, (long)((rows + kMmRows - 1) / kMmRows) * p.groups);
  const long nblocks = std::max(1, k / d);
  const long s = std::max<long>(1, std::min(nblocks, std::min(target_ctas, kMmMaxCtas) / tiles));
  p.blocks_per_split = (int)((nblocks + s - 1) / s);
  p.splits = (int)((nblocks + p.blocks_per_split - 1) / p.blocks_per_split);
  p.frag_words = (size_t)nblocks * p.groups * (p.inputs_per_group / 4) * (d / 16) * 64;
  p.scale_floats = (size_t)nblocks * p.groups * p.inputs_per_group;
  return p;
}

size_t lut_matmul_workspace_bytes(const MatmulPlan& plan, int rows, int m) {
  const size_t partials = plan.splits > 1 ? (size_t)plan.splits * m * rows : 0;
  return (plan.frag_words + plan.scale_floats + partials) * 4;
}

cudaError_t launch_lut_matmul(const Tables& tb, const uint8_t* codes, const uint16_t* norms, int rows,
                              int k, const void* x, int dtype, int m, float* y, float* workspace,
                              cudaStream_t stream) {
  // the workspace is laid out for the largest plan; a launch's plan never splits more
  const MatmulPlan bound = plan_lut_matmul(rows, k, m, tb.d, kMmMaxCtas);
  uint32_t* frag = reinterpret_cast<uint32_t*>(workspace);   // 16-byte multiples, in order
  float* scale = workspace + bound.frag_words;
  float* partials = scale + bound.scale_floats;
  switch (tb.d) {
    case 64: return launch_mm_dim<64>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
    case 128: return launch_mm_dim<128>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
    case 256: return launch_mm_dim<256>(tb, codes, norms, rows, k, x, dtype, m, frag, scale, partials, y, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace tq
