// Fused decode attention on the packed TurboQuant cache (kernel template).
//
// The grid is one wave of CTAs.  The token tiles of all (batch row, KV head)
// units are laid end to end and every CTA takes an equal share of them, read
// from the lengths on the device, so ragged batches stay balanced; each unit
// a CTA meets (a segment) is processed for all G query heads sharing that KV
// head ("How to Use TurboQuant ...", "What is
// TurboQuant?": fused scoring kernels on packed low-bit data with query heads
// repeated over a shared KV head; "TurboQuant Performance Benefits ...",
// "Custom Metal Kernel Implementation": scoring fused with value aggregation,
// no dequantization pass; "mlx-turboquant" README, "The 1-bit QJL residual":
// the sketch correction).
//
// For a GQA group the score and the aggregation are small dense contractions
// (G rows of queries against a tile of tokens), so both run on the tensor
// cores with mma.sync m16n8k16 (fp16 operands, fp32 accumulation):
//   scores  S[token][col]  = K_hat[token][ch] . Qt[ch][col]
//   output  O^T[ch][col]  += V_hat^T[ch][token] . P^T[token][col]
// where a column is (head, part): the query and the probabilities are split
// into fp16 hi + lo parts, so their products carry about 22 bits.  Key and
// value centroids enter as single fp16 values of lambda * c, with a per-table
// scale lambda in [1, 2) chosen on the host so that these roundings are
// nearly exact (lambda is divided out in fp32).  The packed codes never
// become a dequantized cache: each thread turns its own code bits into MMA
// fragment registers through small tables in shared memory (pairs: two codes
// -> two fp16 values; quads: a byte of four 2-bit codes -> four), replicated
// so that a warp's lookups never share a bank.  Where a table index is a
// whole code byte, the tables' entries are 256 bytes apart and one byte
// permute forms the index (see DecodeGeom).
//
// The MMA reduction order is free, so channels are assigned to fragment
// slots such that every thread reads one contiguous slice of each packed row:
//   keys  : thread quarter q owns channels [q*d/4, (q+1)*d/4) of tokens g, g+8
//   values: thread group g owns channels [g*d/8, (g+1)*d/8) of tokens
//           2q, 2q+1, 2q+8, 2q+9
//   signs : like keys, pairing bits (j, j+16) of a word so one shift places
//           both sign bits of a half2 (+-1.0 needs no table)
// Tiles of 64 tokens (one 16-token slab per warp) are staged by cp.async in a
// 3-stage pipeline.  Each warp aggregates the values of its previous slab at
// the top of its next one (from registers and the value table), so that work
// overlaps the next slab's scoring.  Each warp keeps its own online-softmax
// state; the four warps are merged in a fixed order and each segment's
// partial (max, sum, output) goes to the workspace, where the combine kernel
// merges the partials of every unit and applies the inverse rotation.
//
// AFF instantiates the same kernel for the affine group-64 comparison codec
// ("mlx-turboquant" README, "Quantize the KV cache (long-context inference)",
// "How it plugs in"): the tables hold the integer levels, a thread quarter
// reads 16 channels of every 64-channel group (so each k-block lies in one
// group), MMA rows g and g+8 are two tokens, the score sums
// scale * <levels, q> + bias * sum(q) over the groups, values become
// scale * level + bias by one hfma2 per operand pair, and nothing is rotated
// back (values are stored unrotated).
#pragma once

#include "tq_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

namespace tq {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecTile = 16 * kDecWarps;  // tokens per pipeline stage
constexpr int kDecStages = 3;
constexpr float kLazyLog2 = 8.0f;  // online-softmax slack before a rescale (log2 units)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
// 8-byte form, for rows whose length is not a multiple of 16 bytes (d = 64
// with 3-bit codes); both addresses are 8-byte aligned.
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem) : "memory");
}
template <int CB>
__device__ __forceinline__ void cp_async_chunk(void* smem, const void* gmem) {
  if constexpr (CB == 16) cp_async16(smem, gmem);
  else cp_async8(smem, gmem);
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float load_any(const void* p, long i, int dtype) {
  switch (dtype) {
    case kBF16: return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    case kF16: return __half2float(static_cast<const __half*>(p)[i]);
    default: return static_cast<const float*>(p)[i];
  }
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// (x, part): the fp16 hi part of x, or the fp16 rounding of the remainder.
__device__ __forceinline__ __half split_part(float x, int part) {
  const __half hi = __float2half_rn(x);
  return part ? __float2half_rn(x - __half2float(hi)) : hi;
}

// 2^x with the hardware approximation (relative error ~2^-22); x <= 0 here.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(x) with the hardware approximation (x > 0 here).
__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-window address at which the dynamic shared memory of the decode
// kernel starts: after the 1 KB the hardware reserves per CTA (the kernel
// declares no static shared memory).  The host checks both facts before the
// first launch and the kernel checks the address on entry.
constexpr uint32_t kDynSmemBase = 0x400;

// 32-bit load from a code table at shared-window address OFF + idx: the
// table's address is an immediate of the load, so a lookup costs the index
// arithmetic alone.
template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds_table(uint32_t idx) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(idx), "n"(OFF));
  return v;
}

template <uint32_t OFF>
__device__ __forceinline__ uint2 lds_table64(uint32_t idx) {
  uint2 v;
  asm("ld.shared.v2.b32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(idx), "n"(OFF));
  return v;
}

// (a, b) -> half2 of their fp16 roundings (hi) and of the remainders (lo).
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - f.x, b - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Bits [off, off + width) of a little-endian stream held in registers w[0..n),
// returned shifted left by `scale` (a byte offset into a table of 2^scale-byte
// entries).  All arguments are compile-time constants after unrolling, so the
// branches fold and w[] stays in registers.
__device__ __forceinline__ uint32_t field_scaled(const uint32_t* w, int n, int off, int width,
                                                 int scale) {
  const uint32_t mask = ((1u << width) - 1u) << scale;
  if (off < scale) return (w[0] << (scale - off)) & mask;
  const int o = off - scale, wi = o >> 5, s = o & 31;
  if (s == 0) return w[wi] & mask;
  if (wi + 1 < n) return __funnelshift_r(w[wi], w[wi + 1], s) & mask;
  return (w[wi] >> s) & mask;
}

// s * c + b on a half2 of two tokens' values (one fp16 rounding, as fma).
__device__ __forceinline__ uint32_t hfma2_bits(uint32_t s, uint32_t c, uint32_t b) {
  const __half2 r = __hfma2(*reinterpret_cast<const __half2*>(&s), *reinterpret_cast<const __half2*>(&c),
                            *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// a * b on half2 bit patterns
__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// +-1.0 half2 from the two sign bits at positions 15 and 31 (bit 1 -> +1)
__device__ __forceinline__ uint32_t sign_pair(uint32_t x) { return (x & 0x80008000u) ^ 0xBC00BC00u; }

// Unnormalized Walsh-Hadamard transform of a d-vector spread over a warp
// (lane l holds channels l*E .. l*E+E-1): in-lane butterflies, then shuffles.
template <int E>
__device__ __forceinline__ void warp_fwht(float (&u)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1)
#pragma unroll
    for (int j = 0; j < E; ++j)
      if ((j & h) == 0) {
        const float a = u[j], c = u[j + h];
        u[j] = a + c;
        u[j + h] = a - c;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float p = __shfl_xor_sync(0xffffffffu, u[e], m);
      u[e] = (lane & m) ? p - u[e] : u[e] + p;
    }
}

// Shared-memory row strides (32-bit words) of the staged codes, chosen so the
// fragment loads below are free of bank conflicts (or as close as the access
// pattern allows); multiples of 4 words for 16-byte copies.
constexpr int k_stride_words(int d, int bits) { return (d == 256 && bits == 4) ? 36 : bits * d / 32; }
constexpr int v_stride_words(int d, int bits) {
  return d == 64 ? (bits == 2 ? 4 : 12)
                 : d == 128 ? (bits == 4 ? 20 : 12) : (bits == 2 ? 20 : bits == 3 ? 28 : 36);
}

template <int D, int G, int KB, int VB, bool QJL, bool AFF>
struct DecodeGeom {
  static constexpr int NT = G > 4 ? 2 : 1;    // n-tiles of 8 columns (4 heads x {hi, lo})
  static constexpr int KBLK = D / 16;         // 16-channel k-blocks of the score MMA
  static constexpr int MBLK = D / 16;         // 16-channel m-blocks of the output MMA
  static constexpr int kRowB = KB * D / 8;    // bytes of one packed row in global memory
  static constexpr int vRowB = VB * D / 8;
  static constexpr int sRowB = D / 8;
  // 3-bit keys and 4-bit values at head_dim 128: the PV layout below
  static constexpr bool PV = D == 128 && KB == 3 && VB == 4 && !AFF;
  static constexpr int KS = k_stride_words(D, KB);
  // PV with the QJL sketch: value rows unpadded and swizzled (v_row_off);
  // measured faster than padded rows there, and slower without the sketch
  static constexpr bool VSW = PV && QJL;
  static constexpr int VS = VSW ? VB * D / 32 : v_stride_words(D, VB);
  static constexpr int SS = D / 32;
  static constexpr int QB = KB * D / 4;       // key bits per thread quarter (a slice of the row)
  static constexpr int KW = (QB + 31) / 32;   // words of the slice, aligned to bit 0
  static constexpr int KNW = (QB % 32 == 0) ? QB / 32 : (QB + 16 + 31) / 32;  // words it spans
  static constexpr int SW = D >= 128 ? D / 128 : 1;  // sign words per thread quarter (d = 64: half a word)
  static constexpr int CBK = (kRowB % 16 == 0) ? 16 : 8;  // copy chunk bytes per row
  static constexpr int CBV = (vRowB % 16 == 0) ? 16 : 8;
  static constexpr int VCH = VB * D / 8;      // value bits per thread group
  static constexpr int VCW = (VCH + 31) / 32; // words of the aligned value chunk
  static constexpr int VNW = (VCH % 32 == 0) ? VCH / 32 : (VCH + 16 + 31) / 32;
  // 2-bit codes take quad tables: a byte of four codes -> four fp16 values (8
  // bytes), one 64-bit lookup per two MMA registers; wider codes take pair
  // tables (two codes -> an fp16 pair, 4 bytes).  The affine codec keeps pairs.
  static constexpr bool QK = KB == 2 && !AFF;  // quad key table
  static constexpr bool QV = VB == 2 && !AFF;  // quad value table
  static constexpr int LK = QK ? 256 : 1 << (2 * KB);  // key table entries
  static constexpr int LV = QV ? 256 : 1 << (2 * VB);  // value table entries
  static constexpr int EKL = QK ? 3 : 2;               // log2 bytes of a key entry
  static constexpr int EVL = QV ? 3 : 2;               // log2 bytes of a value entry
  // Each table is replicated so that lanes with different (lane mod copies)
  // never meet in a bank; copy c of entry e sits at byte (e << shift) + c *
  // (entry bytes), with the entry shift KSH / VSH below.
  // 32 copies (a lane's own) keep every lookup free of bank conflicts; the
  // 4-bit tables of head_dim 256 keep 16 to leave room for the stages
  // (64-bit lookups are served per half-warp, so 16 copies already keep the
  // quad tables free of conflicts)
  static constexpr int RKL = QK ? 4 : (KB <= 3 || D <= 128) ? 5 : 4;  // log2 key copies
  static constexpr int RVL = QV ? 4 : (VB <= 3 || D <= 128) ? 5 : 4;  // log2 value copies
  // When both tables are quads, or both are 4-bit pair tables of 32 copies,
  // their 128-byte entries are interleaved, key entry e at byte 256 e and
  // value entry e at 256 e + 128: an index is then the code byte above the
  // lane's copy offset, which one byte permute forms.
  static constexpr bool IQ = (QK && QV) || (KB == 4 && VB == 4 && RKL == 5 && RVL == 5);
  // The 3-bit key / 4-bit value shape at head_dim 128 (PV) does the same for
  // its value pair table (entries 256 bytes apart, 32 copies in the first 128
  // bytes of each).  The other 128 bytes of every entry form a logical space:
  // logical offset x sits at byte 128 + x + (x & ~127).  It holds the key pair
  // table (64 entries of 128 bytes, so key entry e sits at 256 e + 128) and,
  // after it, the stages' key and value rows and the epilogue's merge buffer.
  // The map moves every 128-byte block by a multiple of 128 bytes, so an
  // access keeps the bank it has in a plain layout, and an aligned access of
  // at most 16 bytes never straddles two blocks.
  static constexpr int KSH = (IQ || PV) ? 8 : EKL + RKL;  // byte shift of a key entry index
  static constexpr int VSH = (IQ || PV) ? 8 : EVL + RVL;  // byte shift of a value entry index
  // value quads: y / z bytes per interleaved word (a byte holds two channels)
  static constexpr int BPW = D / 32 < 4 ? D / 32 : 4;
  // affine codec: NG groups of 64 channels, one (scale, bias) word per group
  // and token; thread quarter qd reads channels [64 gg + 16 qd, + 16) of group gg
  static constexpr int NG = D / kAffineGroup;
  static constexpr int MB = AFF ? 4 * NG : 2;  // metadata bytes per token (keys or values)
  static constexpr int QBA = 16 * KB;          // key bits per thread quarter and group
  static constexpr int KWA = (QBA + 31) / 32;
  static constexpr int KNWA = (QBA % 32 == 0) ? QBA / 32 : (QBA + 16 + 31) / 32;
  // one pipeline stage (bytes): the key and value rows (offsets in the
  // logical space when PV), then the sign rows and the norms
  static constexpr int offK = 0;
  static constexpr int offV = offK + kDecTile * KS * 4;
  static constexpr int kvBytes = offV + kDecTile * VS * 4 + (PV ? 0 : 16);
  static constexpr int offS = PV ? 0 : kvBytes;
  static constexpr int offKN = offS + (QJL ? kDecTile * SS * 4 : 0);
  static constexpr int offVN = offKN + kDecTile * MB;
  static constexpr int offRN = offVN + kDecTile * MB;
  static constexpr int stage = offRN + (QJL ? kDecTile * 2 : 0);
  static constexpr int stageA = (stage + 127) / 128 * 128;
  // epilogue merge buffer, reusing the key / value rows of the stages: per
  // warp m[G], l[G], O[G][D]
  static constexpr int mergeBytes = kDecWarps * G * (D + 2) * 4;
  static constexpr int stagesBytes = PV ? kDecStages * stageA
      : (kDecStages * stageA > mergeBytes ? kDecStages * stageA : (mergeBytes + 127) / 128 * 128);
  // PV: the tables fill [0, 64 KB); the rows of stage s start at logical
  // 8192 (s + 1), right after the key table, and the other stage parts after
  // the table region.  Otherwise the stages come first, then the tables.
  static constexpr int kvBase = PV ? 128 + 2 * 8192 : 0;             // byte of stage 0's rows
  static constexpr int kvStride = PV ? 2 * kvBytes : stageA;        // bytes from one stage's rows to the next
  static constexpr int pBase = PV ? 65536 : 0;                      // byte of stage 0's other parts
  static constexpr int offLK = PV ? 128 : stagesBytes;
  static constexpr int offLV = PV ? 0 : IQ ? offLK + 128 : offLK + (LK << KSH);
  static constexpr int offQ = PV ? pBase + stagesBytes                  // float [G][D] rotated query
                           : IQ ? offLK + (LK << 8) : offLV + (LV << VSH);
  // byte of logical offset x (relative to kvBase), and the shift of an
  // offset by a multiple of 128 bytes
  __host__ __device__ static constexpr int kvmap(int x) { return PV ? x + (x & ~127) : x; }
  __host__ __device__ static constexpr int kvshift(int b) { return PV ? 2 * b : b; }
  // Logical offset of byte 4 w of staged value row r.  Swizzled rows (VSW,
  // 64 bytes): rows r and r ^ 2 share a 128-byte block (halves (r >> 1) & 1)
  // and the 16 words of rows with (r >> 2) & 1 set are rotated by 8, so that
  // rows 2q + c (q = 0..3) of any group of 8 occupy the four (half, rotation)
  // pairs: a 64-bit read of words 2g, 2g + 1 by lanes (g, q) is free of bank
  // conflicts.  Otherwise rows are VS words apart.
  __host__ __device__ static constexpr int v_row_off(int r, int w) {
    return VSW ? offV + (((r >> 3) << 2) | (((r >> 2) & 1) << 1) | (r & 1)) * 128 + ((r >> 1) & 1) * 64 +
                     ((w + 8 * ((r >> 2) & 1)) & 15) * 4
               : offV + r * VS * 4 + w * 4;
  }
  static constexpr int offQ2 = offQ + G * D * 4;               // float [G][D] QJL query
  static constexpr int offUs = offQ2 + (QJL ? G * D * 4 : 0);  // float [G][NG] group sums (affine)
  static constexpr int offRed = offUs + (AFF ? (G * NG * 4 + 15) / 16 * 16 : 0);  // float scratch
  // prologue: per-warp query maxima [2 * warps]; epilogue: merge weights
  // [warps][G] then the group maxima [G]
  static constexpr int redFloats = (2 * kDecWarps > (kDecWarps + 1) * G ? 2 * kDecWarps : (kDecWarps + 1) * G) + 16;
  // work schedule: scan scratch (one 64-bit word per warp), then one chunk of
  // rows (index, 64-bit tile prefix)
  static constexpr int offSched = (offRed + redFloats * 4 + 15) / 16 * 16;
  static constexpr int schedBytes = kDecWarps * 8 + kDecThreads * 4 + kDecThreads * 8;
  static constexpr int total = offSched + schedBytes;
  static_assert((KS * 4) % CBK == 0 && (VS * 4) % CBV == 0, "rows aligned to the copy chunk");
  static_assert(VCW <= 4 && VNW <= 4, "value chunk too wide");
  static_assert(!PV || (kvBytes % 128 == 0 && offV % 128 == 0 && VS == (VSW ? 16 : 20) && LK == 64 && LV == 256 &&
                        RVL == 5 && VCH == 64 && QB == 96 && KW == 3 && kDecTile % 8 == 0 &&
                        8192 + kDecStages * kvBytes <= 32768 && mergeBytes <= kDecStages * kvBytes &&
                        (16 * KS * 4) % 128 == 0 && (8 * KS * 4) % 128 == 0),
                "PV layout");
};

// Loads the value chunk of thread group g (bits [g*VCH, (g+1)*VCH)) of one
// staged row into out[0..VCW), aligned to bit 0.
template <int VCH, int VCW, int VNW>
__device__ __forceinline__ void load_value_chunk(const uint32_t* row, int g, uint32_t (&out)[VCW]) {
  const int bit = g * VCH, w0 = bit >> 5, sh = bit & 31;
  uint32_t raw[VNW + 1];
#pragma unroll
  for (int i = 0; i < VNW; ++i) raw[i] = row[w0 + i];
  raw[VNW] = 0u;
  if constexpr (VCH % 32 == 0) {
#pragma unroll
    for (int i = 0; i < VCW; ++i) out[i] = raw[i];
  } else {
#pragma unroll
    for (int i = 0; i < VCW; ++i) out[i] = __funnelshift_r(raw[i], raw[i + 1], sh);
  }
}

// x's bits [pos, pos + width), shifted to bit `scale` (either direction).
__device__ __forceinline__ uint32_t bits_at(uint32_t x, int pos, int width, int scale) {
  const uint32_t mask = ((1u << width) - 1u) << scale;
  return pos >= scale ? (x >> (pos - scale)) & mask : (x << (scale - pos)) & mask;
}

// Index of the table entry named by byte `by` of x (a quad, or a pair of 4-bit
// codes) for a lane whose copy offset is lane_off (< 256): with an entry shift
// of 8 the byte permute places the code byte above the offset in one
// instruction.
template <bool IQ, int SH>
__device__ __forceinline__ uint32_t quad_index(uint32_t x, int by, uint32_t lane_off) {
  if constexpr (IQ) {
    return __byte_perm(x, lane_off, 0x5504u | ((uint32_t)by << 4));
  } else {
    return bits_at(x, 8 * by, 8, SH) | lane_off;
  }
}

// Interleaves the value chunks of two tokens a, b so that each 2*VB-bit field
// holds (code_a | code_b << VB) of one channel: y for even channels, z for odd
// ones (VB = 2 and 4; 3-bit codes are paired field by field instead).
template <int VB, int VCW>
__device__ __forceinline__ void interleave_pairs(const uint32_t (&a)[VCW], const uint32_t (&b)[VCW],
                                                 uint32_t (&y)[VCW], uint32_t (&z)[VCW]) {
#pragma unroll
  for (int w = 0; w < VCW; ++w) {
    if constexpr (VB == 4) {
      y[w] = (a[w] & 0x0F0F0F0Fu) | ((b[w] & 0x0F0F0F0Fu) << 4);
      z[w] = ((a[w] >> 4) & 0x0F0F0F0Fu) | (b[w] & 0xF0F0F0F0u);
    } else if constexpr (VB == 2) {
      y[w] = (a[w] & 0x33333333u) | ((b[w] & 0x33333333u) << 2);
      z[w] = ((a[w] >> 2) & 0x33333333u) | (b[w] & 0xCCCCCCCCu);
    } else {
      y[w] = a[w];
      z[w] = b[w];
    }
  }
}

// Channel, within a thread group's D/8 value channels, of MMA row g (h = 0) or
// g + 8 (h = 1) of m-block mb: consecutive channels 2mb, 2mb + 1 with pair
// tables; with quad tables m-block mb reads byte `by` of the even (y) or odd
// (z) interleaved word w, whose two codes are channels c and c + 2.
template <bool QV, int BPW>
__host__ __device__ constexpr int value_channel(int mb, int h) {
  if (!QV) return 2 * mb + h;
  const int w = mb / (2 * BPW), r = mb % (2 * BPW);
  return 16 * w + 4 * (r % BPW) + 2 * h + (r < BPW ? 0 : 1);
}

// Byte offsets, into this lane's copy of the value pair table, of the pairs
// (token a, token b) for channels 2mb (even) and 2mb + 1 (odd) of the chunk.
template <int VB, int VCW, int VSH>
__device__ __forceinline__ void value_pairs(const uint32_t (&y)[VCW], const uint32_t (&z)[VCW], int mb,
                                            uint32_t lane_off, uint32_t& even, uint32_t& odd) {
  if constexpr (VB == 4) {
    const int w = mb >> 2, k = mb & 3;
    if constexpr (VSH == 8) {  // the byte above the lane's copy offset
      even = __byte_perm(y[w], lane_off, 0x5504u | ((uint32_t)k << 4));
      odd = __byte_perm(z[w], lane_off, 0x5504u | ((uint32_t)k << 4));
    } else {
      even = bits_at(y[w], 8 * k, 8, VSH) | lane_off;
      odd = bits_at(z[w], 8 * k, 8, VSH) | lane_off;
    }
  } else if constexpr (VB == 2) {
    const int w = mb >> 3, k = mb & 7;
    even = bits_at(y[w], 4 * k, 4, VSH) | lane_off;
    odd = bits_at(z[w], 4 * k, 4, VSH) | lane_off;
  } else {
    const int o0 = VB * 2 * mb, o1 = o0 + VB;
    even = field_scaled(y, VCW, o0, VB, VSH) | field_scaled(z, VCW, o0, VB, VSH + VB) | lane_off;
    odd = field_scaled(y, VCW, o1, VB, VSH) | field_scaled(z, VCW, o1, VB, VSH + VB) | lane_off;
  }
}

// Tokens of row b a decode call attends: seq_lens[b] clamped to the row's
// capacity and to the call's max_ctx.
__device__ __forceinline__ int row_len(const CacheView& cv, int b, int max_ctx) {
  return min(min(max(cv.seq_lens[b], 0), cv.capacity), max_ctx);
}
__device__ __forceinline__ int row_tiles(const CacheView& cv, int b, int max_ctx) {
  return (row_len(cv, b, max_ctx) + kDecTile - 1) / kDecTile;
}

// floor(c * T / n), the first tile of CTA c of n over T tiles (32-bit
// division when the product fits, as it does for all but huge contexts).
__device__ __forceinline__ long long tile_bound(long long c, long long T, int n) {
  const long long num = c * T;
  return num < (1ll << 32) ? (long long)((unsigned)num / (unsigned)n) : num / n;
}

// Block-wide exclusive prefix sum of one value per thread (NT threads, all of
// them calling); *total receives the block's sum.  `scratch` holds NT/32
// words of shared memory and is free again when the call returns.
template <int NT>
__device__ __forceinline__ long long block_exclusive_scan(long long x, long long* scratch,
                                                          long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  long long before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const long long v = scratch[w];
    before += w < warp ? v : 0;
    all += v;
  }
  __syncthreads();
  *total = all;
  return before + inc - x;
}

// CTAs per SM the register budget is sized for: d <= 128 fits three CTAs
// (168 registers: measured faster than four CTAs at 128, where the kernel
// spends instructions on register moves), two when the shape carries two
// column tiles and the QJL sketch, or when its shared memory (B200: 228 KB per
// SM, 1 KB reserved per CTA) holds only two; d = 256 fits two.
template <int D, int G, int KB, int VB, bool QJL, bool AFF>
constexpr int decode_min_ctas() {
  return D <= 128 && !(G > 4 && QJL) && 3 * (DecodeGeom<D, G, KB, VB, QJL, AFF>::total + 1024) <= 228 * 1024 ? 3 : 2;
}

template <int D, int G, int KB, int VB, bool QJL, bool AFF>
__global__ void __launch_bounds__(kDecThreads, decode_min_ctas<D, G, KB, VB, QJL, AFF>())
    decode_kernel(const __grid_constant__ Tables tb, const __grid_constant__ CacheView cv,
                  const void* __restrict__ q, int q_dtype, int q_heads, float scale_log2,
                  int max_ctx, int nslots, float* __restrict__ ws) {
  using Geo = DecodeGeom<D, G, KB, VB, QJL, AFF>;
  constexpr int NT = Geo::NT;
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, qd = lane & 3;
  const int H = cv.kv_heads;
  // the code-table lookups address shared memory by immediates that assume
  // where the dynamic shared memory starts (checked on the host as well)
  if ((uint32_t)__cvta_generic_to_shared(smem) != kDynSmemBase) {
    if (tid == 0) atomicOr(cv.status, (int)kFlagLayout);
    return;
  }
  // ---- code tables of the keys and of the values (pairs: two codes -> an
  //      fp16 pair; quads: a byte of four 2-bit codes -> four fp16 values),
  //      each centroid scaled by its table's k_lam / v_lam so that its fp16
  //      rounding is nearly exact.  They depend on the kernel
  //      parameters alone, so they are built before the wait, overlapping the
  //      previous kernel in the stream.
  {
    // each entry is computed once and written to all its copies with 16-byte stores
    constexpr int RK = 1 << Geo::RKL, RV = 1 << Geo::RVL;
    auto quad = [&](const float* c, float lam, int p) {  // byte of four 2-bit codes
      return make_uint2(pack_half2(__float2half_rn(c[p & 3] * lam), __float2half_rn(c[(p >> 2) & 3] * lam)),
                        pack_half2(__float2half_rn(c[(p >> 4) & 3] * lam), __float2half_rn(c[(p >> 6) & 3] * lam)));
    };
    for (int p = tid; p < Geo::LK; p += kDecThreads) {
      uint4* dst = reinterpret_cast<uint4*>(smem + Geo::offLK + (p << Geo::KSH));
      if constexpr (Geo::QK) {
        const uint2 k = quad(tb.k_cent, tb.k_lam, p);
#pragma unroll
        for (int c = 0; c < RK / 2; ++c) dst[c] = make_uint4(k.x, k.y, k.x, k.y);
      } else {
        const uint32_t k = pack_half2(__float2half_rn(tb.k_cent[p & ((1 << KB) - 1)] * tb.k_lam),
                                      __float2half_rn(tb.k_cent[p >> KB] * tb.k_lam));
#pragma unroll
        for (int c = 0; c < RK / 4; ++c) dst[c] = make_uint4(k, k, k, k);
      }
    }
    for (int p = tid; p < Geo::LV; p += kDecThreads) {
      uint4* dst = reinterpret_cast<uint4*>(smem + Geo::offLV + (p << Geo::VSH));
      if constexpr (Geo::QV) {
        const uint2 v = quad(tb.v_cent, tb.v_lam, p);
#pragma unroll
        for (int c = 0; c < RV / 2; ++c) dst[c] = make_uint4(v.x, v.y, v.x, v.y);
      } else {
        const uint32_t v = pack_half2(__float2half_rn(tb.v_cent[p & ((1 << VB) - 1)] * tb.v_lam),
                                      __float2half_rn(tb.v_cent[p >> VB] * tb.v_lam));
#pragma unroll
        for (int c = 0; c < RV / 4; ++c) dst[c] = make_uint4(v, v, v, v);
      }
    }
  }

  pdl_wait();

  // ---- this CTA's tiles [t0, t1) of the T laid end to end over all units
  long long* scan = reinterpret_cast<long long*>(smem + Geo::offSched);
  int* row_n = reinterpret_cast<int*>(scan + kDecWarps);                      // [chunk row] tiles
  long long* row_p = reinterpret_cast<long long*>(row_n + kDecThreads);      // [chunk row] prefix
  // one chunk of rows (the usual case): the scan gives the prefixes and the
  // total at once; otherwise a first pass sums the tiles of every chunk
  const bool one_chunk = cv.batch <= kDecThreads;
  long long rows_total = 0, x0 = 0, p0 = 0;
  if (one_chunk) {
    x0 = tid < cv.batch ? row_tiles(cv, tid, max_ctx) : 0;
    p0 = block_exclusive_scan<kDecThreads>(x0, scan, &rows_total);
  } else {
    for (int b0 = 0; b0 < cv.batch; b0 += kDecThreads) {
      const int r = b0 + tid;
      long long tot;
      block_exclusive_scan<kDecThreads>(r < cv.batch ? row_tiles(cv, r, max_ctx) : 0, scan, &tot);
      rows_total += tot;
    }
  }
  const long long T = rows_total * H;
  const long long t0 = tile_bound(blockIdx.x, T, gridDim.x);
  const long long t1 = tile_bound((long long)blockIdx.x + 1, T, gridDim.x);
  // Everything the next kernel may read before its own wait (the lengths)
  // was complete before this kernel's wait returned, so it may start now; it
  // waits for this grid's completion before it reads any partial.
  pdl_trigger();
  if (t0 >= t1) return;
  // the current segment: tokens [t_begin, t_end) of row b, KV head kvh
  int b = 0, kvh = 0, t_begin = 0, t_end = 0;
  long row_slot = 0;

  // This warp's share of every tile copy: the rows of its own slab, rows
  // [16 warp, 16 warp + 16) of every array, so that a warp waits for its own
  // copies only and the tile loop needs no CTA-wide barrier.  The chunk
  // offsets are the same for all tiles, so they are computed once (stage
  // offset and tile base vary).
  constexpr int WR = 16;  // rows per warp
  constexpr int CK = Geo::kRowB / Geo::CBK, CV = Geo::vRowB / Geo::CBV;
  constexpr int SCH = WR * Geo::sRowB / 16;  // 16-byte chunks of the warp's sign rows
  constexpr int NK = (WR * CK + 31) / 32;
  constexpr int NV = (WR * CV + 31) / 32;
  constexpr int NS = QJL ? (SCH + 31) / 32 : 0;
  static_assert((WR * Geo::sRowB) % 16 == 0 && (WR * 2) % 16 == 0 && (WR * Geo::MB) % 16 == 0,
                "a warp's rows of every array are whole 16-byte chunks");
  int k_dst[NK], k_src[NK], v_dst[NV], v_src[NV];
  bool k_on[NK], v_on[NV];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int c = lane + 32 * i, rr = c / CK, col = c - rr * CK, r = WR * warp + rr;
    k_on[i] = c < WR * CK;
    k_dst[i] = Geo::kvmap(Geo::offK + r * Geo::KS * 4 + col * Geo::CBK);
    k_src[i] = r * Geo::kRowB + col * Geo::CBK;
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = lane + 32 * i, rr = c / CV, col = c - rr * CV, r = WR * warp + rr;
    v_on[i] = c < WR * CV;
    v_dst[i] = Geo::kvmap(Geo::v_row_off(r, col * Geo::CBV / 4));
    v_src[i] = r * Geo::vRowB + col * Geo::CBV;
  }
  auto issue_tile = [&](int stage, int start) {
    // nothing when this warp's slab of the tile is empty; otherwise its 16
    // rows (within capacity: a multiple of 16 past the slab's first token)
    if (WR * warp >= t_end - start) return;
    uint8_t* skv = smem + Geo::kvBase + stage * Geo::kvStride;  // key and value rows
    uint8_t* st = smem + Geo::pBase + stage * Geo::stageA;       // sign rows and norms
    const uint8_t* kb = cv.k_codes + (row_slot + start) * Geo::kRowB;
    const uint8_t* vb = cv.v_codes + (row_slot + start) * Geo::vRowB;
#pragma unroll
    for (int i = 0; i < NK; ++i)
      if (k_on[i]) cp_async_chunk<Geo::CBK>(skv + k_dst[i], kb + k_src[i]);
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (v_on[i]) cp_async_chunk<Geo::CBV>(skv + v_dst[i], vb + v_src[i]);
    const long t0w = row_slot + start + WR * warp;  // the warp's first token
    if constexpr (QJL) {
      const uint8_t* sb = cv.k_signs + t0w * Geo::sRowB;
      uint8_t* sd = st + Geo::offS + WR * warp * Geo::sRowB;
#pragma unroll
      for (int i = 0; i < NS; ++i) {
        const int c = lane + 32 * i;
        if (c < SCH) cp_async16(sd + c * 16, sb + c * 16);
      }
    }
    // per-token metadata: WR * MB bytes of each of the key and value arrays
    // (fp16 norms, or the affine codec's (scale, bias) words), WR * 2 of the
    // QJL residual norms
    constexpr int CM = WR * Geo::MB / 16, CR = QJL ? WR * 2 / 16 : 0;
    for (int c = lane; c < 2 * CM + CR; c += 32) {
      if (c < 2 * CM) {
        const bool vv = c >= CM;
        const int cc = vv ? c - CM : c;
        cp_async16(st + (vv ? Geo::offVN : Geo::offKN) + WR * warp * Geo::MB + cc * 16,
                   reinterpret_cast<const uint8_t*>(vv ? cv.v_norm : cv.k_norm) + t0w * Geo::MB + cc * 16);
      } else {
        const int cc = c - 2 * CM;
        cp_async16(st + Geo::offRN + WR * warp * 2 + cc * 16,
                   reinterpret_cast<const uint8_t*>(cv.k_rnorm + t0w) + cc * 16);
      }
    }
  };

  auto segment = [&]() {
  const int n_tiles = (t_end - t_begin + kDecTile - 1) / kDecTile;
  issue_tile(0, t_begin);
  cp_async_commit();
  if (n_tiles > 1) issue_tile(1, t_begin + kDecTile);
  cp_async_commit();

  // ---- rotate the G queries once, one warp per head, in registers:
  //      u = H (s1 * q); QJL: w = H (s2 * u)
  float* qs = reinterpret_cast<float*>(smem + Geo::offQ);
  float* qs2 = reinterpret_cast<float*>(smem + Geo::offQ2);
  float* red = reinterpret_cast<float*>(smem + Geo::offRed);
  const long q_base = ((long)b * q_heads + (long)kvh * G) * D;
  float amax = 0.f, amax2 = 0.f;
  for (int h = warp; h < G; h += kDecWarps) {
    constexpr int E = D / 32;
    float u[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int ch = lane * E + e;
      const float x = load_any(q, q_base + (long)h * D + ch, q_dtype);
      u[e] = ((tb.s1[ch >> 5] >> (ch & 31)) & 1u) ? -x : x;
    }
    warp_fwht<E>(u, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qs[h * D + lane * E + e] = u[e];
      amax = fmaxf(amax, fabsf(u[e]));
    }
    if constexpr (AFF) {
      // sum of the rotated query over each 64-channel group (GG lanes each)
      constexpr int GG = kAffineGroup / E;
      float t = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) t += u[e];
#pragma unroll
      for (int m = 1; m < GG; m <<= 1) t += __shfl_xor_sync(0xffffffffu, t, m);
      if ((lane & (GG - 1)) == 0)
        reinterpret_cast<float*>(smem + Geo::offUs)[h * Geo::NG + lane / GG] = t;
    }
    if constexpr (QJL) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int ch = lane * E + e;
        u[e] = ((tb.s2[ch >> 5] >> (ch & 31)) & 1u) ? -u[e] : u[e];
      }
      warp_fwht<E>(u, lane);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        qs2[h * D + lane * E + e] = u[e];
        amax2 = fmaxf(amax2, fabsf(u[e]));
      }
    }
  }
  // power-of-two scales that bring each query table's largest entry just
  // below 2^8, keeping the fp16 hi/lo parts in the normal range
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    amax2 = fmaxf(amax2, __shfl_xor_sync(0xffffffffu, amax2, o));
  }
  if (lane == 0) {
    red[warp] = amax;
    red[kDecWarps + warp] = amax2;
  }
  __syncthreads();
  amax = red[0];
  amax2 = red[kDecWarps];
#pragma unroll
  for (int w = 1; w < kDecWarps; ++w) {
    amax = fmaxf(amax, red[w]);
    amax2 = fmaxf(amax2, red[kDecWarps + w]);
  }
  int e1 = 0, e2 = 0;
  frexpf(amax > 0.f ? amax : 1.f, &e1);
  frexpf(amax2 > 0.f ? amax2 : 1.f, &e2);
  const float qsc = ldexpf(1.f, 8 - e1), qsc2 = ldexpf(1.f, 8 - e2);
  // score = post * (tensor-core sum): undoes the query scale and folds the
  // softmax scale, log2(e), the rotation's and the dequantization's 1/sqrt(d)
  // (and sqrt(pi/(2d)) of the QJL estimate)
  // (affine: the keys are in the orthonormal frame, only the query's H is unnormalized)
  const float kpost = AFF ? scale_log2 / (sqrtf((float)D) * qsc) : scale_log2 / ((float)D * qsc * tb.k_lam);
  const float qpost = scale_log2 * sqrtf(3.14159265358979f / (2.0f * D)) / ((float)D * qsc2);

  // ---- B fragments (query columns) in registers
  uint32_t bk[NT][Geo::KBLK][2];
  uint32_t bq[NT][QJL ? Geo::KBLK : 1][2];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int head = 4 * j + (g >> 1), part = g & 1;
    const bool live = head < G;
    const float* r = qs + (live ? head : 0) * D;
#pragma unroll
    for (int kb = 0; kb < Geo::KBLK; ++kb) {
      // key slots 2q,2q+1 -> c0,c0+1; 2q+8,2q+9 -> c0+2,c0+3 (affine: k-block kb
      // lies in group kb / 4, so every MMA sums channels of one group)
      const int c0 = AFF ? kAffineGroup * (kb >> 2) + 16 * qd + 4 * (kb & 3) : qd * (D / 4) + 4 * kb;
      const float4 x = *reinterpret_cast<const float4*>(r + c0);
      uint32_t h01, l01, h23, l23;
      split_pair(x.x * qsc, x.y * qsc, h01, l01);
      split_pair(x.z * qsc, x.w * qsc, h23, l23);
      bk[j][kb][0] = live ? (part ? l01 : h01) : 0u;
      bk[j][kb][1] = live ? (part ? l23 : h23) : 0u;
      if constexpr (QJL) {
        // d >= 128: sign slots 2q,2q+1 -> bits (j0, j0+16) of word kb/8 of the
        // quarter, 2q+8,2q+9 -> (j0+8, j0+24).  d = 64 (16 bits per quarter):
        // slots 2q,2q+1 -> bits (kb, kb+8), 2q+8,2q+9 -> (kb+4, kb+12).
        const int base = D >= 128 ? qd * (D / 4) + 32 * (kb >> 3) + (kb & 7) : qd * 16 + kb;
        constexpr int P1 = D >= 128 ? 16 : 8, P2 = D >= 128 ? 8 : 4, P3 = D >= 128 ? 24 : 12;
        const float* r2 = qs2 + (live ? head : 0) * D;
        uint32_t a_h, a_l, b_h, b_l;
        split_pair(r2[base] * qsc2, r2[base + P1] * qsc2, a_h, a_l);
        split_pair(r2[base + P2] * qsc2, r2[base + P3] * qsc2, b_h, b_l);
        bq[j][kb][0] = live ? (part ? a_l : a_h) : 0u;
        bq[j][kb][1] = live ? (part ? b_l : b_h) : 0u;
      }
    }
  }

  // affine: the query's group sums (times the query scale) for the bias term
  float usc[NT][AFF ? Geo::NG : 1];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int head = 4 * j + qd;
#pragma unroll
    for (int gg = 0; gg < (AFF ? Geo::NG : 1); ++gg)
      usc[j][gg] = (AFF && head < G) ? reinterpret_cast<const float*>(smem + Geo::offUs)[head * Geo::NG + gg] * qsc : 0.f;
  }

  // ---- per-warp online softmax state and output accumulators
  float m_run[NT], l_part[NT];
  float acc[NT][Geo::MBLK][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    m_run[j] = -INFINITY;
    l_part[j] = 0.f;
#pragma unroll
    for (int mb = 0; mb < Geo::MBLK; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][mb][e] = 0.f;
  }
  const uint32_t k_lane = (uint32_t)(lane & ((1 << Geo::RKL) - 1)) << Geo::EKL;
  const uint32_t v_lane = (uint32_t)(lane & ((1 << Geo::RVL) - 1)) << Geo::EVL;
  const int src1 = 8 * qd + (g >> 1), src2 = src1 + 4;  // lanes holding P of tokens 2q(+8), 2q+1(+9)

  // value aggregation of the warp's previous slab, run at the top of its next
  // slab so that it overlaps that slab's score work (registers and the value
  // table only: the stage it came from may already be refilled)
  uint32_t pva[Geo::VCW], pvb[Geo::VCW], pvc[Geo::VCW], pvd[Geo::VCW], ppb[NT][2];
  // affine: (scale, bias) half2 pairs of tokens (2q, 2q+1) and (2q+8, 2q+9)
  uint32_t psab = 0u, pbab = 0u, pscd = 0u, pbcd = 0u;
#pragma unroll
  for (int w = 0; w < Geo::VCW; ++w) pva[w] = pvb[w] = pvc[w] = pvd[w] = 0u;
#pragma unroll
  for (int j = 0; j < NT; ++j) ppb[j][0] = ppb[j][1] = 0u;
  auto aggregate = [&]() {
    uint32_t y0[Geo::VCW], z0[Geo::VCW], y1[Geo::VCW], z1[Geo::VCW];
    interleave_pairs<VB, Geo::VCW>(pva, pvb, y0, z0);
    interleave_pairs<VB, Geo::VCW>(pvc, pvd, y1, z1);
#pragma unroll
    for (int mb = 0; mb < Geo::MBLK; ++mb) {
      uint32_t a0, a1, a2, a3;
      if constexpr (Geo::QV) {
        // byte `by` of y (even channels) or z (odd channels) of word w holds
        // channels c and c + 2 of tokens (a, b): rows g and g + 8 of m-block mb
        constexpr int BPW = Geo::BPW;
        const int w = mb / (2 * BPW), r = mb % (2 * BPW), by = r % BPW;
        const uint32_t* s0 = r < BPW ? y0 : z0;
        const uint32_t* s1 = r < BPW ? y1 : z1;
        const uint2 q0 = lds_table64<kDynSmemBase + Geo::offLV>(quad_index<Geo::IQ, Geo::VSH>(s0[w], by, v_lane));
        const uint2 q1 = lds_table64<kDynSmemBase + Geo::offLV>(quad_index<Geo::IQ, Geo::VSH>(s1[w], by, v_lane));
        a0 = q0.x;
        a1 = q0.y;
        a2 = q1.x;
        a3 = q1.y;
      } else {
        uint32_t e0, o0, e1, o1;
        value_pairs<VB, Geo::VCW, Geo::VSH>(y0, z0, mb, v_lane, e0, o0);
        value_pairs<VB, Geo::VCW, Geo::VSH>(y1, z1, mb, v_lane, e1, o1);
        a0 = lds_table<kDynSmemBase + Geo::offLV>(e0);
        a1 = lds_table<kDynSmemBase + Geo::offLV>(o0);
        a2 = lds_table<kDynSmemBase + Geo::offLV>(e1);
        a3 = lds_table<kDynSmemBase + Geo::offLV>(o1);
      }
      if constexpr (AFF) {  // integer levels -> scale * level + bias of each token
        a0 = hfma2_bits(psab, a0, pbab);
        a1 = hfma2_bits(psab, a1, pbab);
        a2 = hfma2_bits(pscd, a2, pbcd);
        a3 = hfma2_bits(pscd, a3, pbcd);
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) mma16816(acc[j][mb], a0, a1, a2, a3, ppb[j][0], ppb[j][1]);
    }
  };

  for (int it = 0; it < n_tiles; ++it) {
    cp_async_wait<1>();  // this thread's copies of tile it have landed
    __syncwarp();        // and the warp's (its slab's rows only), and the stage refilled
                         // next is no longer read by this warp
    if (it + 2 < n_tiles) issue_tile((it + 2) % kDecStages, t_begin + (it + 2) * kDecTile);
    cp_async_commit();

    const int sidx = it % kDecStages;
    const uint8_t* skv = smem + Geo::kvBase + sidx * Geo::kvStride;  // key and value rows
    const uint8_t* st = smem + Geo::pBase + sidx * Geo::stageA;       // sign rows and norms
    const int n_valid = min(16, t_end - (t_begin + it * kDecTile + 16 * warp));
    if (n_valid <= 0) continue;
    const int r0 = 16 * warp;  // the warp's slab: rows r0 .. r0+15 of the stage
    aggregate();               // O^T += V_hat^T . P^T of the previous slab, on the tensor cores

    // value code chunks of tokens 2q, 2q+1, 2q+8, 2q+9, loaded early so their
    // latency overlaps the score work
    uint32_t va[Geo::VCW], vb2[Geo::VCW], vc[Geo::VCW], vd[Geo::VCW];
    {
      if constexpr (Geo::PV) {
        // words 2g, 2g + 1 of rows 2q, 2q + 1, 2q + 8, 2q + 9 of the slab, as
        // mapped 8-byte pieces (an aligned piece never straddles two blocks)
        uint2 x0, x1, x2, x3;
        if constexpr (Geo::VSW) {  // the rows sit 128, 512, 640 logical bytes after the first
          const uint8_t* v0 = skv + Geo::kvshift(Geo::v_row_off(r0, 0) - Geo::offV) +
                              Geo::kvmap(Geo::v_row_off(2 * qd, 2 * g));
          static_assert(!Geo::VSW || (Geo::v_row_off(1, 0) - Geo::v_row_off(0, 0) == 128 &&
                                      Geo::v_row_off(8, 0) - Geo::v_row_off(0, 0) == 512), "value row blocks");
          x0 = *reinterpret_cast<const uint2*>(v0);
          x1 = *reinterpret_cast<const uint2*>(v0 + Geo::kvshift(128));
          x2 = *reinterpret_cast<const uint2*>(v0 + Geo::kvshift(512));
          x3 = *reinterpret_cast<const uint2*>(v0 + Geo::kvshift(640));
        } else {  // padded rows: rows 2q and 2q + 1 mapped separately, + 8 rows = whole blocks
          const uint8_t* v0 = skv + Geo::kvshift(r0 * Geo::VS * 4);
          const int o0 = Geo::kvmap(Geo::v_row_off(2 * qd, 2 * g));
          const int o1 = Geo::kvmap(Geo::v_row_off(2 * qd + 1, 2 * g));
          constexpr int R8 = Geo::kvshift(8 * Geo::VS * 4);
          x0 = *reinterpret_cast<const uint2*>(v0 + o0);
          x1 = *reinterpret_cast<const uint2*>(v0 + o1);
          x2 = *reinterpret_cast<const uint2*>(v0 + o0 + R8);
          x3 = *reinterpret_cast<const uint2*>(v0 + o1 + R8);
        }
        va[0] = x0.x; va[1] = x0.y;
        vb2[0] = x1.x; vb2[1] = x1.y;
        vc[0] = x2.x; vc[1] = x2.y;
        vd[0] = x3.x; vd[1] = x3.y;
      } else {
        const uint32_t* vrow = reinterpret_cast<const uint32_t*>(skv + Geo::offV) + (r0 + 2 * qd) * Geo::VS;
        load_value_chunk<Geo::VCH, Geo::VCW, Geo::VNW>(vrow, g, va);
        load_value_chunk<Geo::VCH, Geo::VCW, Geo::VNW>(vrow + Geo::VS, g, vb2);
        load_value_chunk<Geo::VCH, Geo::VCW, Geo::VNW>(vrow + 8 * Geo::VS, g, vc);
        load_value_chunk<Geo::VCH, Geo::VCW, Geo::VNW>(vrow + 9 * Geo::VS, g, vd);
      }
    }
    uint32_t vsab = 0u, vbab = 0u, vscd = 0u, vbcd = 0u;
    if constexpr (AFF) {
      // the (scale, bias) words of this thread's value group for its four
      // tokens; tokens past the end get (0, 0), so that their products with a
      // zero probability stay zero whatever the staged bytes hold
      const uint32_t* vm = reinterpret_cast<const uint32_t*>(st + Geo::offVN) + r0 * Geo::NG + (g * (D / 8)) / kAffineGroup;
      const uint32_t ma = 2 * qd < n_valid ? vm[(2 * qd) * Geo::NG] : 0u;
      const uint32_t mb = 2 * qd + 1 < n_valid ? vm[(2 * qd + 1) * Geo::NG] : 0u;
      const uint32_t mc = 2 * qd + 8 < n_valid ? vm[(2 * qd + 8) * Geo::NG] : 0u;
      const uint32_t md = 2 * qd + 9 < n_valid ? vm[(2 * qd + 9) * Geo::NG] : 0u;
      vsab = __byte_perm(ma, mb, 0x5410);  // scales (low halves)
      vbab = __byte_perm(ma, mb, 0x7632);  // biases (high halves)
      vscd = __byte_perm(mc, md, 0x5410);
      vbcd = __byte_perm(mc, md, 0x7632);
    }

    float s0[NT], s1[NT];
    if constexpr (!AFF) {
      // ---- scores: S = K_hat . Qt on the tensor cores; MMA rows g and g + 8
      // are tokens g and g + 8, each k-block split over even / odd
      // accumulators so that the MMA accumulation chains are half as long
      float sacc[2][NT][4];
#pragma unroll
      for (int par = 0; par < 2; ++par)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[par][j][e] = 0.f;
      {
        uint32_t kw0[Geo::KW], kw1[Geo::KW];
        if constexpr (Geo::PV) {
          // words 3 qd .. 3 qd + 2 of rows g and g + 8, each mapped (a row may
          // straddle two 128-byte blocks)
          const uint8_t* k0 = skv + Geo::kvshift(r0 * Geo::KS * 4);
          constexpr int R8 = Geo::kvshift(8 * Geo::KS * 4);
#pragma unroll
          for (int i = 0; i < Geo::KW; ++i) {
            const int o = Geo::kvmap(Geo::offK + g * Geo::KS * 4 + (Geo::KW * qd + i) * 4);
            kw0[i] = *reinterpret_cast<const uint32_t*>(k0 + o);
            kw1[i] = *reinterpret_cast<const uint32_t*>(k0 + o + R8);
          }
        } else {
          const uint32_t* k0 = reinterpret_cast<const uint32_t*>(skv + Geo::offK) + (r0 + g) * Geo::KS;
          load_value_chunk<Geo::QB, Geo::KW, Geo::KNW>(k0, qd, kw0);  // bits of quarter qd, tokens g
          load_value_chunk<Geo::QB, Geo::KW, Geo::KNW>(k0 + 8 * Geo::KS, qd, kw1);  // and g + 8
        }
#pragma unroll
        for (int kb = 0; kb < Geo::KBLK; ++kb) {
          const int o1 = KB * 4 * kb, o2 = o1 + 2 * KB;  // code pairs (c0,c0+1) and (c0+2,c0+3)
          uint32_t a0, a1, a2, a3;
          if constexpr (Geo::QK) {  // the byte of channels c0 .. c0+3: one quad per token
            const uint2 p = lds_table64<kDynSmemBase + Geo::offLK>(quad_index<Geo::IQ, Geo::KSH>(kw0[o1 >> 5], (o1 & 31) >> 3, k_lane));
            const uint2 q = lds_table64<kDynSmemBase + Geo::offLK>(quad_index<Geo::IQ, Geo::KSH>(kw1[o1 >> 5], (o1 & 31) >> 3, k_lane));
            a0 = p.x;
            a1 = q.x;
            a2 = p.y;
            a3 = q.y;
          } else {
            if constexpr (Geo::IQ) {  // 4-bit pairs: whole bytes
              a0 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw0[o1 >> 5], (o1 & 31) >> 3, k_lane));
              a1 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw1[o1 >> 5], (o1 & 31) >> 3, k_lane));
              a2 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw0[o2 >> 5], (o2 & 31) >> 3, k_lane));
              a3 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw1[o2 >> 5], (o2 & 31) >> 3, k_lane));
            } else {
              a0 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw0, Geo::KW, o1, 2 * KB, Geo::KSH) | k_lane);
              a1 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw1, Geo::KW, o1, 2 * KB, Geo::KSH) | k_lane);
              a2 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw0, Geo::KW, o2, 2 * KB, Geo::KSH) | k_lane);
              a3 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw1, Geo::KW, o2, 2 * KB, Geo::KSH) | k_lane);
            }
          }
#pragma unroll
          for (int j = 0; j < NT; ++j) mma16816(sacc[kb & 1][j], a0, a1, a2, a3, bk[j][kb][0], bk[j][kb][1]);
        }
      }
      const uint16_t* kn = reinterpret_cast<const uint16_t*>(st + Geo::offKN) + r0;
      const float kn0 = __half2float(__ushort_as_half(kn[g])) * kpost;
      const float kn1 = __half2float(__ushort_as_half(kn[g + 8])) * kpost;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        s0[j] = ((sacc[0][j][0] + sacc[0][j][1]) + (sacc[1][j][0] + sacc[1][j][1])) * kn0;
        s1[j] = ((sacc[0][j][2] + sacc[0][j][3]) + (sacc[1][j][2] + sacc[1][j][3])) * kn1;
      }
    } else {
      // ---- affine scores: rows g and g + 8 are two tokens (integer levels are
      // exact in fp16); one accumulator per group, then
      // s = sum_gg scale_gg * <levels, q>_gg + bias_gg * sum_gg(q)
      float sacc[Geo::NG][NT][4];
#pragma unroll
      for (int gg = 0; gg < Geo::NG; ++gg)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[gg][j][e] = 0.f;
      uint32_t kw0[Geo::NG][Geo::KWA], kw1[Geo::NG][Geo::KWA];
      const uint32_t* k0 = reinterpret_cast<const uint32_t*>(skv + Geo::offK) + (r0 + g) * Geo::KS;
#pragma unroll
      for (int gg = 0; gg < Geo::NG; ++gg) {
        load_value_chunk<Geo::QBA, Geo::KWA, Geo::KNWA>(k0 + gg * 2 * KB, qd, kw0[gg]);
        load_value_chunk<Geo::QBA, Geo::KWA, Geo::KNWA>(k0 + 8 * Geo::KS + gg * 2 * KB, qd, kw1[gg]);
      }
#pragma unroll
      for (int kb = 0; kb < Geo::KBLK; ++kb) {
        const int gg = kb >> 2, o1 = KB * 4 * (kb & 3), o2 = o1 + 2 * KB;
        uint32_t a0, a1, a2, a3;
        if constexpr (Geo::IQ) {  // 4-bit pairs: whole bytes
          a0 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw0[gg][o1 >> 5], (o1 & 31) >> 3, k_lane));
          a1 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw1[gg][o1 >> 5], (o1 & 31) >> 3, k_lane));
          a2 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw0[gg][o2 >> 5], (o2 & 31) >> 3, k_lane));
          a3 = lds_table<kDynSmemBase + Geo::offLK>(quad_index<true, 8>(kw1[gg][o2 >> 5], (o2 & 31) >> 3, k_lane));
        } else {
          a0 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw0[gg], Geo::KWA, o1, 2 * KB, Geo::KSH) | k_lane);
          a1 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw1[gg], Geo::KWA, o1, 2 * KB, Geo::KSH) | k_lane);
          a2 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw0[gg], Geo::KWA, o2, 2 * KB, Geo::KSH) | k_lane);
          a3 = lds_table<kDynSmemBase + Geo::offLK>(field_scaled(kw1[gg], Geo::KWA, o2, 2 * KB, Geo::KSH) | k_lane);
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(sacc[gg][j], a0, a1, a2, a3, bk[j][kb][0], bk[j][kb][1]);
      }
      const uint32_t* km = reinterpret_cast<const uint32_t*>(st + Geo::offKN) + r0 * Geo::NG;
#pragma unroll
      for (int j = 0; j < NT; ++j) s0[j] = s1[j] = 0.f;
#pragma unroll
      for (int gg = 0; gg < Geo::NG; ++gg) {
        const float2 m0 = __half22float2(*reinterpret_cast<const __half2*>(km + g * Geo::NG + gg));
        const float2 m1 = __half22float2(*reinterpret_cast<const __half2*>(km + (g + 8) * Geo::NG + gg));
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          s0[j] = fmaf(m0.x, sacc[gg][j][0] + sacc[gg][j][1], fmaf(m0.y, usc[j][gg], s0[j]));
          s1[j] = fmaf(m1.x, sacc[gg][j][2] + sacc[gg][j][3], fmaf(m1.y, usc[j][gg], s1[j]));
        }
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        s0[j] *= kpost;
        s1[j] *= kpost;
      }
    }
    if constexpr (QJL) {
      float qacc[2][NT][4];
#pragma unroll
      for (int par = 0; par < 2; ++par)
#pragma unroll
        for (int j = 0; j < NT; ++j) qacc[par][j][0] = qacc[par][j][1] = qacc[par][j][2] = qacc[par][j][3] = 0.f;
      uint32_t sw0[Geo::SW], sw1[Geo::SW];
      const uint32_t* srow = reinterpret_cast<const uint32_t*>(st + Geo::offS) + (r0 + g) * Geo::SS;
      if constexpr (D >= 128) {
#pragma unroll
        for (int w = 0; w < Geo::SW; ++w) {
          sw0[w] = srow[qd * Geo::SW + w];
          sw1[w] = srow[8 * Geo::SS + qd * Geo::SW + w];
        }
      } else {
        // the quarter's 16 bits h, with a copy shifted up by 8: then bit 15 and
        // bit 31 of (x << (15 - kb)) are h[kb] and h[kb + 8]
        const int sh = 16 * (qd & 1);
        const uint32_t h0 = (srow[qd >> 1] >> sh) & 0xffffu, h1 = (srow[8 * Geo::SS + (qd >> 1)] >> sh) & 0xffffu;
        sw0[0] = h0 | (h0 << 8);
        sw1[0] = h1 | (h1 << 8);
      }
#pragma unroll
      for (int kb = 0; kb < Geo::KBLK; ++kb) {
        const int wi = D >= 128 ? kb >> 3 : 0, j0 = D >= 128 ? kb & 7 : kb;
        constexpr int S2 = D >= 128 ? 7 : 11;  // shift that brings the second pair to bits 15, 31
        const uint32_t a0 = sign_pair(sw0[wi] << (15 - j0)), a1 = sign_pair(sw1[wi] << (15 - j0));
        const uint32_t a2 = sign_pair(sw0[wi] << (S2 - j0)), a3 = sign_pair(sw1[wi] << (S2 - j0));
#pragma unroll
        for (int j = 0; j < NT; ++j) mma16816(qacc[kb & 1][j], a0, a1, a2, a3, bq[j][kb][0], bq[j][kb][1]);
      }
      const uint16_t* rn = reinterpret_cast<const uint16_t*>(st + Geo::offRN) + r0;
      const float rn0 = __half2float(__ushort_as_half(rn[g])) * qpost;
      const float rn1 = __half2float(__ushort_as_half(rn[g + 8])) * qpost;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        s0[j] = fmaf((qacc[0][j][0] + qacc[1][j][0]) + (qacc[0][j][1] + qacc[1][j][1]), rn0, s0[j]);
        s1[j] = fmaf((qacc[0][j][2] + qacc[1][j][2]) + (qacc[0][j][3] + qacc[1][j][3]), rn1, s1[j]);
      }
    }
    const bool ok0 = g < n_valid, ok1 = g + 8 < n_valid;

    // ---- value magnitude of tokens g, g + 8: ev ~ log2 |v| and the factor
    //      vm = |v| that stays with the weight.  The running maximum below is
    //      taken over s + ev, so every weight p * |v| = 2^(s - max) |v| stays
    //      below 2^(lazy slack) whatever the norms are (tiny, huge or mixed)
    //      and the hi/lo split of P keeps its ~22 bits in fp16's normal range.
    //      Lloyd-Max: |v| is the stored fp16 norm and ev its hardware log2
    //      (2^-30 added, so a zero norm gives -30).  Affine: |v| = 2^ev with ev
    //      the exponent of the token's largest |scale| or |bias| (clamped to
    //      [-14, 14]); the value side scales (scale, bias) by 2^-ev exactly.
    float vm0, vm1, ev0, ev1;
    uint32_t vfac = 0u;  // affine: fp16 bits of 2^-ev of tokens g (low) and g + 8 (high)
    if constexpr (!AFF) {
      const uint16_t* vn = reinterpret_cast<const uint16_t*>(st + Geo::offVN) + r0;
      const uint32_t b0 = vn[g], b1 = vn[g + 8];
      vm0 = __half2float(__ushort_as_half((uint16_t)b0));
      vm1 = __half2float(__ushort_as_half((uint16_t)b1));
      ev0 = ok0 ? fast_log2(vm0 + 0x1p-30f) : 0.f;  // zero norms give -30
      ev1 = ok1 ? fast_log2(vm1 + 0x1p-30f) : 0.f;
    } else {
      const uint32_t* vmw = reinterpret_cast<const uint32_t*>(st + Geo::offVN) + (r0 + g) * Geo::NG;
      uint32_t f0 = 1u, f1 = 1u;  // largest fp16 exponent field among |scale|, |bias|
#pragma unroll
      for (int gg = 0; gg < Geo::NG; ++gg) {
        const uint32_t x0 = vmw[gg], x1 = vmw[8 * Geo::NG + gg];
        f0 = max(f0, max((x0 >> 10) & 31u, (x0 >> 26) & 31u));
        f1 = max(f1, max((x1 >> 10) & 31u, (x1 >> 26) & 31u));
      }
      const int e0 = min((int)f0, 29) - 15, e1 = min((int)f1, 29) - 15;  // [-14, 14]
      ev0 = (float)e0;
      ev1 = (float)e1;
      vm0 = __int_as_float((e0 + 127) << 23);  // 2^ev exactly
      vm1 = __int_as_float((e1 + 127) << 23);
      vfac = (uint32_t)((15 - e0) << 10) | ((uint32_t)((15 - e1) << 10) << 16);
    }

    // ---- online softmax (per warp, per head), P in fp16 hi/lo for the output MMA
    uint32_t pb[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (!ok0) s0[j] = -INFINITY;
      if (!ok1) s1[j] = -INFINITY;
      float mx = fmaxf(s0[j] + ev0, s1[j] + ev1);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      // lazy rescale: the running maximum moves only when a score passes it by
      // more than kLazyLog2, so p stays below 2^kLazyLog2 and the weights below
      // 2^(kLazyLog2 + 1) (well inside fp16); the vote keeps the branch uniform
      // and, after the first slabs, almost never taken
      if (__any_sync(0xffffffffu, mx > m_run[j] + kLazyLog2)) {
        const float mn = fmaxf(m_run[j], mx);
        const float alpha = fast_exp2(m_run[j] - mn);
        l_part[j] *= alpha;
#pragma unroll
        for (int mb = 0; mb < Geo::MBLK; ++mb)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[j][mb][e] *= alpha;
        m_run[j] = mn;
      }
      const float p0 = ok0 ? fast_exp2(s0[j] - m_run[j]) : 0.f;
      const float p1 = ok1 ? fast_exp2(s1[j] - m_run[j]) : 0.f;
      l_part[j] += p0 + p1;
      const float w0 = ok0 ? p0 * vm0 : 0.f, w1 = ok1 ? p1 * vm1 : 0.f;
      uint32_t whi, wlo;
      split_pair(w0, w1, whi, wlo);
      const uint32_t x1h = __shfl_sync(0xffffffffu, whi, src1), x1l = __shfl_sync(0xffffffffu, wlo, src1);
      const uint32_t x2h = __shfl_sync(0xffffffffu, whi, src2), x2l = __shfl_sync(0xffffffffu, wlo, src2);
      const uint32_t x1 = (g & 1) ? x1l : x1h, x2 = (g & 1) ? x2l : x2h;
      pb[j][0] = __byte_perm(x1, x2, 0x5410);  // tokens 2q, 2q+1
      pb[j][1] = __byte_perm(x1, x2, 0x7632);  // tokens 2q+8, 2q+9
    }

    // ---- hand this slab's value codes and P to the next slab's aggregation
#pragma unroll
    for (int w = 0; w < Geo::VCW; ++w) {
      pva[w] = va[w];
      pvb[w] = vb2[w];
      pvc[w] = vc[w];
      pvd[w] = vd[w];
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      ppb[j][0] = pb[j][0];
      ppb[j][1] = pb[j][1];
    }
    if constexpr (AFF) {
      // (scale, bias) of tokens 2q, 2q+1 and 2q+8, 2q+9 times their 2^-ev
      // (exact: powers of two), from the lanes that scored those tokens
      const uint32_t x1 = __shfl_sync(0xffffffffu, vfac, src1), x2 = __shfl_sync(0xffffffffu, vfac, src2);
      const uint32_t fab = __byte_perm(x1, x2, 0x5410), fcd = __byte_perm(x1, x2, 0x7632);
      psab = hmul2_bits(vsab, fab);
      pbab = hmul2_bits(vbab, fab);
      pscd = hmul2_bits(vscd, fcd);
      pbcd = hmul2_bits(vbcd, fcd);
    }
  }
  aggregate();  // the warp's last slab

  // ---- epilogue: merge the four warps (fixed order) into the CTA's partial
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float l = l_part[j];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    l_part[j] = l;
  }
  __syncthreads();  // every warp is done with the stages (no copies are in flight)
  // merge buffer over the stages' key / value rows: m[warp][G], l[warp][G],
  // O[warp][G][D] (floats; float i at logical byte 4 i)
  auto mrg = [&](int i) -> float& { return *reinterpret_cast<float*>(smem + Geo::kvBase + Geo::kvmap(4 * i)); };
  constexpr int LW = kDecWarps * G, OW = 2 * kDecWarps * G;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int head = 4 * j + qd;
    if (head < G) {
      if (g == 0) {
        mrg(warp * G + head) = m_run[j];
        mrg(LW + warp * G + head) = l_part[j];
      }
      const int o = OW + (warp * G + head) * D + g * (D / 8);
#pragma unroll
      for (int mb = 0; mb < Geo::MBLK; ++mb) {
        mrg(o + value_channel<Geo::QV, Geo::BPW>(mb, 0)) = acc[j][mb][0] + acc[j][mb][1];
        mrg(o + value_channel<Geo::QV, Geo::BPW>(mb, 1)) = acc[j][mb][2] + acc[j][mb][3];
      }
    }
  }
  __syncthreads();
  // workspace: o partials [slot][G][D], then (m, l) [slot][G][2]; slot = CTA + unit
  float* wt = reinterpret_cast<float*>(smem + Geo::offRed);   // [warp][G] merge weights
  if (tid < kDecWarps * G) {
    const int w = tid / G, h = tid % G;
    float M = mrg(h);
#pragma unroll
    for (int v = 1; v < kDecWarps; ++v) M = fmaxf(M, mrg(v * G + h));
    const float m = mrg(w * G + h);
    wt[tid] = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
    if (w == 0) red[kDecWarps * G + h] = M;
  }
  __syncthreads();
  const long slot = (long)blockIdx.x + (long)b * H + kvh;
  float* dst_o = ws + slot * (G * D);
  float* dst_ml = ws + (long)nslots * (G * D) + slot * (G * 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int h = i / D, ch = i % D;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) v = fmaf(mrg(OW + (w * G + h) * D + ch), wt[w * G + h], v);
    dst_o[i] = v;
  }
  if (tid < G) {
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) l = fmaf(mrg(LW + w * G + tid), wt[w * G + tid], l);
    dst_ml[2 * tid] = red[kDecWarps * G + tid];
    dst_ml[2 * tid + 1] = l;
  }
  __syncthreads();  // the merge buffers alias the stages the next segment fills
  };

  // ---- walk the rows whose tiles meet [t0, t1), one chunk of rows at a time
  long long base = 0;  // tiles per KV head of the rows before the chunk
  for (int b0 = 0; b0 < cv.batch && base * H < t1; b0 += kDecThreads) {
    long long x = x0, p = p0, tot = rows_total;
    if (!one_chunk) {
      const int r = b0 + tid;
      x = r < cv.batch ? row_tiles(cv, r, max_ctx) : 0;
      p = base + block_exclusive_scan<kDecThreads>(x, scan, &tot);
    }
    row_n[tid] = (int)x;
    row_p[tid] = p;
    __syncthreads();
    // the prefixes never decrease: search the first row ending after t0
    const int rows = min(kDecThreads, cv.batch - b0);
    int lo = 0, hi = rows;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if ((row_p[mid] + row_n[mid]) * H > t0) hi = mid; else lo = mid + 1;
    }
    for (int i = lo; i < rows && row_p[i] * H < t1; ++i) {
      const int n = row_n[i];
      if (n == 0) continue;
      b = b0 + i;
      const long long rs = row_p[i] * H;  // first tile of the row
      const int L = row_len(cv, b, max_ctx);
      const int h_lo = t0 > rs ? (int)((t0 - rs) / n) : 0;
      const int h_hi = (int)min((long long)(H - 1), (t1 - 1 - rs) / n);
      for (kvh = h_lo; kvh <= h_hi; ++kvh) {
        const long long us = rs + (long long)kvh * n;
        t_begin = (int)(max(t0, us) - us) * kDecTile;
        t_end = min((int)(min(t1, us + n) - us) * kDecTile, L);
        row_slot = ((long)b * H + kvh) * cv.capacity;
        segment();
      }
    }
    base += tot;
    __syncthreads();  // the row arrays are rewritten by the next chunk
  }
}

// Per-kernel record of the devices it has been configured on (each kernel
// owns one: kernels of one signature share a function-pointer type, so the
// record cannot be keyed on the type).
struct KernelConfig {
  static constexpr int kMaxDevices = 64;
  std::mutex mu;
  int occupancy[kMaxDevices] = {};  // 0: not yet configured on that device
};

// Sets the kernel's shared-memory attribute and measures how many of its CTAs
// fit on one SM, once per device; thread-safe (host threads may drive
// different GPUs at once).
template <typename Kernel>
cudaError_t configure_kernel(KernelConfig& cfg, Kernel kern, int smem_bytes, int threads,
                             int* ctas_per_sm) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= KernelConfig::kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(cfg.mu);
  if (cfg.occupancy[dev] == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem_bytes);
    if (e != cudaSuccess) return e;
    cfg.occupancy[dev] = n > 0 ? n : 1;
  }
  if (ctas_per_sm) *ctas_per_sm = cfg.occupancy[dev];
  return cudaSuccess;
}

// The decode kernel of one compile-time shape: configured, and its CTAs per SM.
template <int D, int G, int KB, int VB, bool QJL, bool AFF>
cudaError_t configure_shape(int* ctas_per_sm) {
  using Geo = DecodeGeom<D, G, KB, VB, QJL, AFF>;
  static KernelConfig cfg;  // one per shape
  auto kern = decode_kernel<D, G, KB, VB, QJL, AFF>;
  // the dynamic shared memory must start at kDynSmemBase: no static shared
  // memory, and the per-CTA reserved shared memory of that size
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  int dev = 0, reserved = -1;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  if (fa.sharedSizeBytes != 0 || reserved != (int)kDynSmemBase) return cudaErrorNotSupported;
  return configure_kernel(cfg, kern, Geo::total, kDecThreads, ctas_per_sm);
}

// Launches decode_kernel for one compile-time shape (grid: plan.ctas CTAs).
template <int D, int G, int KB, int VB, bool QJL, bool AFF>
cudaError_t launch_decode_shape(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                                int q_heads, float scale_log2, int max_ctx,
                                const DecodePlan& plan, float* ws, cudaStream_t stream) {
  using Geo = DecodeGeom<D, G, KB, VB, QJL, AFF>;
  auto kern = decode_kernel<D, G, KB, VB, QJL, AFF>;
  cudaError_t e = configure_shape<D, G, KB, VB, QJL, AFF>(nullptr);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.ctas);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = Geo::total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tb, cv, q, dtype, q_heads, scale_log2, max_ctx,
                            plan.slots, ws);
}

// Per-head-dim, per-codec dispatch over (group, k_bits, v_bits, qjl);
// instantiated in the tq_decode_d<D>.cu (Lloyd-Max) and tq_decode_affine_d<D>.cu
// (affine) translation units.
template <int D, bool AFF>
cudaError_t decode_occupancy_dim(const Tables& tb, int group, int* ctas_per_sm);

template <int D, bool AFF>
cudaError_t dispatch_occupancy_dim(const Tables& tb, int G, int* ctas_per_sm) {
#define TQ_CASE(GG, KB, VB, QJ)                                             \
  if (G == GG && tb.k_bits == KB && tb.v_bits == VB && (tb.qjl != 0) == QJ) \
    return configure_shape<D, GG, KB, VB, QJ, AFF>(ctas_per_sm);
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

template <int D, bool AFF>
cudaError_t launch_decode_dim(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                              int q_heads, float scale_log2, int max_ctx, const DecodePlan& plan,
                              float* ws, cudaStream_t stream);

template <int D, bool AFF>
cudaError_t dispatch_decode_dim(const Tables& tb, const CacheView& cv, const void* q, int dtype,
                                int q_heads, float scale_log2, int max_ctx,
                                const DecodePlan& plan, float* ws, cudaStream_t stream) {
  const int G = q_heads / cv.kv_heads;
#define TQ_CASE(GG, KB, VB, QJ)                                                                \
  if (G == GG && tb.k_bits == KB && tb.v_bits == VB && (tb.qjl != 0) == QJ)                    \
    return launch_decode_shape<D, GG, KB, VB, QJ, AFF>(tb, cv, q, dtype, q_heads, scale_log2, \
                                                       max_ctx, plan, ws, stream);
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
