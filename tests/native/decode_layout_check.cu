// Host-side check of the decode kernel's shared-memory layouts (no GPU):
// every staged row, table entry and merge float lands where the kernel's
// index arithmetic says, inside its region, without overlap, and the reads a
// warp issues at once fall on distinct banks where the layout promises it.
// Built and run by tests/test_decode_layout.py; prints "bad N" per shape.
#include "tq_decode_impl.cuh"
#include "tq_lutmm.cu"

#include <cstdio>
#include <set>

using namespace tq;

static int g_bad = 0;
#define CHECK(c)                                                        \
  do {                                                                  \
    if (!(c)) {                                                         \
      if (g_bad < 20) std::printf("  failed: %s (line %d)\n", #c, __LINE__); \
      ++g_bad;                                                          \
    }                                                                   \
  } while (0)

// 3-bit keys / 4-bit values at d 128: tables and staged rows share [0, 64 KB)
template <int G, bool QJL>
void check_pv() {
  using Geo = DecodeGeom<128, G, 3, 4, QJL, false>;
  static_assert(Geo::PV, "PV shape");
  const int before = g_bad;
  // value entries fill the first half of every 256 bytes, key entries the
  // second half of the first 64
  for (int e = 0; e < 256; ++e) CHECK(Geo::offLV + (e << Geo::VSH) == 256 * e);
  for (int e = 0; e < 64; ++e) CHECK(Geo::offLK + (e << Geo::KSH) == 256 * e + 128);
  // every logical byte of the stages and of the merge buffer maps into a
  // second half, past the key table, below 64 KB, one to one
  std::set<int> seen;
  for (int s = 0; s < kDecStages; ++s)
    for (int x = 0; x < Geo::kvBytes; x += 4) {
      const int p = Geo::kvBase + s * Geo::kvStride + Geo::kvmap(x);
      CHECK((p & 255) >= 128 && p >= 16384 + 128 && p + 4 <= 65536);
      CHECK(seen.insert(p).second);
    }
  for (int x = 0; x < Geo::mergeBytes; x += 4) {
    const int p = Geo::kvBase + Geo::kvmap(x);
    CHECK((p & 255) >= 128 && p >= 16384 + 128 && p + 4 <= 65536);
  }
  // the other stage parts and the rest come after the table region
  CHECK(Geo::pBase == 65536 && Geo::offQ >= Geo::pBase + kDecStages * Geo::stageA);
  // value rows: a bijection onto [offV, offV + 64 VS words), 16-byte chunks whole
  std::set<int> vx;
  for (int r = 0; r < kDecTile; ++r)
    for (int w = 0; w < 16; ++w) {
      const int x = Geo::v_row_off(r, w);
      CHECK(x >= Geo::offV && x + 4 <= Geo::offV + kDecTile * Geo::VS * 4 && x % 4 == 0);
      CHECK(vx.insert(x).second);
      if (w % 4) CHECK(x == Geo::v_row_off(r, w - w % 4) + 4 * (w % 4));
      else CHECK(x % 16 == 0);
    }
  for (int r = 0; r < kDecTile; ++r)
    for (int w = 0; w < Geo::KS; ++w) CHECK(Geo::offK + r * Geo::KS * 4 + 4 * w + 4 <= Geo::offV);
  // the kernel's value reads (rows r0 + 2q + c, words 2g and 2g + 1) and key
  // reads (words 3q + i of rows r0 + g, r0 + g + 8), as it computes them
  for (int warp = 0; warp < kDecWarps; ++warp) {
    const int r0 = 16 * warp;
    for (int c : {0, 1, 8, 9})
      for (int half = 0; half < 2; ++half) {
        std::set<int> banks;
        for (int lane = 16 * half; lane < 16 * half + 16; ++lane) {
          const int g = lane >> 2, q = lane & 3;
          const int want = Geo::kvmap(Geo::v_row_off(r0 + 2 * q + c, 2 * g));
          int got;
          if (Geo::VSW)
            got = Geo::kvshift(Geo::v_row_off(r0, 0) - Geo::offV) + Geo::kvmap(Geo::v_row_off(2 * q, 2 * g)) +
                  Geo::kvshift(c == 0 ? 0 : c == 1 ? 128 : c == 8 ? 512 : 640);
          else
            got = Geo::kvshift(r0 * Geo::VS * 4) + Geo::kvmap(Geo::v_row_off(2 * q + (c & 1), 2 * g)) +
                  (c >= 8 ? Geo::kvshift(8 * Geo::VS * 4) : 0);
          CHECK(got == want);
          CHECK(Geo::kvmap(Geo::v_row_off(r0 + 2 * q + c, 2 * g + 1)) == want + 4);  // one 8-byte piece
          const int p = Geo::kvBase + want;
          banks.insert((p / 4) % 32);
          banks.insert((p / 4 + 1) % 32);
        }
        CHECK(banks.size() == 32);  // 64-bit loads, served per half-warp
      }
    for (int rr : {0, 8})
      for (int i = 0; i < 3; ++i) {
        std::set<int> banks;
        for (int lane = 0; lane < 32; ++lane) {
          const int g = lane >> 2, q = lane & 3;
          const int want = Geo::kvmap(Geo::offK + (r0 + g + rr) * Geo::KS * 4 + (3 * q + i) * 4);
          const int got = Geo::kvshift(r0 * Geo::KS * 4) + Geo::kvmap(Geo::offK + g * Geo::KS * 4 + (3 * q + i) * 4) +
                          (rr ? Geo::kvshift(8 * Geo::KS * 4) : 0);
          CHECK(got == want);
          banks.insert(((Geo::kvBase + want) / 4) % 32);
        }
        CHECK(banks.size() == 32);
      }
  }
  // three CTAs per SM where the register budget assumes it
  if (decode_min_ctas<128, G, 3, 4, QJL, false>() == 3) CHECK(3 * (Geo::total + 1024) <= 228 * 1024);
  std::printf("pv G%d qjl%d total %d bad %d\n", G, (int)QJL, Geo::total, g_bad - before);
}

// interleaved key / value tables (2-bit quads, 4-bit pairs)
template <int D, int KB, int VB, bool QJL, bool AFF>
void check_interleaved() {
  using Geo = DecodeGeom<D, 4, KB, VB, QJL, AFF>;
  static_assert(Geo::IQ, "interleaved shape");
  const int before = g_bad;
  const int kbytes = (1 << Geo::RKL) << Geo::EKL, vbytes = (1 << Geo::RVL) << Geo::EVL;
  CHECK(kbytes == 128 && vbytes == 128 && Geo::LK == 256 && Geo::LV == 256);
  for (int e = 0; e < 256; ++e) {
    CHECK(Geo::offLK + (e << Geo::KSH) == Geo::offLK + 256 * e);
    CHECK(Geo::offLV + (e << Geo::VSH) == Geo::offLK + 256 * e + 128);
  }
  CHECK(Geo::offLK >= kDecStages * Geo::stageA && Geo::offQ == Geo::offLK + 65536);
  std::printf("interleaved d%d k%d v%d qjl%d affine%d total %d bad %d\n", D, KB, VB, (int)QJL, (int)AFF,
              Geo::total, g_bad - before);
}

// LUT matmul, 4-bit codes at d <= 128: table entries 256 bytes apart, the
// stages' code rows in the entries' second halves
template <int D, int NT>
void check_lut() {
  using Geo = MmGeom<D, 4, NT>;
  static_assert(Geo::BP, "byte-permute layout");
  const int before = g_bad;
  for (int e = 0; e < 256; ++e) CHECK(Geo::offLK + (e << Geo::KSH) == 256 * e);
  std::set<int> seen;
  for (int s = 0; s < Geo::STG; ++s)
    for (int r = 0; r < kMmRows; ++r) {
      for (int w = 0; w < Geo::KS; ++w) {
        const int p = Geo::code_off(s, r * Geo::KS * 4 + 4 * w);
        CHECK((p & 255) >= 128 && p + 4 <= 65536);
        CHECK(seen.insert(p).second);
        CHECK(p == Geo::code_off(s, r * Geo::KS * 4) + 4 * w);  // a row never straddles two blocks
      }
      if (r + 8 < kMmRows)  // the kernel's row g + 8: 2 * 8 * KS words further
        CHECK(Geo::code_off(s, (r + 8) * Geo::KS * 4) == Geo::code_off(s, r * Geo::KS * 4) + 2 * 8 * Geo::KS * 4);
    }
  // a quarter-warp's 16-byte code reads (rows r0 + g, words 4 q .. 4 q + 3) cover 32 banks
  for (int r0 = 0; r0 < kMmRows; r0 += 16)
    for (int quarter = 0; quarter < 4; ++quarter) {
      std::set<int> banks;
      for (int lane = 8 * quarter; lane < 8 * quarter + 8; ++lane) {
        const int g = lane >> 2, q = lane & 3;
        const int p = Geo::code_off(0, (r0 + g) * Geo::KS * 4) + 16 * (q % (Geo::KS / 4));
        for (int k = 0; k < 4; ++k) banks.insert((p / 4 + k) % 32);
      }
      if (Geo::KS == 16) CHECK(banks.size() == 32);
    }
  CHECK(Geo::pBase == 65536 && Geo::total == Geo::pBase + Geo::STG * Geo::stageA);
  std::printf("lut d%d nt%d total %d bad %d\n", D, NT, Geo::total, g_bad - before);
}

int main() {
  check_lut<128, 1>();
  check_lut<64, 1>();
  check_pv<1, false>();
  check_pv<4, false>();
  check_pv<8, false>();
  check_pv<1, true>();
  check_pv<4, true>();
  check_pv<8, true>();
  check_interleaved<64, 2, 2, false, false>();
  check_interleaved<128, 2, 2, true, false>();
  check_interleaved<256, 2, 2, true, false>();
  check_interleaved<64, 4, 4, false, false>();
  check_interleaved<128, 4, 4, true, false>();
  check_interleaved<128, 4, 4, false, true>();
  std::printf("total bad %d\n", g_bad);
  return g_bad ? 1 : 0;
}
