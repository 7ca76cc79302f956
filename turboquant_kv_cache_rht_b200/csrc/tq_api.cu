// C ABI of libtq: argument validation, codebook/sign construction on the host,
// and kernel dispatch.  See include/tq.h for the contract of every entry point.
#include "../../include/tq.h"
#include "tq_internal.cuh"

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

struct tq_codebook {
  tq_params params;
  tq::Tables tables;
};

namespace {

thread_local std::string g_last_error;

tq_status fail(tq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

tq_status ok() {
  g_last_error.clear();
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// Lloyd-Max quantizer of the standard normal distribution ("How to Use
// TurboQuant with the MLX-VLM Python API", "What is TurboQuant?": _codebook;
// "mlx-turboquant" README: Lloyd-Max codebook for the near-Gaussian rotated
// coordinates).  Lloyd's two conditions are iterated in double precision until
// no level moves by 1e-14: boundaries at the midpoints of adjacent levels,
// levels at the conditional means of their cells.
// ---------------------------------------------------------------------------
double normal_density(double x) {
  if (std::isinf(x)) return 0.0;
  return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
}

// P(X > x)
double normal_tail(double x) { return 0.5 * std::erfc(x / std::sqrt(2.0)); }

// P(lo < X < hi), arranged so that neither tail is obtained by cancellation.
double normal_mass(double lo, double hi) {
  if (lo >= 0.0) return normal_tail(lo) - normal_tail(hi);
  if (hi <= 0.0) return normal_tail(-hi) - normal_tail(-lo);
  return 1.0 - normal_tail(-lo) - normal_tail(hi);
}

double normal_cell_mean(double lo, double hi) {
  return (normal_density(lo) - normal_density(hi)) / normal_mass(lo, hi);
}

// The exact distribution of a rotated coordinate.  For a fixed x, each
// coordinate of R x / ||x|| is a coordinate of a uniformly random unit vector
// of R^d, so Z = sqrt(d) (R x)_i / ||x|| has density
// f(z) = C_d (1 - z^2/d)^((d-3)/2) on |z| < sqrt(d), C_d = Gamma(d/2) /
// (sqrt(pi d) Gamma((d-1)/2)); the rotated coordinates are only near-Gaussian
// ("mlx-turboquant" README, introduction).  Cell masses are integrated
// directly (composite 10-point Gauss-Legendre on pieces at most 1/4 wide,
// compensated sums), so a small outer cell is not the difference of two
// nearly equal cumulative integrals.
struct Sphere {
  int d;
  double c;  // C_d
};

struct GaussLegendre10 {
  double x[10], w[10];
  GaussLegendre10() {  // roots of the Legendre polynomial P_10 by Newton's method
    for (int i = 0; i < 10; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / 10.5), dp = 1.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;  // P_0, P_1, then the three-term recurrence
        for (int k = 2; k <= 10; ++k) {
          const double pk = ((2 * k - 1) * z * p1 - (k - 1) * p0) / k;
          p0 = p1;
          p1 = pk;
        }
        dp = 10 * (z * p1 - p0) / (z * z - 1.0);
        const double step = p1 / dp;
        z -= step;
        if (std::fabs(step) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

// (1 - z^2/d)^k as exp(k log1p(-z^2/d)): a power of the rounded base would
// carry k times the base's rounding error, which is what limits Lloyd's
// iteration near its tolerance.
double sphere_power(double z, int d, double k) {
  const double x = z * z / d;
  return x >= 1.0 ? 0.0 : std::exp(k * std::log1p(-x));
}

double sphere_density(const Sphere& sp, double z) { return sp.c * sphere_power(z, sp.d, (sp.d - 3) / 2.0); }

double sphere_mass(const Sphere& sp, double lo, double hi) {
  static const GaussLegendre10 gl;
  const double r = std::sqrt((double)sp.d);
  lo = std::fmax(lo, -r);
  hi = std::fmin(hi, r);
  if (!(hi > lo)) return 0.0;
  const int pieces = std::max(1, (int)std::ceil((hi - lo) * 4.0));
  const double h = (hi - lo) / pieces;
  double sum = 0.0, comp = 0.0;  // Kahan summation
  for (int p = 0; p < pieces; ++p) {
    const double mid = lo + (p + 0.5) * h;
    for (int i = 0; i < 10; ++i) {
      const double term = gl.w[i] * sphere_density(sp, mid + 0.5 * h * gl.x[i]) * 0.5 * h - comp;
      const double next = sum + term;
      comp = (next - sum) - term;
      sum = next;
    }
  }
  return sum;
}

// Integral of z f(z) over (lo, hi): an antiderivative of z (1 - z^2/d)^k is
// -(d / (2 (k + 1))) (1 - z^2/d)^(k + 1), here with k = (d - 3) / 2.
double sphere_cell_mean(const Sphere& sp, double lo, double hi) {
  const double d = sp.d, r = std::sqrt(d);
  auto g = [&](double z) { return std::fabs(z) >= r ? 0.0 : sphere_power(z, sp.d, (d - 1) / 2); };
  return sp.c * d / (d - 1) * (g(lo) - g(hi)) / sphere_mass(sp, lo, hi);
}

// Lloyd's iteration from `lv` (levels ascending) with the given cell-mean rule.
template <typename CellMean>
bool lloyd_iterate(int levels, double* lv, CellMean cell_mean) {
  double next[16], edge[17];
  for (int iter = 0; iter < 1000000; ++iter) {
    edge[0] = -INFINITY;
    edge[levels] = INFINITY;
    for (int j = 1; j < levels; ++j) edge[j] = 0.5 * (lv[j - 1] + lv[j]);
    double moved = 0.0;
    for (int j = 0; j < levels; ++j) {
      next[j] = cell_mean(edge[j], edge[j + 1]);
      moved = std::fmax(moved, std::fabs(next[j] - lv[j]));
    }
    std::memcpy(lv, next, sizeof(double) * levels);
    if (moved < 1e-14) return true;
  }
  return false;
}

// Levels of the Lloyd-Max quantizer of N(0,1) (kind 0) or of the rotated-
// coordinate distribution for head_dim d (kind 1, started from the N(0,1)
// solution).
bool lloyd_max(int levels, int kind, int d, double* lv) {
  for (int j = 0; j < levels; ++j) lv[j] = -2.0 + 4.0 * (j + 0.5) / levels;
  if (!lloyd_iterate(levels, lv, normal_cell_mean)) return false;
  if (kind == 0) return true;
  const Sphere sp{d, std::exp(std::lgamma(d / 2.0) - std::lgamma((d - 1) / 2.0)) /
                         std::sqrt(M_PI * d)};
  return lloyd_iterate(levels, lv, [&](double lo, double hi) { return sphere_cell_mean(sp, lo, hi); });
}

// float32 table: odd-symmetric levels, boundaries = float32 midpoints.
bool build_codebook(int bits, int kind, int d, float* cent, float* bnd) {
  const int levels = 1 << bits, half = levels / 2;
  double lv[16];
  if (!lloyd_max(levels, kind, d, lv)) return false;
  for (int j = 0; j < half; ++j) {
    const float pos = (float)((lv[half + j] - lv[half - 1 - j]) / 2.0);
    cent[half + j] = pos;
    cent[half - 1 - j] = -pos;
  }
  for (int j = 0; j + 1 < levels; ++j) {
    volatile float s = cent[j] + cent[j + 1];  // two float32 roundings, no contraction
    bnd[j] = s * 0.5f;
  }
  for (int j = levels - 1; j < 16; ++j) bnd[j] = INFINITY;
  for (int j = levels; j < 16; ++j) cent[j] = 0.0f;
  return true;
}

// fp16 rounding of a float in fp16's normal range, to nearest even (the
// table scale search below only meets magnitudes in [2^-14, 2^15)).
double round_fp16_normal(float x) {
  int e = 0;
  const double m = std::frexp((double)x, &e);       // x = m 2^e, 0.5 <= |m| < 1
  return std::ldexp(std::nearbyint(std::ldexp(m, 11)), e - 11);  // 11 significant bits
}

// Scale lam in [1, 2) under which the fp16 roundings of lam * c_j (formed as
// an fp32 product, as the decode kernel forms it) come closest to the exact
// products: the largest relative rounding error over the nonzero entries is
// minimal.  The decode kernel's code tables hold fp16(lam * c_j) and undo lam
// in fp32, so a table of 4, 8 or 16 Lloyd-Max levels carries ~2^-22, ~2^-16
// or ~2^-13 relative error instead of fp16's 2^-12.
float fp16_table_scale(const float* cent, int levels) {
  constexpr int kSteps = 1 << 16;
  float best = 1.0f;
  double best_err = INFINITY;
  for (int i = 0; i < kSteps; ++i) {
    const float lam = 1.0f + (float)i / (float)kSteps;
    double err = 0.0;
    for (int j = levels / 2; j < levels && err < best_err; ++j) {  // odd symmetry
      const float x = cent[j] * lam;
      if (x == 0.0f) continue;
      err = std::max(err, std::fabs(round_fp16_normal(x) - (double)x) / std::fabs((double)x));
    }
    if (err < best_err) {
      best_err = err;
      best = lam;
    }
  }
  return best;
}

// Affine codec tables: the integer levels 0 .. 2^bits - 1 and their midpoints
// (the decode kernel's pair tables turn code pairs into these levels).
void build_affine_levels(int bits, float* cent, float* bnd) {
  const int levels = 1 << bits;
  for (int j = 0; j < 16; ++j) {
    cent[j] = j < levels ? (float)j : 0.0f;
    bnd[j] = j + 1 < levels ? (float)j + 0.5f : INFINITY;
  }
}

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the sign of channel i is the
// top bit of the i-th output.
void build_signs(uint64_t state, int d, uint32_t* mask) {
  for (int w = 0; w < 8; ++w) mask[w] = 0;
  for (int i = 0; i < d; ++i) {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    if (z >> 63) mask[i >> 5] |= 1u << (i & 31);
  }
}

tq_status check_params(const tq_params* p) {
  if (!p) return fail(TQ_ERR_INVALID, "params is NULL");
  if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256)
    return fail(TQ_ERR_INVALID, "head_dim %d: supported values are 64, 128 and 256", p->head_dim);
  if (p->k_bits < 2 || p->k_bits > 4 || p->v_bits < 2 || p->v_bits > 4)
    return fail(TQ_ERR_INVALID, "k_bits=%d v_bits=%d: each must be 2, 3 or 4", p->k_bits,
                p->v_bits);
  if (p->qjl != 0 && p->qjl != 1) return fail(TQ_ERR_INVALID, "qjl must be 0 or 1");
  if (p->codebook != TQ_CODEBOOK_GAUSSIAN && p->codebook != TQ_CODEBOOK_SPHERE &&
      p->codebook != TQ_CODEBOOK_AFFINE)
    return fail(TQ_ERR_INVALID,
                "codebook %d: must be TQ_CODEBOOK_GAUSSIAN, TQ_CODEBOOK_SPHERE or TQ_CODEBOOK_AFFINE",
                p->codebook);
  return TQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tq_status check_cache(const tq_codebook* cb, const tq_cache* c) {
  if (!cb) return fail(TQ_ERR_INVALID, "codebook is NULL");
  if (!c) return fail(TQ_ERR_INVALID, "cache is NULL");
  if (c->batch <= 0 || c->kv_heads <= 0 || c->capacity <= 0)
    return fail(TQ_ERR_INVALID, "cache sizes must be positive (batch=%d kv_heads=%d capacity=%d)",
                c->batch, c->kv_heads, c->capacity);
  if (c->capacity % 16 != 0)
    return fail(TQ_ERR_INVALID, "capacity %d is not a multiple of 16", c->capacity);
  // the append, conversion and merge grids index batch rows by blockIdx.y
  if (c->batch > 65535) return fail(TQ_ERR_INVALID, "batch %d: at most 65535 rows", c->batch);
  const void* need[] = {c->k_codes, c->v_codes, c->k_norm, c->v_norm, c->seq_lens, c->status,
                        c->append_sync};
  const char* names[] = {"k_codes", "v_codes", "k_norm", "v_norm", "seq_lens", "status",
                         "append_sync"};
  for (int i = 0; i < 7; ++i) {
    if (!need[i]) return fail(TQ_ERR_INVALID, "cache.%s is NULL", names[i]);
    if (i < 4 && !aligned16(need[i]))
      return fail(TQ_ERR_INVALID, "cache.%s is not 16-byte aligned", names[i]);
  }
  if (cb->params.qjl) {
    if (!c->k_signs || !c->k_rnorm)
      return fail(TQ_ERR_INVALID, "QJL codebook needs cache.k_signs and cache.k_rnorm");
    if (!aligned16(c->k_signs) || !aligned16(c->k_rnorm))
      return fail(TQ_ERR_INVALID, "cache.k_signs / k_rnorm are not 16-byte aligned");
  }
  const double slots = (double)c->batch * c->kv_heads * c->capacity;
  if (slots * 128.0 > 9.0e18) return fail(TQ_ERR_INVALID, "cache too large");
  return TQ_OK;
}

tq::CacheView view_of(const tq_cache* c) {
  tq::CacheView v;
  v.k_codes = c->k_codes;
  v.v_codes = c->v_codes;
  v.k_signs = c->k_signs;
  v.k_norm = c->k_norm;
  v.v_norm = c->v_norm;
  v.k_rnorm = c->k_rnorm;
  v.seq_lens = c->seq_lens;
  v.status = c->status;
  v.append_sync = c->append_sync;
  v.batch = c->batch;
  v.kv_heads = c->kv_heads;
  v.capacity = c->capacity;
  return v;
}

tq_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace tq {
int record_error(int status, const char* message) {
  g_last_error = message;
  return status;
}
}  // namespace tq

extern "C" {

tq_status tq_codebook_init(const tq_params* params, tq_codebook** out, tq_layout* layout) {
  if (!out) return fail(TQ_ERR_INVALID, "out is NULL");
  *out = nullptr;
  tq_status st = check_params(params);
  if (st != TQ_OK) return st;
  tq_codebook* cb = new (std::nothrow) tq_codebook;
  if (!cb) return fail(TQ_ERR_NOMEM, "host allocation of the codebook failed");
  std::memset(cb, 0, sizeof *cb);
  cb->params = *params;
  tq::Tables& t = cb->tables;
  t.d = params->head_dim;
  t.k_bits = params->k_bits;
  t.v_bits = params->v_bits;
  t.qjl = params->qjl;
  const int kind = params->codebook, d = params->head_dim;
  t.affine = kind == TQ_CODEBOOK_AFFINE;
  if (t.affine) {
    build_affine_levels(params->k_bits, t.k_cent, t.k_bnd);
    build_affine_levels(params->v_bits, t.v_cent, t.v_bnd);
  } else if (!build_codebook(params->k_bits, kind, d, t.k_cent, t.k_bnd) ||
             !build_codebook(params->v_bits, kind, d, t.v_cent, t.v_bnd)) {
    delete cb;
    return fail(TQ_ERR_INVALID, "Lloyd-Max iteration did not converge");
  }
  t.k_lam = t.affine ? 1.0f : fp16_table_scale(t.k_cent, 1 << params->k_bits);
  t.v_lam = t.affine ? 1.0f : fp16_table_scale(t.v_cent, 1 << params->v_bits);
  build_signs(params->seed, params->head_dim, t.s1);
  build_signs(params->seed ^ 0x9E3779B97F4A7C15ull, params->head_dim, t.s2);
  if (layout) {
    layout->k_code_bytes = (size_t)params->k_bits * params->head_dim / 8;
    layout->v_code_bytes = (size_t)params->v_bits * params->head_dim / 8;
    layout->k_sign_bytes = params->qjl ? (size_t)params->head_dim / 8 : 0;
    layout->norm_halves = t.affine ? (size_t)2 * params->head_dim / tq::kAffineGroup : 1;
  }
  *out = cb;
  return ok();
}

tq_status tq_codebook_tables(const tq_codebook* cb, float* k_centroids, float* k_boundaries,
                             float* v_centroids, float* v_boundaries, int8_t* signs1,
                             int8_t* signs2) {
  if (!cb) return fail(TQ_ERR_INVALID, "codebook is NULL");
  const tq::Tables& t = cb->tables;
  const int lk = 1 << t.k_bits, lv = 1 << t.v_bits;
  if (k_centroids) std::memcpy(k_centroids, t.k_cent, sizeof(float) * lk);
  if (k_boundaries) std::memcpy(k_boundaries, t.k_bnd, sizeof(float) * (lk - 1));
  if (v_centroids) std::memcpy(v_centroids, t.v_cent, sizeof(float) * lv);
  if (v_boundaries) std::memcpy(v_boundaries, t.v_bnd, sizeof(float) * (lv - 1));
  for (int i = 0; i < t.d; ++i) {
    if (signs1) signs1[i] = ((t.s1[i >> 5] >> (i & 31)) & 1u) ? -1 : 1;
    if (signs2) signs2[i] = ((t.s2[i >> 5] >> (i & 31)) & 1u) ? -1 : 1;
  }
  return ok();
}

tq_status tq_quantize_append(const tq_codebook* cb, const tq_cache* cache, const void* k,
                             const void* v, tq_dtype dtype, int n_new, void* stream) {
  tq_status st = check_cache(cb, cache);
  if (st != TQ_OK) return st;
  if (n_new < 0) return fail(TQ_ERR_INVALID, "n_new %d is negative", n_new);
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (n_new == 0) return ok();
  if (!k || !v) return fail(TQ_ERR_INVALID, "k or v is NULL");
  if (n_new > cache->capacity)
    return fail(TQ_ERR_INVALID, "n_new %d exceeds capacity %d", n_new, cache->capacity);
  const size_t esz = dtype == TQ_F32 ? 4 : 2;
  const size_t vec_bytes = esz * cb->params.head_dim;
  if (((uintptr_t)k % vec_bytes) % 8 != 0 || ((uintptr_t)v % vec_bytes) % 8 != 0 ||
      !aligned16(k) || !aligned16(v))
    return fail(TQ_ERR_INVALID, "k and v must be 16-byte aligned");
  return cuda_status(tq::launch_quantize_append(cb->tables, view_of(cache), k, v, (int)dtype,
                                                n_new, (cudaStream_t)stream),
                     "quantize-append launch");
}

tq_status tq_quantize_cache(const tq_codebook* cb, const tq_cache* cache, const void* k,
                            const void* v, tq_dtype dtype, int64_t stride_b, int64_t stride_h,
                            int64_t stride_t, const int32_t* lengths, int max_len, void* stream) {
  tq_status st = check_cache(cb, cache);
  if (st != TQ_OK) return st;
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (max_len < 0) return fail(TQ_ERR_INVALID, "max_len %d is negative", max_len);
  if (max_len == 0) return ok();
  if (!k || !v || !lengths) return fail(TQ_ERR_INVALID, "k, v or lengths is NULL");
  if (stride_b < 0 || stride_h < 0 || stride_t < 0)
    return fail(TQ_ERR_INVALID, "negative stride");
  const int64_t esz = dtype == TQ_F32 ? 4 : 2;
  if ((stride_b * esz) % 16 || (stride_h * esz) % 16 || (stride_t * esz) % 16)
    return fail(TQ_ERR_INVALID, "strides (%lld, %lld, %lld) are not multiples of 16 bytes",
                (long long)stride_b, (long long)stride_h, (long long)stride_t);
  if (!aligned16(k) || !aligned16(v)) return fail(TQ_ERR_INVALID, "k and v must be 16-byte aligned");
  if ((uintptr_t)lengths % 4) return fail(TQ_ERR_INVALID, "lengths must be 4-byte aligned");
  return cuda_status(tq::launch_quantize_cache(cb->tables, view_of(cache), k, v, (int)dtype,
                                               stride_b, stride_h, stride_t, lengths, max_len,
                                               (cudaStream_t)stream),
                     "quantize-cache launch");
}

static tq_status check_weights(const tq_codebook* cb, int rows, int k, tq_dtype dtype) {
  if (!cb) return fail(TQ_ERR_INVALID, "codebook is NULL");
  if (cb->tables.affine)
    return fail(TQ_ERR_UNSUPPORTED, "the weights regime takes a Lloyd-Max codebook, not the affine codec");
  if (rows <= 0 || rows % 16) return fail(TQ_ERR_INVALID, "rows %d: a positive multiple of 16", rows);
  const int d = cb->params.head_dim;
  if (k <= 0 || k % d) return fail(TQ_ERR_INVALID, "k %d: a positive multiple of head_dim %d", k, d);
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_INVALID, "unknown dtype %d", (int)dtype);
  return TQ_OK;
}

tq_status tq_weights_quantize(const tq_codebook* cb, const void* w, tq_dtype dtype, int rows, int k,
                              uint8_t* codes, uint16_t* norms, void* stream) {
  tq_status st = check_weights(cb, rows, k, dtype);
  if (st != TQ_OK) return st;
  if (!w || !codes || !norms) return fail(TQ_ERR_INVALID, "w, codes or norms is NULL");
  if (!aligned16(w) || !aligned16(codes) || !aligned16(norms))
    return fail(TQ_ERR_INVALID, "w, codes and norms must be 16-byte aligned");
  return cuda_status(tq::launch_weights_quantize(cb->tables, w, (int)dtype, rows, k, codes, norms,
                                                 (cudaStream_t)stream),
                     "weights-quantize launch");
}

size_t tq_lut_matmul_workspace_bytes(const tq_codebook* cb, int rows, int k, int m) {
  if (!cb || rows <= 0 || rows % 16 || k <= 0 || k % cb->params.head_dim || m <= 0) return 0;
  return tq::lut_matmul_workspace_bytes(tq::plan_lut_matmul(rows, k, m, cb->params.head_dim, tq::kLutMatmulMaxCtas), rows, m);
}

tq_status tq_lut_matmul(const tq_codebook* cb, const uint8_t* codes, const uint16_t* norms, int rows,
                        int k, const void* x, tq_dtype dtype, int m, float* y, void* workspace,
                        size_t workspace_bytes, void* stream) {
  tq_status st = check_weights(cb, rows, k, dtype);
  if (st != TQ_OK) return st;
  if (m <= 0 || m > 65535 * 4) return fail(TQ_ERR_INVALID, "m %d out of range", m);
  if (!codes || !norms || !x || !y) return fail(TQ_ERR_INVALID, "codes, norms, x or y is NULL");
  if (!aligned16(codes) || !aligned16(norms) || !aligned16(x) || !aligned16(y))
    return fail(TQ_ERR_INVALID, "codes, norms, x and y must be 16-byte aligned");
  const size_t need =
      tq::lut_matmul_workspace_bytes(tq::plan_lut_matmul(rows, k, m, cb->params.head_dim, tq::kLutMatmulMaxCtas), rows, m);
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(TQ_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  if (need > 0 && !aligned16(workspace)) return fail(TQ_ERR_INVALID, "workspace must be 16-byte aligned");
  return cuda_status(tq::launch_lut_matmul(cb->tables, codes, norms, rows, k, x, (int)dtype, m, y,
                                           (float*)workspace, (cudaStream_t)stream),
                     "lut-matmul launch");
}

size_t tq_decode_workspace_bytes(const tq_codebook* cb, int batch, int q_heads, int kv_heads,
                                 int max_ctx) {
  if (!cb || batch <= 0 || q_heads <= 0 || kv_heads <= 0 || max_ctx < 0 ||
      q_heads % kv_heads != 0)
    return 0;
  const tq::DecodePlan plan = tq::plan_decode(batch, kv_heads, max_ctx, tq::kMaxTargetCtas);
  return tq::decode_workspace_bytes(plan, q_heads, kv_heads, cb->params.head_dim);
}

tq_status tq_decode_attention(const tq_codebook* cb, const tq_cache* cache, const void* q,
                              tq_dtype dtype, int q_heads, float softmax_scale, int max_ctx,
                              float* out, void* workspace, size_t workspace_bytes,
                              void* stream) {
  tq_status st = check_cache(cb, cache);
  if (st != TQ_OK) return st;
  if (!q || !out) return fail(TQ_ERR_INVALID, "q or out is NULL");
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (q_heads <= 0 || q_heads % cache->kv_heads != 0)
    return fail(TQ_ERR_INVALID, "q_heads %d is not a positive multiple of kv_heads %d", q_heads,
                cache->kv_heads);
  if (max_ctx < 0 || max_ctx > cache->capacity)
    return fail(TQ_ERR_INVALID, "max_ctx %d outside [0, capacity %d]", max_ctx, cache->capacity);
  if (!aligned16(q) || !aligned16(out))
    return fail(TQ_ERR_INVALID, "q and out must be 16-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(TQ_ERR_INVALID, "softmax_scale is not finite");
  const int d = cb->params.head_dim;
  const int group = q_heads / cache->kv_heads;
  if (!tq::decode_supported(d, group, cb->params.k_bits, cb->params.v_bits, cb->params.qjl))
    return fail(TQ_ERR_UNSUPPORTED,
                "no decode kernel for head_dim=%d group=%d k_bits=%d v_bits=%d qjl=%d "
                "(group must be 1, 2, 4 or 8; v_bits must be k_bits or k_bits + 1)",
                d, group, cb->params.k_bits, cb->params.v_bits, cb->params.qjl);
  const tq::DecodePlan plan = tq::plan_decode(cache->batch, cache->kv_heads, max_ctx, tq::kMaxTargetCtas);
  const size_t need = tq::decode_workspace_bytes(plan, q_heads, cache->kv_heads, d);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(TQ_ERR_CAPACITY, "workspace of %zu bytes is smaller than the %zu needed",
                workspace_bytes, need);
  if (need > 0 && !aligned16(workspace))
    return fail(TQ_ERR_INVALID, "workspace must be 16-byte aligned");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  return cuda_status(tq::launch_decode(cb->tables, view_of(cache), q, (int)dtype, q_heads, scale,
                                       max_ctx, out, (float*)workspace, (cudaStream_t)stream),
                     "decode launch");
}

void tq_free(tq_codebook* cb) { delete cb; }

const char* tq_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
