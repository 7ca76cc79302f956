/*
 * tq.h -- C ABI of libtq: the TurboQuant KV-cache codec and the fused decode
 * attention that reads it, for NVIDIA B200 (sm_100a).
 *
 * What the operations are (cited by page title and section):
 *  - "TurboQuant Performance Benefits: Memory Reduction and Speed Optimization
 *    in MLX-VLM", sections "What Is TurboQuant?" and "Fractional-Bit Precision
 *    Support": KV vectors are rotated with a random Hadamard transform, then
 *    quantized with an MSE codebook to 2-4 bits per dimension; 3.5 bits means
 *    3-bit keys and 4-bit values.
 *  - same page, "Custom Metal Kernel Implementation": attention scores and the
 *    value aggregation are computed directly on the packed codes during decode,
 *    without dequantizing the cache.
 *  - "How to Use TurboQuant with the MLX-VLM Python API: A Complete Guide",
 *    section "What is TurboQuant?": the rotation helpers (_rotation_matrix,
 *    _rht_forward, _rht_inverse) and the codebook generator (_codebook).
 *  - "mlx-turboquant" README, section "The 1-bit QJL residual (unbiased
 *    inner-product estimator)": keys may carry sign(RHT2(r)) and ||r|| of the
 *    residual r = Rk - k_hat; the score adds
 *    sqrt(pi/(2d)) * ||r|| * <RHT2(Rq), sign(RHT2(r))>.
 *  - same README, "Quantize the KV cache (long-context inference)" and "How
 *    it plugs in": the affine group-64 cache with rotated keys, built here as
 *    a comparison codec (TQ_CODEBOOK_AFFINE) on the same kernels.
 *
 * Conventions shared by every call:
 *  - Pointers are plain host or device addresses as stated per argument; the
 *    library never takes ownership of caller memory and never allocates device
 *    memory.  The only object it allocates is the host-side tq_codebook.
 *    The library checks device pointers for NULL and alignment only: it does
 *    not ask the driver whether an address is device memory (that would cost
 *    a runtime call per pointer on every launch), so a host address passed
 *    where device memory is required reaches the kernels and faults there.
 *    Callers check placement (the Python binding does, before each call).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Device work is enqueued on it and the call returns; results are
 *    visible after the caller synchronizes that stream.
 *  - A call that returns a status other than TQ_OK enqueued nothing, except
 *    TQ_ERR_CUDA from a launch, which reports a failed launch.
 *    tq_last_error() then describes the problem (thread-local string).
 *  - Errors found on the device (a sequence that would pass the cache
 *    capacity, a context longer than the decode call was sized for) never trap
 *    and never wait: the kernel skips the affected work and ORs a TQ_FLAG_*
 *    bit into *cache->status, which the caller reads after synchronizing.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID = 1,      /* bad argument: null pointer, size, alignment   */
  TQ_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, bits, group    */
  TQ_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed          */
  TQ_ERR_CAPACITY = 4,     /* workspace too small                           */
  TQ_ERR_NOMEM = 5         /* host allocation failed                        */
} tq_status;

/* Sticky device-side flags ORed into *tq_cache.status. */
#define TQ_FLAG_CAPACITY 1u  /* an append would pass `capacity`: that batch row was skipped */
#define TQ_FLAG_MAXCTX 2u    /* a sequence was longer than the decode's max_ctx: its tail was not attended */
#define TQ_FLAG_LAYOUT 4u    /* the decode kernel found its shared memory placed other than the host
                                checked (never expected on sm_100a): its outputs are not valid */

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* Codebook choices (tq_params.codebook).
 *   TQ_CODEBOOK_GAUSSIAN : Lloyd-Max quantizer of N(0, 1), the pages' reading
 *       of the rotated coordinates as near-Gaussian ("How to Use TurboQuant
 *       ...", "What is TurboQuant?": _codebook; "mlx-turboquant" README).
 *   TQ_CODEBOOK_SPHERE : Lloyd-Max quantizer of their exact distribution: for a
 *       fixed x, sqrt(d) (R x)_i / ||x|| is sqrt(d) times a coordinate of a
 *       uniformly random unit vector of R^d, with density proportional to
 *       (1 - z^2/d)^((d-3)/2) on |z| < sqrt(d); it depends on head_dim and
 *       tends to N(0, 1) as head_dim grows.
 *   TQ_CODEBOOK_AFFINE : the comparison codec of the "mlx-turboquant" README
 *       ("Quantize the KV cache (long-context inference)", kv_group_size 64;
 *       "How it plugs in": an affine quantized cache whose keys are rotated).
 *       Keys are coded in the rotated frame y = R k, values as they are.  Per
 *       group of 64 consecutive channels, scale = (max - min) / (2^bits - 1)
 *       and bias = min, both fp16; a channel's code is round((y - bias) / scale),
 *       ties to even, clamped to [0, 2^bits - 1] (0 when scale is 0), and
 *       y_hat = scale * code + bias.  With qjl the key sketch codes the
 *       residual y - y_hat as for the other codebooks.  The tables hold the
 *       integer levels 0 .. 2^bits - 1 (centroids) and their midpoints.
 *       Inputs are expected to be finite. */
#define TQ_CODEBOOK_GAUSSIAN 0
#define TQ_CODEBOOK_SPHERE 1
#define TQ_CODEBOOK_AFFINE 2

/* Codec parameters.
 *   head_dim : d, 64, 128 or 256
 *   k_bits, v_bits : code widths in {2, 3, 4} ("3.5 bits" = 3 and 4)
 *   qjl      : 1 = keys also carry the 1-bit QJL residual sketch
 *   seed     : seeds the sign vectors of R (and of R2 = RHT2 for QJL).  One R
 *              is shared by keys, values, all heads and all batch rows.
 *   codebook : TQ_CODEBOOK_GAUSSIAN (0, the default when zero-initialized),
 *              TQ_CODEBOOK_SPHERE or TQ_CODEBOOK_AFFINE. */
typedef struct {
  int head_dim;
  int k_bits;
  int v_bits;
  int qjl;
  uint64_t seed;
  int codebook;
} tq_params;

/* Bytes stored per cached vector, in each per-vector array of tq_cache. */
typedef struct {
  size_t k_code_bytes;   /* k_bits * head_dim / 8 */
  size_t v_code_bytes;   /* v_bits * head_dim / 8 */
  size_t k_sign_bytes;   /* head_dim / 8 with QJL, else 0 */
  size_t norm_halves;    /* fp16 entries per vector in k_norm and v_norm: 1 (the
                            norm), or 2 * head_dim / 64 for TQ_CODEBOOK_AFFINE
                            (scale, bias of each group, in channel order) */
} tq_layout;

typedef struct tq_codebook tq_codebook;  /* opaque, host memory, owned by the library */

/* The compressed cache: caller-owned DEVICE memory (e.g. torch tensors).
 * Row r = b * kv_heads + h of every per-vector array holds `capacity` slots;
 * slot t is token t of batch row b, KV head h.
 *   k_codes : uint8 [batch][kv_heads][capacity][k_code_bytes]
 *   v_codes : uint8 [batch][kv_heads][capacity][v_code_bytes]
 *   k_signs : uint8 [batch][kv_heads][capacity][k_sign_bytes] (QJL only, else NULL)
 *   k_norm, v_norm : fp16 bit patterns [batch][kv_heads][capacity][norm_halves]
 *                    (||x||; or the affine codec's (scale, bias) pairs)
 *   k_rnorm : fp16 bit patterns [batch][kv_heads][capacity] (QJL ||Rk - k_hat||, else NULL)
 *   seq_lens : int32 [batch], tokens currently stored per batch row
 *   status   : one int32, sticky TQ_FLAG_* bits (caller clears it)
 *   append_sync : int32 [batch], zero before the first append; every
 *                 tq_quantize_append leaves it zero again
 * Packed code layout of one vector: a little-endian bit stream in which
 * channel i's b-bit code occupies bits [b*i, b*i + b), bit 0 being the least
 * significant bit of byte 0; the sign plane is the same stream with b = 1.
 * capacity must be a multiple of 16 and batch at most 65535.  Every pointer
 * must be 16-byte aligned. */
typedef struct {
  uint8_t *k_codes, *v_codes, *k_signs;
  uint16_t *k_norm, *v_norm, *k_rnorm;
  int32_t *seq_lens;
  int32_t *status;
  int32_t *append_sync;
  int batch, kv_heads, capacity;
} tq_cache;

/* Builds the codebooks and rotation signs for `params` (host work only: no
 * GPU is needed).  Codebook: the Lloyd-Max MSE quantizer with 2^bits levels of
 * N(0, 1) or of the exact rotated-coordinate distribution (params->codebook),
 * solved in double precision, made exactly odd-symmetric and rounded to
 * float32; boundaries are the float32 midpoints of adjacent centroids ("How
 * to Use TurboQuant ...", "What is TurboQuant?": _codebook).
 * Signs: channel i of D1 is -1 when the top bit of the i-th SplitMix64 output
 * from state `seed` is set; D2 uses state seed ^ 0x9E3779B97F4A7C15.
 * On success *out owns the tables (release with tq_free) and *layout, if not
 * NULL, receives the per-vector byte counts. */
tq_status tq_codebook_init(const tq_params* params, tq_codebook** out, tq_layout* layout);

/* Copies the tables of `cb` into caller HOST buffers (any may be NULL):
 * k_centroids[2^k_bits], k_boundaries[2^k_bits - 1], v_centroids[2^v_bits],
 * v_boundaries[2^v_bits - 1], signs1[head_dim], signs2[head_dim] (+1/-1). */
tq_status tq_codebook_tables(const tq_codebook* cb, float* k_centroids, float* k_boundaries,
                             float* v_centroids, float* v_boundaries,
                             int8_t* signs1, int8_t* signs2);

/* Quantizes n_new new tokens per batch row and appends them at slots
 * [seq_lens[b], seq_lens[b] + n_new), then adds n_new to seq_lens[b].
 * k, v : DEVICE, dtype `dtype`, contiguous [batch][kv_heads][n_new][head_dim].
 * Per vector x (fp32 arithmetic, fixed operation order, see the pages' codec):
 *   n = ||x|| (pairwise sum of squares, correctly rounded sqrt), stored fp16;
 *   u = H (s1 * x) (unnormalized Walsh-Hadamard, Sylvester order);
 *   z = u * (1/n) (0 when n == 0);  code_i = #{j : boundary_j < z_i};
 *   QJL keys: r = u - fp16(n) * c[code]; ||r||/sqrt(d) stored fp16;
 *             sign bit_i = (H (s2 * r))_i >= 0.
 * TQ_CODEBOOK_AFFINE instead (same rounding discipline):
 *   y = u * fp32(1 / fp32(sqrt(d))) for keys, y = x for values; per group of
 *   64 channels (min and max as values, a zero extreme being +0)
 *   scale = fp16((max y - min y) / (2^b - 1)), bias = fp16(min y),
 *   code_i = rint((y_i - bias) / scale) clamped (0 when scale == 0);
 *   QJL keys: r = y - (scale * code + bias); ||r|| stored fp16; sign bits as above.
 * A batch row whose append would pass `capacity` is skipped and sets
 * TQ_FLAG_CAPACITY.  n_new == 0 is a no-op.  NaN/Inf inputs are undefined; a
 * norm above 65504 stores an infinite fp16 norm. */
tq_status tq_quantize_append(const tq_codebook* cb, const tq_cache* cache, const void* k,
                             const void* v, tq_dtype dtype, int n_new, void* stream);

/* Converts an existing dense K/V cache into the compressed one: the prefill of
 * a whole context at once, or the conversion of a cache filled by an
 * unquantized model ("How to Use TurboQuant with the MLX-VLM Python API",
 * "What is TurboQuant?": a filled KVCache is converted by from_cache).  Every
 * vector goes through the same codec as tq_quantize_append.
 * k, v : DEVICE, dtype `dtype`; element (b, h, t, i) of k is
 *        k[b*stride_b + h*stride_h + t*stride_t + i] (strides in elements,
 *        the channel stride is 1; v uses the same strides), so both
 *        [batch][kv_heads][T][d] and [batch][T][kv_heads][d] caches are read in
 *        place.  Every stride times the element size must be a multiple of 16
 *        bytes, and k and v 16-byte aligned.
 * lengths : DEVICE int32 [batch], tokens of row b to convert (t < lengths[b]).
 * max_len : host upper bound of every lengths[b] (it sizes the grid).
 * Row b's slots [0, lengths[b]) are overwritten and seq_lens[b] is set to
 * lengths[b] (earlier contents of the row are discarded).  A row longer than
 * `capacity` is skipped and sets TQ_FLAG_CAPACITY; a length above max_len
 * converts the first max_len tokens and sets TQ_FLAG_MAXCTX; a negative
 * length counts as 0.  No counterpart of append_sync is used. */
tq_status tq_quantize_cache(const tq_codebook* cb, const tq_cache* cache, const void* k,
                            const void* v, tq_dtype dtype, int64_t stride_b, int64_t stride_h,
                            int64_t stride_t, const int32_t* lengths, int max_len, void* stream);

/* Workspace bytes tq_decode_attention needs for these sizes (0 on bad sizes).
 * Size workspaces by calling this function: the figure follows the decode
 * kernel's grid and may change with the library version.  For information,
 * this version returns (min(592, U * ceil(max_ctx / 64)) + U - 1) *
 * (q_heads / kv_heads) * (head_dim + 2) * 4 with U = batch * kv_heads: one
 * partial result per (CTA, unit) the work partition can produce, for grids of
 * at most 592 CTAs (4 per SM on 148 SMs).  It depends on the sizes alone, so
 * one workspace serves every call (and every captured graph) of those sizes. */
size_t tq_decode_workspace_bytes(const tq_codebook* cb, int batch, int q_heads, int kv_heads,
                                 int max_ctx);

/* Decode attention of one new query per head over the compressed cache.
 * q   : DEVICE, dtype `dtype`, [batch][q_heads][head_dim]; query head h reads
 *       KV head h / (q_heads / kv_heads).
 * out : DEVICE float32 [batch][q_heads][head_dim].
 * softmax_scale <= 0 selects 1/sqrt(head_dim).
 * max_ctx : host upper bound of every seq_lens[b] (at most capacity); it
 *       bounds the work partition and the workspace.  Tokens past it are not
 *       attended and set TQ_FLAG_MAXCTX.  The partition itself is computed on
 *       the device from seq_lens: every CTA takes an equal share of the token
 *       tiles of all (batch row, KV head) pairs, so ragged batches stay
 *       balanced.
 * workspace : DEVICE scratch of at least
 *       tq_decode_workspace_bytes(cb, batch, q_heads, kv_heads, max_ctx) bytes
 *       (TQ_ERR_CAPACITY otherwise); it holds the partial results.  Its
 *       contents need no initialization.
 * Computes, for every (b, h), over tokens t < seq_lens[b]:
 *   s_t = scale * (<Rq, n_t c_K[code_t]/sqrt(d)>
 *                  + sqrt(pi/(2d)) * rho_t * <R2 R q, 2 bit_t - 1>)   (QJL term if enabled)
 *   out = R^T (sum_t softmax(s)_t * m_t c_V[vcode_t] / sqrt(d)),
 * and with TQ_CODEBOOK_AFFINE, y_hat = scale * code + bias of each group:
 *   s_t = scale * (<Rq, k_hat_t> + the same QJL term),  out = sum_t softmax(s)_t v_hat_t
 * (values are not rotated), never writing a dequantized cache.  seq_lens[b] == 0 gives zeros.  The
 * result is deterministic (fixed-order merge of the splits). */
tq_status tq_decode_attention(const tq_codebook* cb, const tq_cache* cache, const void* q,
                              tq_dtype dtype, int q_heads, float softmax_scale, int max_ctx,
                              float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Decode attention exactly like tq_decode_attention, for callers that cannot
 * allocate device memory (and so cannot provide a workspace): for example a
 * runtime whose device memory is reserved up front and managed by its own
 * pool, a plugin that only receives input and output pointers from its host,
 * or code that must not call cudaMalloc because an allocation can synchronize
 * the device or fail at an unpredictable time.  The paper has no counterpart;
 * this is a library-usability entry point.
 *   - The per-split scratch lives in a static 8 MiB device array compiled into
 *     the library; every GPU that loads the library holds it until the process
 *     exits.  Nothing is allocated: no cudaMalloc, cudaFree or allocating
 *     library routine is called.
 *   - A decode whose scratch (tq_decode_workspace_bytes for the same sizes)
 *     exceeds 8 MiB is rejected with TQ_ERR_CAPACITY and enqueues nothing.
 *   - Every call looks up the array's address in the current context (no
 *     allocation), so a reset of the context (cudaDeviceReset) needs nothing
 *     special; the first call on a device loads the array's module, so make
 *     it before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (every partial is written before
 *     it is read), but calls that overlap on the GPU (different streams, or
 *     different threads without ordering) race on it: serialize them.
 * Arguments, semantics and errors are otherwise those of tq_decode_attention. */
tq_status tq_decode_attention_noalloc(const tq_codebook* cb, const tq_cache* cache, const void* q,
                                      tq_dtype dtype, int q_heads, float softmax_scale,
                                      int max_ctx, float* out, void* stream);

/* Weights regime ("mlx-turboquant" README, introduction: "Weights (MSE
 * regime)", rotate each weight matrix, then quantize; "The Metal kernels"
 * item 1: LUT dequant + matmul directly on packed indices).  Each row of a
 * weight matrix W [rows][k] is cut into k / head_dim blocks of head_dim input
 * channels, and every block is encoded exactly as a key vector is (fp16 norm,
 * rotation, k_bits Lloyd-Max codes; the codebook's QJL setting is ignored).
 *
 * tq_weights_quantize: w DEVICE [rows][k] of `dtype`, 16-byte aligned;
 *   codes DEVICE uint8 [k / head_dim][rows][k_bits * head_dim / 8];
 *   norms DEVICE fp16 bits [k / head_dim][rows]; both 16-byte aligned.
 *   rows must be a multiple of 16 and k a multiple of head_dim.
 *   A TQ_CODEBOOK_AFFINE codebook is rejected (TQ_ERR_UNSUPPORTED) by this
 *   call and by tq_lut_matmul. */
tq_status tq_weights_quantize(const tq_codebook* cb, const void* w, tq_dtype dtype, int rows, int k,
                              uint8_t* codes, uint16_t* norms, void* stream);

/* Workspace bytes tq_lut_matmul needs for these sizes (0 when it needs none,
 * or on bad sizes).  The matmul splits the k blocks over CTAs when rows x m
 * alone give too few, and the workspace holds the per-split partial sums:
 * splits * m * rows * 4 bytes. */
size_t tq_lut_matmul_workspace_bytes(const tq_codebook* cb, int rows, int k, int m);

/* Y = X W_hat^T on the codes of tq_weights_quantize, never forming W_hat:
 *   y[i][n] = sum_j (norm_{n,j} / sqrt(d)) <centroid[codes_{n,j}], R x_{i,j}>
 * with x_{i,j} block j of input row i and R the codebook's rotation.
 * x DEVICE [m][k] of `dtype`; y DEVICE float32 [m][rows]; workspace DEVICE of
 * at least tq_lut_matmul_workspace_bytes (TQ_ERR_CAPACITY otherwise; NULL
 * when that is 0).  All 16-byte aligned.  The result is deterministic: the
 * split partials are added in a fixed order. */
tq_status tq_lut_matmul(const tq_codebook* cb, const uint8_t* codes, const uint16_t* norms, int rows,
                        int k, const void* x, tq_dtype dtype, int m, float* y, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Releases a codebook (NULL is ignored). */
void tq_free(tq_codebook* cb);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* tq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
