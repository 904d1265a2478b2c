/*
 * tq.h -- C ABI of the TurboQuant KV-cache library for NVIDIA B200 (sm_100a).
 *
 * The library implements the data-parallel hot path of TurboQuant as the
 * pages describe it: a seeded random rotation, a per-block norm, Lloyd-Max
 * scalar quantization of every rotated coordinate to 2/3/4-bit indices with
 * bit packing, an optional QJL stage that keeps the sign of a Gaussian
 * projection of the residual, and decode attention that reads the packed
 * cache directly.
 *
 * Sources (page title, section):
 *   [G] "TurboQuant+ upstream guide: llama.cpp KV cache compression, 4-phase
 *       PR roadmap" -- sec. 3 finding 6 (seeded rotation, QR -> Haar,
 *       det = +1), sec. 4 (dense rotation vs D1 @ H @ D2), sec. 5.1 (MSE-only
 *       PolarQuant, block 32, per-block norm), sec. 5.2 (block struct,
 *       centroid table, CPU quantize/dequantize), sec. 5.3 (pre-rotated
 *       queries, fp16 centroid LUT, float norm broadcast), sec. 5.4
 *       (turbo2/turbo4, asymmetric K/V), sec. 6.1 (inverse-rotation fix).
 *   [O] "Plan de Integracion: TurboQuant en Orion" -- "Implementacion
 *       conceptual" (one sign bit per residual value).
 *   [T] "Google TurboQuant deep dive" -- sec. 2.2 (QJL: Gaussian projection
 *       of the residual, sign binarisation, full-precision query),
 *       sec. 4.2 (JL lemma), sec. 4.3 (softmax(Q K^T / sqrt(d)) V).
 *
 * Conventions (all entry points):
 *   - Fixed-width integers in every signature.  Enum values carry the enum
 *     prefix.  No torch or CUDA types appear: a CUDA stream is passed as
 *     `void *` (a cudaStream_t; NULL = the legacy default stream).
 *   - "device" pointers must be device-accessible memory of the CURRENT CUDA
 *     device; "host" pointers are ordinary CPU memory.  The caller owns every
 *     buffer it passes; the library only reads or writes it during the call's
 *     stream work.  The library allocates device memory only inside
 *     tq_make_rotation (released by tq_free_rotation).
 *   - No call synchronises the device.  Errors that the host can detect
 *     (null pointers, unsupported sizes, misalignment, too small a
 *     workspace) are returned before anything is launched.  A failed launch
 *     returns TQ_ERR_CUDA.  tq_last_error() gives a one-line reason for the
 *     last failure on the calling thread.
 *   - Cache rows are ordered [batch][kv_head][token]; one row is one token of
 *     one KV head.  Queries are [batch][q_head][head_dim]; q_head h reads
 *     kv_head h / (n_q_heads / n_kv_heads).
 *   - Supported: head_dim in {64, 128, 256}; bits in {2, 3, 4}; block in
 *     {32, 64, 128} (block <= head_dim; [G] sec. 5.2 reports block 128 at
 *     5.12x); QJL projection rows m in {32, 64, ..., 256} with block 32.
 *     Block 32 with fp16 norms runs on the tensor-core kernels; the other
 *     block sizes and fp32 norms on CUDA-core kernels.
 *   - Device-detected conditions are OR-ed into the caller's `status_dev`
 *     word (may be NULL): TQ_STATUS_NORM_SATURATED when a norm exceeded the
 *     fp16 range and was stored as 65504, TQ_STATUS_NONFINITE when an input
 *     value was NaN or infinite, TQ_STATUS_TIMEOUT when a bounded wait for
 *     tensor-core work gave up (the affected rows are then not written).
 *     Kernels never trap.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Version of the packed cache layout described at tq_quantize_kv. */
#define TQ_FORMAT_VERSION 1

/*
 * Format flags of the _ex entry points (0 = the default format: fp16 norms).
 *   TQ_FMT_NORM_F32:       block norms stored as IEEE fp32 (4 bytes each)
 *                          instead of fp16.  With 4-bit codes and block 128
 *                          this is 4 + 32/128 = 4.25 bits per value, the
 *                          turbo4 figure of [G] sec. 1.2 (reading taken here).
 *   TQ_FMT_NORM_CORRECTED: the stored norm is ||y_blk|| / ||c[idx_blk]||, so
 *                          the dequantized block has the rotated block's own
 *                          norm up to the storage rounding ("norm correction",
 *                          [G] sec. 11); codes are unchanged and readers need
 *                          no flag for it.
 */
#define TQ_FMT_NORM_F32 1u
#define TQ_FMT_NORM_CORRECTED 2u
/*
 *   TQ_FMT_GROUPED:        lane-grouped code order inside each row (head_dim
 *                          128, block 32, fp16 norms): the row's bit stream
 *                          holds the codes of coordinates 4g .. 4g+3 of block
 *                          0, then of block 1, 2, 3, then the same for group
 *                          g + 1; code (block b, coordinate 4g + e) starts at
 *                          bit bits * (4 * (4g + b) + e).  Same bits per row
 *                          as the default order, only moved: the decode lane
 *                          that owns coordinates 4g .. 4g+3 of every block
 *                          reads its 16 * bits bits of a token with one or two
 *                          loads instead of two per block.  Written by
 *                          tq_quantize_kv_ex (bf16 rows, no QJL, no other
 *                          flag); read by tq_decode_attention_ex as the layout
 *                          of the VALUE codes (key codes always use the
 *                          default order; tq_attn_logits_ex rejects it).  The
 *                          pages fix no byte layout; this is the library's.
 */
#define TQ_FMT_GROUPED 4u

#define TQ_STATUS_NORM_SATURATED 1u
#define TQ_STATUS_NONFINITE 2u
#define TQ_STATUS_TIMEOUT 4u   /* a bounded wait inside a kernel gave up */

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,
    TQ_ERR_UNSUPPORTED = 2,
    TQ_ERR_CUDA = 3,
    TQ_ERR_ALLOC = 4
} tq_status;

typedef enum tq_rot_kind {
    TQ_ROT_WHT = 0,   /* R = d^-1/2 * D1 * H * D2 (square, d x d)            */
    TQ_ROT_HAAR = 1,  /* Haar orthogonal, det = +1 (square, d x d)           */
    TQ_ROT_GAUSS = 2  /* QJL projection S, rows x cols, i.i.d. N(0, 1)       */
} tq_rot_kind;

typedef enum tq_dtype {
    TQ_DTYPE_F32 = 0,
    TQ_DTYPE_BF16 = 1
} tq_dtype;

typedef struct tq_rotation tq_rotation; /* opaque; owns its device copy */

/*
 * tq_rotation_generate -- write the dense rows x cols matrix of a seeded
 * rotation (or projection) into host memory `out` (row-major float64).
 * Host only; needs no GPU.  [G] sec. 3 finding 6 and sec. 4.
 *
 * Random stream: SplitMix64 started at `seed` (the pages name no generator);
 * signs = top bit of a draw (set -> -1); uniforms = (draw >> 11) * 2^-53;
 * normals = Box-Muller on uniform pairs (u1 -> 1 - u1), cos output first.
 *   TQ_ROT_WHT:   rows == cols == d (power of two).  D1 = first d signs,
 *                 D2 = next d signs, H[i][j] = (-1)^popcount(i & j).
 *   TQ_ROT_HAAR:  rows == cols == d.  G[i][j] = normal i*d + j; G = QR by
 *                 Householder; Q <- Q diag(sign(diag R)); if det Q < 0 the
 *                 first column is negated.  y = Q x.
 *   TQ_ROT_GAUSS: S[i][j] = normal i*cols + j.
 * Returns TQ_ERR_INVALID_ARG for a null `out` or unsupported sizes.
 */
tq_status tq_rotation_generate(tq_rot_kind kind, int32_t rows, int32_t cols, uint64_t seed,
                               double * out);

/*
 * tq_make_rotation -- generate the matrix above and upload the forms the
 * kernels use to the current device: signs (WHT), fp32 plus bf16 hi/lo
 * splits (HAAR, GAUSS).  `*out` receives a handle owned by the caller and
 * released with tq_free_rotation.  Synchronous (one host-to-device copy).
 * Returns TQ_ERR_ALLOC if device memory cannot be allocated.
 */
tq_status tq_make_rotation(tq_rot_kind kind, int32_t rows, int32_t cols, uint64_t seed,
                           tq_rotation ** out);

/* Release a handle from tq_make_rotation (NULL is ignored). */
void tq_free_rotation(tq_rotation * rot);

/* Copy the handle's float64 matrix (rows x cols, row-major) to host `out`. */
tq_status tq_rotation_copy_host(const tq_rotation * rot, double * out);

/* Kind, rows, cols and seed of a handle (any output pointer may be NULL). */
tq_status tq_rotation_info(const tq_rotation * rot, int32_t * kind, int32_t * rows,
                           int32_t * cols, uint64_t * seed);

/*
 * tq_build_codebook -- Lloyd-Max codebook for `bits` in {1..4} and a block of
 * `block` coordinates (block >= 3).  Host only.  [G] sec. 1.2 / 5.2
 * (Lloyd-Max codebook, centroid table).
 *
 * The fitted density is that of one coordinate of a uniform point on the
 * sphere S^(block-1) -- a rotated block divided by its norm -- i.e.
 * f(x) = (1 - x^2)^((block-3)/2) / B(1/2, (block-1)/2) on [-1, 1].
 * Iterates the centroid / midpoint conditions in float64 until no centroid
 * moves by 1e-14.  The reconstruction table is stored at fp16 precision, as
 * in the upstream GPU path's fp16 centroid lookup table ([G] sec. 5.3, the
 * Metal backend's "fp16 centroid LUT"); the decision boundaries keep the
 * float64 fixed point.
 *   centroids:  host, 2^bits floats, ascending; each the binary16 value
 *               nearest (ties to even) to the float64 centroid, so exactly
 *               representable in fp16.
 *   boundaries: host, 2^bits - 1 floats, the float64 midpoints of adjacent
 *               (unrounded) centroids rounded to fp32.
 */
tq_status tq_build_codebook(int32_t bits, int32_t block, float * centroids, float * boundaries);

/* uint32 words of packed codes per row: (head_dim / block) * bits * block / 32. */
int64_t tq_code_words_per_row(int32_t bits, int32_t block, int32_t head_dim);

/*
 * tq_quantize_kv -- quantize n_rows cache rows on `stream`.  [G] sec. 5.1,
 * 5.2; QJL: [T] sec. 2.2, [O].
 *
 *   rot:        WHT or HAAR handle, head_dim x head_dim.
 *   bits, block, centroids, boundaries: the codebook (host pointers, as
 *               returned by tq_build_codebook; read during the call only).
 *   qjl:        NULL for MSE-only; else a GAUSS handle of m x head_dim.
 *   x:          device, [n_rows][head_dim] of `dtype`, row-major, 16-byte
 *               aligned.
 * Outputs (device, caller-allocated):
 *   codes:      uint32 [n_rows][tq_code_words_per_row(...)], 16-byte aligned.
 *               Per row and per block k the block owns bits*block/32
 *               consecutive words; code j of the block fills bits
 *               [j*bits, j*bits + bits) of their little-endian bit stream.
 *               code = #{i : u_j >= t_i}, u = y_blk / ||y_blk||, y = R x;
 *               a zero block stores 2^(bits-1) everywhere.
 *   norms:      fp16 bits [n_rows][head_dim / block], ||y_blk|| rounded to
 *               nearest even, saturated at 65504.
 *   qjl_signs:  (QJL only) uint32 [n_rows][m / 32]; bit i = [(S r)_i >= 0],
 *               r = y - fp16(norm) * c[code] in the rotated frame.
 *   qjl_rnorm:  (QJL only) fp16 bits [n_rows], ||r||.
 *   status_dev: device uint32 or NULL (see TQ_STATUS_*).
 * n_rows == 0 is a no-op returning TQ_OK.  Codes have the same layout for
 * every block size (a block of 64 / 128 owns the words of its 32-coordinate
 * pieces in order); the block size only changes the norm, the codebook
 * (tq_build_codebook(bits, block)) and u = y_blk / ||y_blk||.
 */
tq_status tq_quantize_kv(const tq_rotation * rot, int32_t bits, int32_t block,
                         const float * centroids, const float * boundaries,
                         const tq_rotation * qjl,
                         const void * x, tq_dtype dtype, int64_t n_rows, int32_t head_dim,
                         uint32_t * codes, uint16_t * norms,
                         uint32_t * qjl_signs, uint16_t * qjl_rnorm,
                         uint32_t * status_dev, void * stream);

/*
 * tq_quantize_kv_ex -- tq_quantize_kv with format flags (TQ_FMT_*).  `norms`
 * is fp16 bits, or fp32 with TQ_FMT_NORM_F32, [n_rows][head_dim / block],
 * 4-byte aligned.  QJL signs need format 0 and block 32 (TQ_ERR_UNSUPPORTED
 * otherwise).  [G] sec. 5.2 (block size), sec. 1.2 (turbo4 bits per value),
 * sec. 11 (norm correction).
 */
tq_status tq_quantize_kv_ex(const tq_rotation * rot, int32_t bits, int32_t block,
                            const float * centroids, const float * boundaries,
                            const tq_rotation * qjl,
                            const void * x, tq_dtype dtype, int64_t n_rows, int32_t head_dim,
                            uint32_t format, uint32_t * codes, void * norms,
                            uint32_t * qjl_signs, uint16_t * qjl_rnorm,
                            uint32_t * status_dev, void * stream);

/*
 * tq_attn_logits -- raw attention scores of every query head against every
 * cached key, on `stream`.  [G] sec. 5.3 (pre-rotated query:
 * <q, R^T c[idx]> = <R q, c[idx]>); QJL term: [T] sec. 2.2.
 *
 *   logits[b][h][t] = sum_k fp16(norm_tk) * sum_{j in k} (R q_bh)_j c[code_tj]
 *                     + [QJL] sqrt(pi/2)/m * rho_t * sum_i (S R q_bh)_i (2 s_ti - 1)
 * (no 1/sqrt(d) factor).
 *   q:          device [batch][n_q_heads][head_dim] of q_dtype.
 *   k_codes, k_norms: device, layouts of tq_quantize_kv, rows
 *               [batch][n_kv_heads][ctx]; both 16-byte aligned.
 *   qjl, qjl_signs, qjl_rnorm: NULL, or the QJL handle and arrays written by
 *               tq_quantize_kv with the same handle; both arrays 16-byte
 *               aligned.
 *   logits:     device fp32 [batch][n_q_heads][ctx].
 * n_q_heads must be a multiple of n_kv_heads.  ctx == 0 is a no-op.
 * head_dim 64 or 128 with at most 128 QJL rows, where every (batch, kv head)
 * section of codes, norms, sign words and residual norms starts on a 16-byte
 * boundary, runs on the tensor cores; other shapes give the same scores from
 * a CUDA-core kernel.
 */
tq_status tq_attn_logits(const tq_rotation * rot, int32_t k_bits, int32_t block,
                         const float * k_centroids, const tq_rotation * qjl,
                         const void * q, tq_dtype q_dtype,
                         int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                         int32_t head_dim,
                         const uint32_t * k_codes, const uint16_t * k_norms,
                         const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                         float * logits, void * stream);

/*
 * tq_attn_logits_ex -- tq_attn_logits over a cache written with format flags
 * `format` (k_norms fp16 or fp32 as tq_quantize_kv_ex wrote them).
 */
tq_status tq_attn_logits_ex(const tq_rotation * rot, int32_t k_bits, int32_t block,
                            const float * k_centroids, const tq_rotation * qjl,
                            const void * q, tq_dtype q_dtype,
                            int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                            int32_t head_dim, uint32_t format,
                            const uint32_t * k_codes, const void * k_norms,
                            const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                            float * logits, void * stream);

/*
 * tq_decode_workspace_size -- bytes of device workspace tq_decode_attention
 * needs for this shape on the CURRENT device (the split of the context
 * depends on its SM count).
 */
size_t tq_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                int64_t ctx, int32_t head_dim);

/*
 * tq_decode_attention -- one decode step of attention over the packed cache,
 * on `stream`.  [T] sec. 4.3; [G] sec. 5.3 (rotated query, centroid LUT,
 * norm broadcast), sec. 5.4 (asymmetric K/V bits), sec. 6.1 (inverse
 * rotation of the output).
 *
 *   out[b][h] = R^T * sum_t softmax_t(scale * logits[b][h][t]) * v_hat_rot[t]
 * with v_hat_rot[t] = fp16(v_norm) * v_centroids[v_code] in the rotated
 * frame; K and V share `rot`.  scale <= 0 selects 1/sqrt(head_dim).
 *   q:          device [batch][n_q_heads][head_dim] of q_dtype.
 *   k_*, v_*:   device packed caches (layouts of tq_quantize_kv), code and
 *               norm arrays 16-byte aligned.
 *   qjl, ...:   as in tq_attn_logits (NULL for MSE-only keys).  Keys with QJL
 *               signs run on the tensor cores for head_dim 64 / 128 and at
 *               most 128 projection rows when ctx is a multiple of 8 (every
 *               section 16-byte aligned); other shapes on CUDA cores.
 *   out:        device fp32 [batch][n_q_heads][head_dim].
 *   workspace:  device scratch of at least tq_decode_workspace_size(...)
 *               bytes, 16-byte aligned; contents need no initialisation (the
 *               call writes everything it later reads, on `stream`).
 * ctx must be >= 1.
 */
tq_status tq_decode_attention(const tq_rotation * rot, int32_t k_bits, int32_t v_bits,
                              int32_t block, const float * k_centroids,
                              const float * v_centroids, const tq_rotation * qjl,
                              const void * q, tq_dtype q_dtype,
                              int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                              int32_t head_dim,
                              const uint32_t * k_codes, const uint16_t * k_norms,
                              const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                              const uint32_t * v_codes, const uint16_t * v_norms,
                              float scale, float * out,
                              void * workspace, size_t workspace_bytes, void * stream);

/*
 * tq_decode_attention_ex -- tq_decode_attention over caches written with
 * format flags `format` (K and V norms fp16 or fp32 as tq_quantize_kv_ex
 * wrote them); tq_decode_workspace_size covers every format.
 */
tq_status tq_decode_attention_ex(const tq_rotation * rot, int32_t k_bits, int32_t v_bits,
                                 int32_t block, const float * k_centroids,
                                 const float * v_centroids, const tq_rotation * qjl,
                                 const void * q, tq_dtype q_dtype,
                                 int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                 int64_t ctx, int32_t head_dim, uint32_t format,
                                 const uint32_t * k_codes, const void * k_norms,
                                 const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                                 const uint32_t * v_codes, const void * v_norms,
                                 float scale, float * out,
                                 void * workspace, size_t workspace_bytes, void * stream);

/*
 * tq_decode_attention_static -- tq_decode_attention for callers that cannot
 * allocate device memory: an engine plugin whose enqueue path must never
 * allocate, a server that gives out device memory only from an arena it
 * reserved at start-up, or a decode loop that must not risk the implicit
 * device synchronisation of cudaMalloc / cudaFree.  The pages have no
 * counterpart; this is a convenience of this library.
 *
 * Same arguments, results and errors as tq_decode_attention, minus the
 * workspace: the per-split partials go to a fixed array of
 * TQ_DECODE_STATIC_SCRATCH_BYTES in the library's own device memory, which
 * every GPU that loads the library holds until the process exits.  The call
 * allocates nothing.
 *   - Shapes whose partials for these bit widths and key kind would not fit
 *     the array are rejected with TQ_ERR_UNSUPPORTED before anything is
 *     launched.
 *   - The first call on a device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress) and caches it together
 *     with the CUDA context it was looked up in; a later call made in a
 *     different context (after cudaDeviceReset recreated the primary
 *     context, or under a context the caller pushed) looks it up again.
 *     Make the first call on a device, and the first after such a change,
 *     before any stream capture.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents (nothing in it needs to start at zero).  Calls whose
 *     GPU work overlaps -- on different streams, or from different host
 *     threads -- race on it: serialise them on one stream.
 */
#define TQ_DECODE_STATIC_SCRATCH_BYTES (16u << 20)

tq_status tq_decode_attention_static(const tq_rotation * rot, int32_t k_bits, int32_t v_bits,
                                     int32_t block, const float * k_centroids,
                                     const float * v_centroids, const tq_rotation * qjl,
                                     const void * q, tq_dtype q_dtype,
                                     int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                     int64_t ctx, int32_t head_dim,
                                     const uint32_t * k_codes, const uint16_t * k_norms,
                                     const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                                     const uint32_t * v_codes, const uint16_t * v_norms,
                                     float scale, float * out, void * stream);

/*
 * tq_decode_append_paged -- one decode step over a paged cache that first
 * appends the step's own token: the new K and V rows of every (batch, kv
 * head) are quantized (as tq_quantize_kv defines it) into token ctx - 1 of
 * the cache, then decode attention runs over tokens 0 .. ctx - 1 exactly as
 * in tq_decode_attention.  Two launches on `stream`: the append rides in the
 * query-rotation kernel, and the attention kernel waits for it through
 * programmatic dependent launch.  [G] sec. 5.2 (KV-cache allocation and the
 * graph-side quantize of each new token), sec. 5.3; [T] sec. 4.3.
 *
 *   k_boundaries, v_boundaries: host, the codebooks' decision boundaries (as
 *               tq_build_codebook returns them) for the append.
 *   k_new, v_new: device [batch][n_kv_heads][head_dim] of kv_dtype.
 *   Page storage (device, caller-owned, 16-byte aligned):
 *     k_codes / v_codes  uint32 [n_pages][n_kv_heads][page_size][words per row]
 *     k_norms / v_norms  fp16   [n_pages][n_kv_heads][page_size][head_dim / 32]
 *   block_table: device int32 [batch][max_pages]; entry j of sequence b is the
 *               page holding its tokens [j * page_size, (j + 1) * page_size).
 *               Entries must lie in [0, n_pages); the kernels clamp any other
 *               value into that range rather than read outside the storage.
 *   page_size:  a power of two in [16, 65536]; ctx <= max_pages * page_size.
 *   ctx:        tokens per sequence after the append (all sequences alike).
 *   workspace:  >= tq_decode_workspace_size(batch, n_q_heads, n_kv_heads, ctx,
 *               head_dim) bytes.
 *   status_dev: TQ_STATUS_* of the append (may be NULL).
 * Block 32 with fp16 norms, keys without QJL signs, head_dim 64 / 128 / 256;
 * other shapes return TQ_ERR_UNSUPPORTED before anything is launched.
 */
tq_status tq_decode_append_paged(const tq_rotation * rot, int32_t k_bits, int32_t v_bits,
                                 int32_t block, const float * k_centroids,
                                 const float * k_boundaries, const float * v_centroids,
                                 const float * v_boundaries, const void * q, tq_dtype q_dtype,
                                 const void * k_new, const void * v_new, tq_dtype kv_dtype,
                                 int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                                 int32_t head_dim, int32_t page_size, int32_t n_pages,
                                 const int32_t * block_table, int32_t max_pages,
                                 uint32_t * k_codes, uint16_t * k_norms, uint32_t * v_codes,
                                 uint16_t * v_norms, float scale, float * out, void * workspace,
                                 size_t workspace_bytes, uint32_t * status_dev, void * stream);

/*
 * tq_search_workspace_size -- device workspace bytes of tq_search_topk on the
 * current device (the size depends on its SM count: call it with the device
 * current that the search will run on).
 */
size_t tq_search_workspace_size(int32_t n_queries, int64_t n_db, int32_t head_dim, int32_t k);

/*
 * tq_search_topk -- maximum-inner-product search over a database of packed
 * rows, on `stream`.  [T] sec. 3.4 (the codes serve vector search); the score
 * is the pre-rotated inner product of [G] sec. 5.3:
 *   score(i, j) = <R q_i, x_hat_j> = sum_k fp16(norm_jk) sum_{l in k} (R q_i)_l c[code_jl]
 * (tq_attn_logits' raw score), and the k largest scores of every query are
 * returned, largest first, equal scores by ascending row.
 *   q:          device [n_queries][head_dim] of q_dtype, 16-byte aligned.
 *   db_codes, db_norms: device, n_db rows written by tq_quantize_kv with
 *               `rot`, `bits` and block 32 (fp16 norms), 16-byte aligned.
 *   top_scores: device fp32 [n_queries][k]; top_rows: device int32
 *               [n_queries][k] (row indices into the database).
 *   workspace:  device, >= tq_search_workspace_size(...) bytes, 256-byte
 *               aligned; holds the candidate lists, the rotated queries and
 *               a per-query score bound (with k > 32, the score matrix
 *               instead of the lists).
 * 1 <= k <= min(256, n_db); n_db < 2^31 - 1; n_queries <= 65535.
 * head_dim 64 / 128 with k <= 16 run on the tensor cores (a sample pass sets
 * a bound that k rows reach, the main pass keeps the candidates above it);
 * every other shape on CUDA-core score MMAs.  Both return the exact top k of
 * the score above (fp16 operands, fp32 sums).  A kernel that gave up waiting
 * on its own pipeline (bounded at 1 s) returns rows -1 with NaN scores.
 */
tq_status tq_search_topk(const tq_rotation * rot, int32_t bits, int32_t block,
                         const float * centroids, const void * q, tq_dtype q_dtype,
                         int32_t n_queries, int32_t head_dim, const uint32_t * db_codes,
                         const uint16_t * db_norms, int64_t n_db, int32_t k, float * top_scores,
                         int32_t * top_rows, void * workspace, size_t workspace_bytes,
                         void * stream);

/* Static string for a status code. */
const char * tq_status_string(tq_status s);

/* One-line reason for the last non-OK status returned on this thread. */
const char * tq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
