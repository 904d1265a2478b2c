// C entry points of the TurboQuant library that touch the device: rotation
// handles, argument validation and kernel dispatch.  Every host-checkable
// error is reported before anything is launched; no entry point synchronises.

#include <algorithm>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <utility>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace tq {

int32_t device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    return sms > 0 ? sms : 148;
}

int ensure_dynamic_smem(const void * func, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> set_bytes;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    std::lock_guard<std::mutex> lock(mu);
    int & cur = set_bytes[{func, dev}];
    if (cur >= bytes) return 0;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return (int)e;
    cur = bytes;
    return 0;
}

namespace {

uint16_t f32_to_bf16_bits(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16);  // inf / nan
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;  // round to nearest even
    return (uint16_t)(u >> 16);
}

float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

bool aligned(const void * p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool supported_dim(int32_t d) { return d == 64 || d == 128 || d == 256; }
bool supported_bits(int32_t b) { return b >= 2 && b <= 4; }

tq_status build_codebook_params(int32_t bits, const float * centroids, const float * boundaries,
                                CodebookParams * out, bool need_boundaries) {
    if (!centroids) return fail(TQ_ERR_INVALID_ARG, "centroids is NULL");
    if (need_boundaries && !boundaries) return fail(TQ_ERR_INVALID_ARG, "boundaries is NULL");
    std::memset(out, 0, sizeof(*out));
    const int n = 1 << bits;
    for (int i = 0; i < n; ++i) {
        if (!std::isfinite(centroids[i])) return fail(TQ_ERR_INVALID_ARG, "non-finite centroid");
        if (i > 0 && !(centroids[i] > centroids[i - 1]))
            return fail(TQ_ERR_INVALID_ARG, "centroids must be strictly ascending");
        out->centroid[i] = centroids[i];
    }
    if (need_boundaries) {
        // The kernels search |u| against the positive boundaries; the table
        // must be symmetric about zero with its middle boundary at zero.
        const int half = n / 2;
        if (boundaries[half - 1] != 0.0f)
            return fail(TQ_ERR_INVALID_ARG, "middle boundary must be 0 (symmetric codebook)");
        for (int k = 0; k + 1 < half; ++k) {
            const float tp = boundaries[half + k];
            const float tn = boundaries[half - 2 - k];
            if (!(tp > 0.0f) || tp != -tn)
                return fail(TQ_ERR_INVALID_ARG, "boundaries must be symmetric about 0");
            out->pos_boundary[k] = tp;
        }
    }
    return TQ_OK;
}

tq_status upload_dense(tq_rotation * r) {
    const size_t n = (size_t)r->rows * r->cols;
    std::vector<float> f(n);
    std::vector<uint16_t> hi(n), lo(n);
    for (size_t i = 0; i < n; ++i) {
        f[i] = (float)r->host[i];
        hi[i] = f32_to_bf16_bits(f[i]);
        lo[i] = f32_to_bf16_bits(f[i] - bf16_bits_to_f32(hi[i]));
    }
    if (cudaGetDevice(&r->device) != cudaSuccess) {
        cudaGetLastError();
        return fail(TQ_ERR_CUDA, "no CUDA device");
    }
    if (cudaMalloc(&r->dev_f32, n * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&r->dev_hi, n * sizeof(uint16_t)) != cudaSuccess ||
        cudaMalloc(&r->dev_lo, n * sizeof(uint16_t)) != cudaSuccess) {
        cudaGetLastError();
        return fail(TQ_ERR_ALLOC, "cudaMalloc failed for rotation");
    }
    if (cudaMemcpy(r->dev_f32, f.data(), n * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(r->dev_hi, hi.data(), n * sizeof(uint16_t), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(r->dev_lo, lo.data(), n * sizeof(uint16_t), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaGetLastError();
        return fail(TQ_ERR_CUDA, "cudaMemcpy failed for rotation");
    }
    return TQ_OK;
}

tq_status check_rotation(const tq_rotation * rot, int32_t head_dim) {
    if (!rot) return fail(TQ_ERR_INVALID_ARG, "rotation handle is NULL");
    if (rot->kind != TQ_ROT_WHT && rot->kind != TQ_ROT_HAAR)
        return fail(TQ_ERR_INVALID_ARG, "rotation must be WHT or HAAR");
    if (rot->rows != head_dim || rot->cols != head_dim)
        return fail(TQ_ERR_INVALID_ARG, "rotation size does not match head_dim");
    if (!supported_dim(head_dim)) return fail(TQ_ERR_UNSUPPORTED, "head_dim must be 64, 128 or 256");
    return TQ_OK;
}

tq_status check_qjl(const tq_rotation * qjl, int32_t head_dim) {
    if (!qjl) return TQ_OK;
    if (qjl->kind != TQ_ROT_GAUSS) return fail(TQ_ERR_INVALID_ARG, "qjl handle must be GAUSS");
    if (qjl->cols != head_dim) return fail(TQ_ERR_INVALID_ARG, "qjl cols must equal head_dim");
    if (qjl->rows < 32 || qjl->rows > 256 || qjl->rows % 32)
        return fail(TQ_ERR_UNSUPPORTED, "qjl rows must be a multiple of 32 in [32, 256]");
    return TQ_OK;
}

tq_status cuda_status(int err, const char * what) {
    if (err == 0) return TQ_OK;
    return fail(TQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString((cudaError_t)err));
}

}  // namespace
}  // namespace tq

namespace tq {
size_t decode_need_bytes(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                         int32_t head_dim, int32_t k_bits, int32_t v_bits, int32_t qjl_m) {
    if (qjl_m >= 0) {
        const MmaDecodePlan plan = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim,
                                                   k_bits, v_bits, qjl_m);
        if (plan.ok) return plan.partial_bytes + plan.qfrag_bytes;
    }
    const int32_t splits = decode_splits(batch, n_q_heads, n_kv_heads, ctx, head_dim);
    return decode_workspace_bytes(batch, n_q_heads, splits, head_dim);
}
}  // namespace tq

using namespace tq;

// Block sizes and format flags of the packed cache.
static tq_status check_format(int32_t block, int32_t head_dim, uint32_t format) {
    if (block != 32 && block != 64 && block != 128)
        return fail(TQ_ERR_UNSUPPORTED, "block must be 32, 64 or 128");
    if (block > head_dim) return fail(TQ_ERR_UNSUPPORTED, "block larger than head_dim");
    if (format & ~(uint32_t)(TQ_FMT_NORM_F32 | TQ_FMT_NORM_CORRECTED | TQ_FMT_GROUPED))
        return fail(TQ_ERR_INVALID_ARG, "unknown format flags");
    if ((format & TQ_FMT_GROUPED) && (head_dim != 128 || block != 32))
        return fail(TQ_ERR_UNSUPPORTED, "lane-grouped codes: head_dim 128, block 32");
    return TQ_OK;
}


extern "C" {

tq_status tq_make_rotation(tq_rot_kind kind, int32_t rows, int32_t cols, uint64_t seed,
                           tq_rotation ** out) {
    if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (rows < 1 || cols < 1 || (int64_t)rows * cols > (1 << 24))
        return fail(TQ_ERR_INVALID_ARG, "bad rotation size");
    tq_rotation * r = new (std::nothrow) tq_rotation();
    if (!r) return fail(TQ_ERR_ALLOC, "host allocation failed");
    r->kind = (int32_t)kind;
    r->rows = rows;
    r->cols = cols;
    r->seed = seed;
    r->host.resize((size_t)rows * cols);
    std::string why;
    if (!generate_matrix((int32_t)kind, rows, cols, seed, r->host.data(), &why)) {
        delete r;
        return fail(TQ_ERR_INVALID_ARG, why);
    }
    if (kind == TQ_ROT_WHT) {
        if (rows > 256) {
            delete r;
            return fail(TQ_ERR_UNSUPPORTED, "WHT rotation handles support d <= 256");
        }
        std::vector<double> s((size_t)2 * rows);
        signs_fill(seed, s.data(), 2 * rows);
        for (int i = 0; i < rows; ++i) {
            if (s[i] < 0) r->d1_bits[i >> 5] |= 1u << (i & 31);
            if (s[rows + i] < 0) r->d2_bits[i >> 5] |= 1u << (i & 31);
        }
        if (cudaGetDevice(&r->device) != cudaSuccess) cudaGetLastError();
    } else {
        tq_status st = upload_dense(r);
        if (st != TQ_OK) {
            tq_free_rotation(r);
            return st;
        }
    }
    *out = r;
    return TQ_OK;
}

void tq_free_rotation(tq_rotation * rot) {
    if (!rot) return;
    if (rot->dev_f32) cudaFree(rot->dev_f32);
    if (rot->dev_hi) cudaFree(rot->dev_hi);
    if (rot->dev_lo) cudaFree(rot->dev_lo);
    delete rot;
}

tq_status tq_rotation_copy_host(const tq_rotation * rot, double * out) {
    if (!rot || !out) return fail(TQ_ERR_INVALID_ARG, "null pointer");
    std::memcpy(out, rot->host.data(), sizeof(double) * rot->host.size());
    return TQ_OK;
}

tq_status tq_rotation_info(const tq_rotation * rot, int32_t * kind, int32_t * rows,
                           int32_t * cols, uint64_t * seed) {
    if (!rot) return fail(TQ_ERR_INVALID_ARG, "rotation handle is NULL");
    if (kind) *kind = rot->kind;
    if (rows) *rows = rot->rows;
    if (cols) *cols = rot->cols;
    if (seed) *seed = rot->seed;
    return TQ_OK;
}

tq_status tq_quantize_kv(const tq_rotation * rot, int32_t bits, int32_t block,
                         const float * centroids, const float * boundaries,
                         const tq_rotation * qjl,
                         const void * x, tq_dtype dtype, int64_t n_rows, int32_t head_dim,
                         uint32_t * codes, uint16_t * norms,
                         uint32_t * qjl_signs, uint16_t * qjl_rnorm,
                         uint32_t * status_dev, void * stream) {
    return tq_quantize_kv_ex(rot, bits, block, centroids, boundaries, qjl, x, dtype, n_rows,
                             head_dim, 0u, codes, norms, qjl_signs, qjl_rnorm, status_dev, stream);
}

tq_status tq_quantize_kv_ex(const tq_rotation * rot, int32_t bits, int32_t block,
                            const float * centroids, const float * boundaries,
                            const tq_rotation * qjl,
                            const void * x, tq_dtype dtype, int64_t n_rows, int32_t head_dim,
                            uint32_t format, uint32_t * codes, void * norms_out,
                            uint32_t * qjl_signs, uint16_t * qjl_rnorm,
                            uint32_t * status_dev, void * stream) {
    uint16_t * norms = static_cast<uint16_t *>(norms_out);
    tq_status st = check_rotation(rot, head_dim);
    if (st != TQ_OK) return st;
    if ((st = check_qjl(qjl, head_dim)) != TQ_OK) return st;
    if (!supported_bits(bits)) return fail(TQ_ERR_UNSUPPORTED, "bits must be 2, 3 or 4");
    if ((st = check_format(block, head_dim, format)) != TQ_OK) return st;
    if (qjl && (block != kBlock || format != 0u))
        return fail(TQ_ERR_UNSUPPORTED, "QJL signs need block 32 with fp16 norms and no norm correction");
    if (dtype != TQ_DTYPE_F32 && dtype != TQ_DTYPE_BF16)
        return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
    if ((format & TQ_FMT_GROUPED) && (dtype != TQ_DTYPE_BF16 || format != TQ_FMT_GROUPED))
        return fail(TQ_ERR_UNSUPPORTED, "lane-grouped codes: bf16 rows, fp16 norms, no norm correction");
    if (n_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows < 0");
    CodebookParams cb;
    if ((st = build_codebook_params(bits, centroids, boundaries, &cb, true)) != TQ_OK) return st;
    if (n_rows == 0) return TQ_OK;
    if (!x || !codes || !norms) return fail(TQ_ERR_INVALID_ARG, "null x / codes / norms");
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(norms, 4))
        return fail(TQ_ERR_INVALID_ARG, "x and codes must be 16-byte aligned, norms 4-byte");
    if (qjl) {
        if (!qjl_signs || !qjl_rnorm) return fail(TQ_ERR_INVALID_ARG, "QJL outputs are NULL");
        if (!aligned(qjl_signs, 16) || !aligned(qjl_rnorm, 2))
            return fail(TQ_ERR_INVALID_ARG, "qjl_signs must be 16-byte aligned");
        if ((int64_t)qjl->rows * head_dim > 16384)
            return fail(TQ_ERR_UNSUPPORTED, "QJL needs m * head_dim <= 16384");
    }
    QuantizeArgs a{};
    a.x = x;
    a.n_rows = n_rows;
    a.codes = codes;
    a.norms = norms;
    a.qjl_signs = qjl_signs;
    a.qjl_rnorm = qjl_rnorm;
    a.status = status_dev;
    a.rot_f32 = rot->dev_f32;
    a.rot_hi = rot->dev_hi;
    a.rot_lo = rot->dev_lo;
    a.qjl_f32 = qjl ? qjl->dev_f32 : nullptr;
    a.qjl_hi = qjl ? qjl->dev_hi : nullptr;
    a.qjl_lo = qjl ? qjl->dev_lo : nullptr;
    a.qjl_m = qjl ? qjl->rows : 0;
    a.inv_sqrt_d = 1.0f / std::sqrt((float)head_dim);
    a.norm_block = block;
    a.norm_f32 = (format & TQ_FMT_NORM_F32) ? 1 : 0;
    a.norm_corr = (format & TQ_FMT_NORM_CORRECTED) ? 1 : 0;
    a.grouped = (format & TQ_FMT_GROUPED) ? 1 : 0;
    for (int i = 0; i < (1 << bits); ++i) a.centroid_sq[i] = centroids[i] * centroids[i];
    for (int i = 0; i < 16; ++i) a.boundary[i] = i < (1 << bits) - 1 ? boundaries[i] : 0.0f;
    const bool variant = block != kBlock || (format & (TQ_FMT_NORM_F32 | TQ_FMT_NORM_CORRECTED)) != 0u;
    SearchTable tab;
    std::string why;
    if (!build_search_table(bits, boundaries, &tab, &why)) {
        // the variant kernels search the boundaries directly and need no table
        if (!variant) return fail(TQ_ERR_UNSUPPORTED, why);
        std::memset(&tab, 0, sizeof(tab));
        tab.size = 1;
    }
    return cuda_status(launch_quantize(rot, qjl, bits, dtype == TQ_DTYPE_BF16, head_dim, cb, tab, a,
                                       stream),
                       "quantize launch");
}

static tq_status check_attn_common(const tq_rotation * rot, const tq_rotation * qjl,
                                   int32_t k_bits, int32_t block, const void * q, tq_dtype q_dtype,
                                   int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                   int64_t ctx, int32_t head_dim, const uint32_t * k_codes,
                                   const uint16_t * k_norms, const uint32_t * qjl_signs,
                                   const uint16_t * qjl_rnorm) {
    tq_status st = check_rotation(rot, head_dim);
    if (st != TQ_OK) return st;
    if ((st = check_qjl(qjl, head_dim)) != TQ_OK) return st;
    if (!supported_bits(k_bits)) return fail(TQ_ERR_UNSUPPORTED, "k_bits must be 2, 3 or 4");
    if (block != 32 && block != 64 && block != 128)
        return fail(TQ_ERR_UNSUPPORTED, "block must be 32, 64 or 128");
    if (block > head_dim) return fail(TQ_ERR_UNSUPPORTED, "block larger than head_dim");
    if (qjl && block != kBlock) return fail(TQ_ERR_UNSUPPORTED, "QJL signs need block 32");
    if (q_dtype != TQ_DTYPE_F32 && q_dtype != TQ_DTYPE_BF16)
        return fail(TQ_ERR_INVALID_ARG, "unknown q dtype");
    if (batch < 1 || n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads)
        return fail(TQ_ERR_INVALID_ARG, "heads: n_q_heads must be a positive multiple of n_kv_heads");
    if (n_q_heads / n_kv_heads > 8) return fail(TQ_ERR_UNSUPPORTED, "query group larger than 8");
    if (ctx < 0) return fail(TQ_ERR_INVALID_ARG, "ctx < 0");
    if ((int64_t)batch * n_kv_heads > 65535) return fail(TQ_ERR_UNSUPPORTED, "batch * kv heads > 65535");
    if (!q || !k_codes || !k_norms) return fail(TQ_ERR_INVALID_ARG, "null q / k_codes / k_norms");
    if (!aligned(k_codes, 16) || !aligned(k_norms, 16) || !aligned(q, 16))
        return fail(TQ_ERR_INVALID_ARG, "q, k_codes and k_norms must be 16-byte aligned");
    if (qjl && (!qjl_signs || !qjl_rnorm))
        return fail(TQ_ERR_INVALID_ARG, "QJL handle given without signs / rnorm");
    if (qjl && (!aligned(qjl_signs, 16) || !aligned(qjl_rnorm, 16)))
        return fail(TQ_ERR_INVALID_ARG, "qjl_signs and qjl_rnorm must be 16-byte aligned");
    if (!qjl && (qjl_signs || qjl_rnorm))
        return fail(TQ_ERR_INVALID_ARG, "QJL arrays given without a QJL handle");
    return TQ_OK;
}

tq_status tq_attn_logits(const tq_rotation * rot, int32_t k_bits, int32_t block,
                         const float * k_centroids, const tq_rotation * qjl,
                         const void * q, tq_dtype q_dtype,
                         int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                         int32_t head_dim,
                         const uint32_t * k_codes, const uint16_t * k_norms,
                         const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                         float * logits, void * stream) {
    return tq_attn_logits_ex(rot, k_bits, block, k_centroids, qjl, q, q_dtype, batch, n_q_heads,
                             n_kv_heads, ctx, head_dim, 0u, k_codes, k_norms, qjl_signs, qjl_rnorm,
                             logits, stream);
}

tq_status tq_attn_logits_ex(const tq_rotation * rot, int32_t k_bits, int32_t block,
                            const float * k_centroids, const tq_rotation * qjl,
                            const void * q, tq_dtype q_dtype,
                            int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                            int32_t head_dim, uint32_t format,
                            const uint32_t * k_codes, const void * k_norms_in,
                            const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                            float * logits, void * stream) {
    const uint16_t * k_norms = static_cast<const uint16_t *>(k_norms_in);
    if (tq_status sf = check_format(block, head_dim, format)) return sf;
    if (format & TQ_FMT_GROUPED)
        return fail(TQ_ERR_UNSUPPORTED, "key codes are read in the block order (lane-grouped rows are value rows)");
    tq_status st = check_attn_common(rot, qjl, k_bits, block, q, q_dtype, batch, n_q_heads,
                                     n_kv_heads, ctx, head_dim, k_codes, k_norms, qjl_signs,
                                     qjl_rnorm);
    if (st != TQ_OK) return st;
    CodebookParams kcb;
    if ((st = build_codebook_params(k_bits, k_centroids, nullptr, &kcb, false)) != TQ_OK) return st;
    if (!logits) return fail(TQ_ERR_INVALID_ARG, "logits is NULL");
    if (ctx == 0) return TQ_OK;
    AttnArgs a{};
    a.q = q;
    a.q_bf16 = q_dtype == TQ_DTYPE_BF16;
    a.batch = batch;
    a.n_q_heads = n_q_heads;
    a.n_kv_heads = n_kv_heads;
    a.head_dim = head_dim;
    a.ctx = ctx;
    a.k_codes = k_codes;
    a.k_norms = k_norms;
    a.qjl_signs = qjl_signs;
    a.qjl_rnorm = qjl_rnorm;
    a.k_bits = k_bits;
    a.rot_kind = rot->kind;
    a.rot_f32 = rot->dev_f32;
    a.qjl_f32 = qjl ? qjl->dev_f32 : nullptr;
    a.qjl_m = qjl ? qjl->rows : 0;
    a.logits = logits;
    a.norm_block = block;
    a.norm_f32 = (format & TQ_FMT_NORM_F32) ? 1 : 0;
    return cuda_status(launch_logits(rot, kcb, a, stream), "logits launch");
}


size_t tq_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                int64_t ctx, int32_t head_dim) {
    if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || ctx < 1 || head_dim < 1) return 0;
    const int32_t s = decode_splits(batch, n_q_heads, n_kv_heads, ctx, head_dim);
    size_t need = decode_workspace_bytes(batch, n_q_heads, s, head_dim);
    // the tensor-core path (any bit widths, keys with or without QJL signs)
    // may need more
    for (int32_t m : {0, 32, 64, 96, 128})
        need = std::max(need, decode_need_bytes(batch, n_q_heads, n_kv_heads, ctx, head_dim, 4, 4, m));
    // a paged cache takes the tensor-core path at any context length
    const MmaDecodePlan pp = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim, 4, 4, 0, true);
    if (pp.ok) need = std::max(need, pp.partial_bytes + pp.qfrag_bytes);
    return need;
}

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
                              void * workspace, size_t workspace_bytes, void * stream) {
    return tq_decode_attention_ex(rot, k_bits, v_bits, block, k_centroids, v_centroids, qjl, q,
                                  q_dtype, batch, n_q_heads, n_kv_heads, ctx, head_dim, 0u,
                                  k_codes, k_norms, qjl_signs, qjl_rnorm, v_codes, v_norms, scale,
                                  out, workspace, workspace_bytes, stream);
}

tq_status tq_decode_attention_ex(const tq_rotation * rot, int32_t k_bits, int32_t v_bits,
                                 int32_t block, const float * k_centroids,
                                 const float * v_centroids, const tq_rotation * qjl,
                                 const void * q, tq_dtype q_dtype,
                                 int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                                 int32_t head_dim, uint32_t format,
                                 const uint32_t * k_codes, const void * k_norms_in,
                                 const uint32_t * qjl_signs, const uint16_t * qjl_rnorm,
                                 const uint32_t * v_codes, const void * v_norms_in,
                                 float scale, float * out,
                                 void * workspace, size_t workspace_bytes, void * stream) {
    const uint16_t * k_norms = static_cast<const uint16_t *>(k_norms_in);
    const uint16_t * v_norms = static_cast<const uint16_t *>(v_norms_in);
    if (tq_status sf = check_format(block, head_dim, format)) return sf;
    tq_status st = check_attn_common(rot, qjl, k_bits, block, q, q_dtype, batch, n_q_heads,
                                     n_kv_heads, ctx, head_dim, k_codes, k_norms, qjl_signs,
                                     qjl_rnorm);
    if (st != TQ_OK) return st;
    if (!supported_bits(v_bits)) return fail(TQ_ERR_UNSUPPORTED, "v_bits must be 2, 3 or 4");
    if (ctx < 1) return fail(TQ_ERR_INVALID_ARG, "decode needs ctx >= 1");
    CodebookParams kcb, vcb;
    if ((st = build_codebook_params(k_bits, k_centroids, nullptr, &kcb, false)) != TQ_OK) return st;
    if ((st = build_codebook_params(v_bits, v_centroids, nullptr, &vcb, false)) != TQ_OK) return st;
    if (!v_codes || !v_norms || !out) return fail(TQ_ERR_INVALID_ARG, "null v_codes / v_norms / out");
    if (!aligned(v_codes, 16) || !aligned(v_norms, 16))
        return fail(TQ_ERR_INVALID_ARG, "v_codes and v_norms must be 16-byte aligned");
    const int32_t qjl_m = qjl ? qjl->rows : 0;
    // the tensor-core path reads fp16 norms per 32-block (value codes in
    // either order)
    const bool v_grouped = (format & TQ_FMT_GROUPED) != 0u;
    const bool std_format = block == kBlock && (format & TQ_FMT_NORM_F32) == 0u;
    MmaDecodePlan plan{};
    plan.ok = false;
    if (std_format)
        plan = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits, v_bits, qjl_m);
    const int32_t splits = plan.ok ? plan.slots
                                   : decode_splits(batch, n_q_heads, n_kv_heads, ctx, head_dim);
    const size_t need = decode_need_bytes(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits,
                                          v_bits, std_format ? qjl_m : -1);
    if (!workspace || workspace_bytes < need)
        return fail(TQ_ERR_INVALID_ARG, "workspace missing or smaller than tq_decode_workspace_size");
    if (!aligned(workspace, 16)) return fail(TQ_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    AttnArgs a{};
    a.q = q;
    a.q_bf16 = q_dtype == TQ_DTYPE_BF16;
    a.batch = batch;
    a.n_q_heads = n_q_heads;
    a.n_kv_heads = n_kv_heads;
    a.head_dim = head_dim;
    a.ctx = ctx;
    a.k_codes = k_codes;
    a.k_norms = k_norms;
    a.qjl_signs = qjl_signs;
    a.qjl_rnorm = qjl_rnorm;
    a.v_codes = v_codes;
    a.v_norms = v_norms;
    a.k_bits = k_bits;
    a.v_bits = v_bits;
    a.rot_kind = rot->kind;
    a.rot_f32 = rot->dev_f32;
    a.qjl_f32 = qjl ? qjl->dev_f32 : nullptr;
    a.qjl_m = qjl ? qjl->rows : 0;
    a.scale = scale > 0.0f ? scale : 1.0f / std::sqrt((float)head_dim);
    a.out = out;
    a.workspace = workspace;
    a.n_splits = splits;
    a.norm_block = block;
    a.norm_f32 = (format & TQ_FMT_NORM_F32) ? 1 : 0;
    a.v_grouped = v_grouped ? 1 : 0;
    if (plan.ok) {
        a.mma_mode = 1;
        a.mma_warps = plan.warps;
        a.mma_groups = plan.groups;
        a.mma_slabs = plan.slabs;
        a.mma_spb = plan.spb;
        a.mma_qfrag = reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(workspace) +
                                                   plan.partial_bytes);
        a.mma_qwords = plan.qfrag_words;
    }
    return cuda_status(launch_decode(rot, kcb, vcb, a, stream), "decode launch");
}

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
                                 size_t workspace_bytes, uint32_t * status_dev, void * stream) {
    tq_status st = check_attn_common(rot, nullptr, k_bits, block, q, q_dtype, batch, n_q_heads,
                                     n_kv_heads, ctx, head_dim, k_codes, k_norms, nullptr, nullptr);
    if (st != TQ_OK) return st;
    if (block != kBlock) return fail(TQ_ERR_UNSUPPORTED, "append decode reads block 32 (fp16 norms)");
    if (!supported_bits(v_bits)) return fail(TQ_ERR_UNSUPPORTED, "v_bits must be 2, 3 or 4");
    if (ctx < 1) return fail(TQ_ERR_INVALID_ARG, "decode needs ctx >= 1");
    if (kv_dtype != TQ_DTYPE_F32 && kv_dtype != TQ_DTYPE_BF16)
        return fail(TQ_ERR_INVALID_ARG, "unknown kv dtype");
    if (page_size < 16 || page_size > 65536 || (page_size & (page_size - 1)) != 0)
        return fail(TQ_ERR_UNSUPPORTED, "page_size must be a power of two in [16, 65536]");
    if (n_pages < 1 || max_pages < 1 || !block_table)
        return fail(TQ_ERR_INVALID_ARG, "n_pages, max_pages and block_table are required");
    if (ctx > (int64_t)max_pages * page_size)
        return fail(TQ_ERR_INVALID_ARG, "ctx exceeds max_pages * page_size");
    if ((int64_t)n_pages * n_kv_heads * page_size + 16 > (int64_t)INT32_MAX)
        return fail(TQ_ERR_UNSUPPORTED, "page storage above 2^31 rows");
    if (!k_new || !v_new || !v_codes || !v_norms || !out || !k_boundaries || !v_boundaries)
        return fail(TQ_ERR_INVALID_ARG, "null k_new / v_new / v cache / out / boundaries");
    if (!aligned(v_codes, 16) || !aligned(v_norms, 16) || !aligned(k_new, 4) || !aligned(v_new, 4) ||
        !aligned(block_table, 4))
        return fail(TQ_ERR_INVALID_ARG, "v cache 16-byte, new rows and block table 4-byte aligned");
    CodebookParams kcb, vcb;
    if ((st = build_codebook_params(k_bits, k_centroids, k_boundaries, &kcb, true)) != TQ_OK) return st;
    if ((st = build_codebook_params(v_bits, v_centroids, v_boundaries, &vcb, true)) != TQ_OK) return st;
    const MmaDecodePlan plan = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits,
                                               v_bits, 0, true);
    if (!plan.ok) return fail(TQ_ERR_UNSUPPORTED, "shape outside the tensor-core decode");
    const size_t need = plan.partial_bytes + plan.qfrag_bytes;
    if (!workspace || workspace_bytes < need)
        return fail(TQ_ERR_INVALID_ARG, "workspace missing or smaller than tq_decode_workspace_size");
    if (!aligned(workspace, 16)) return fail(TQ_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    AttnArgs a{};
    a.q = q;
    a.q_bf16 = q_dtype == TQ_DTYPE_BF16;
    a.batch = batch;
    a.n_q_heads = n_q_heads;
    a.n_kv_heads = n_kv_heads;
    a.head_dim = head_dim;
    a.ctx = ctx;
    a.k_codes = k_codes;
    a.k_norms = k_norms;
    a.v_codes = v_codes;
    a.v_norms = v_norms;
    a.k_bits = k_bits;
    a.v_bits = v_bits;
    a.rot_kind = rot->kind;
    a.rot_f32 = rot->dev_f32;
    a.scale = scale > 0.0f ? scale : 1.0f / std::sqrt((float)head_dim);
    a.out = out;
    a.workspace = workspace;
    a.n_splits = plan.slots;
    a.norm_block = kBlock;
    a.mma_mode = 1;
    a.mma_warps = plan.warps;
    a.mma_groups = plan.groups;
    a.mma_slabs = plan.slabs;
    a.mma_spb = plan.spb;
    a.mma_qfrag = reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(workspace) + plan.partial_bytes);
    a.mma_qwords = plan.qfrag_words;
    a.page_size = page_size;
    int shift = 0;
    while ((1 << shift) < page_size) ++shift;
    a.page_shift = shift;
    a.max_pages = max_pages;
    a.n_pages = n_pages;
    a.block_table = block_table;
    a.mma_wait_first = 1;
    AppendParams ap{};
    ap.enabled = 1;
    ap.kv_bf16 = kv_dtype == TQ_DTYPE_BF16;
    ap.k_new = k_new;
    ap.v_new = v_new;
    ap.k_codes = k_codes;
    ap.k_norms = k_norms;
    ap.v_codes = v_codes;
    ap.v_norms = v_norms;
    ap.status = status_dev;
    for (int i = 0; i < (1 << k_bits) - 1; ++i) ap.k_bound[i] = k_boundaries[i];
    for (int i = 0; i < (1 << v_bits) - 1; ++i) ap.v_bound[i] = v_boundaries[i];
    return cuda_status(launch_decode(rot, kcb, vcb, a, stream, &ap), "append decode launch");
}

size_t tq_search_workspace_size(int32_t n_queries, int64_t n_db, int32_t head_dim, int32_t k) {
    if (n_queries < 1 || n_db < 1 || k < 1 || !supported_dim(head_dim)) return 0;
    return search_workspace_bytes(n_queries, n_db, head_dim, k);
}

tq_status tq_search_topk(const tq_rotation * rot, int32_t bits, int32_t block,
                         const float * centroids, const void * q, tq_dtype q_dtype,
                         int32_t n_queries, int32_t head_dim, const uint32_t * db_codes,
                         const uint16_t * db_norms, int64_t n_db, int32_t k, float * top_scores,
                         int32_t * top_rows, void * workspace, size_t workspace_bytes,
                         void * stream) {
    tq_status st = check_rotation(rot, head_dim);
    if (st != TQ_OK) return st;
    if (!supported_bits(bits)) return fail(TQ_ERR_UNSUPPORTED, "bits must be 2, 3 or 4");
    if (block != kBlock) return fail(TQ_ERR_UNSUPPORTED, "search reads block 32 (fp16 norms)");
    if (q_dtype != TQ_DTYPE_F32 && q_dtype != TQ_DTYPE_BF16)
        return fail(TQ_ERR_INVALID_ARG, "unknown q dtype");
    if (n_queries < 1 || n_db < 1) return fail(TQ_ERR_INVALID_ARG, "n_queries and n_db must be >= 1");
    if (n_db > (int64_t)INT32_MAX - 1) return fail(TQ_ERR_UNSUPPORTED, "n_db >= 2^31 - 1");
    if (n_queries > 65535) return fail(TQ_ERR_UNSUPPORTED, "more than 65535 queries");
    if (k < 1 || k > 256 || (int64_t)k > n_db)
        return fail(TQ_ERR_UNSUPPORTED, "k must be in [1, min(256, n_db)]");
    CodebookParams kcb;
    if ((st = build_codebook_params(bits, centroids, nullptr, &kcb, false)) != TQ_OK) return st;
    if (!q || !db_codes || !db_norms || !top_scores || !top_rows)
        return fail(TQ_ERR_INVALID_ARG, "null q / db_codes / db_norms / outputs");
    if (!aligned(q, 16) || !aligned(db_codes, 16) || !aligned(db_norms, 16))
        return fail(TQ_ERR_INVALID_ARG, "q, db_codes and db_norms must be 16-byte aligned");
    const size_t need = search_workspace_bytes(n_queries, n_db, head_dim, k);
    if (!workspace || workspace_bytes < need)
        return fail(TQ_ERR_INVALID_ARG, "workspace missing or smaller than tq_search_workspace_size");
    if (!aligned(workspace, 256)) return fail(TQ_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    AttnArgs a{};
    a.q = q;
    a.q_bf16 = q_dtype == TQ_DTYPE_BF16;
    a.batch = 1;
    a.n_q_heads = n_queries;
    a.n_kv_heads = 1;
    a.head_dim = head_dim;
    a.ctx = n_db;
    a.k_codes = db_codes;
    a.k_norms = db_norms;
    a.k_bits = bits;
    a.rot_kind = rot->kind;
    a.rot_f32 = rot->dev_f32;
    a.workspace = workspace;
    a.norm_block = kBlock;
    return cuda_status(launch_search(rot, kcb, a, k, top_scores, top_rows, stream), "search launch");
}

}  // extern "C"
