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
                         int32_t head_dim, int32_t k_bits, int32_t v_bits, bool qjl_keys) {
    const MmaDecodePlan plan = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits,
                                               v_bits, qjl_keys);
    if (plan.ok) return plan.partial_bytes + plan.qfrag_bytes;
    const int32_t splits = decode_splits(batch, n_q_heads, n_kv_heads, ctx, head_dim);
    return decode_workspace_bytes(batch, n_q_heads, splits, head_dim);
}
}  // namespace tq

using namespace tq;

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
    tq_status st = check_rotation(rot, head_dim);
    if (st != TQ_OK) return st;
    if ((st = check_qjl(qjl, head_dim)) != TQ_OK) return st;
    if (!supported_bits(bits)) return fail(TQ_ERR_UNSUPPORTED, "bits must be 2, 3 or 4");
    if (block != kBlock) return fail(TQ_ERR_UNSUPPORTED, "block must be 32");
    if (dtype != TQ_DTYPE_F32 && dtype != TQ_DTYPE_BF16)
        return fail(TQ_ERR_INVALID_ARG, "unknown dtype");
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
    SearchTable tab;
    std::string why;
    if (!build_search_table(bits, boundaries, &tab, &why)) return fail(TQ_ERR_UNSUPPORTED, why);
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
    if (block != kBlock) return fail(TQ_ERR_UNSUPPORTED, "block must be 32");
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
    return cuda_status(launch_logits(rot, kcb, a, stream), "logits launch");
}


size_t tq_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                int64_t ctx, int32_t head_dim) {
    if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || ctx < 1 || head_dim < 1) return 0;
    const int32_t s = decode_splits(batch, n_q_heads, n_kv_heads, ctx, head_dim);
    size_t need = decode_workspace_bytes(batch, n_q_heads, s, head_dim);
    // the tensor-core path (any bit widths) may need more
    const MmaDecodePlan p = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim, 4, 4, false);
    if (p.ok) need = std::max(need, p.partial_bytes + p.qfrag_bytes);
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
    const MmaDecodePlan plan = plan_mma_decode(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits,
                                               v_bits, qjl_signs != nullptr);
    const int32_t splits = plan.ok ? plan.slots
                                   : decode_splits(batch, n_q_heads, n_kv_heads, ctx, head_dim);
    const size_t need = decode_need_bytes(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits,
                                          v_bits, qjl_signs != nullptr);
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
    if (plan.ok) {
        a.mma_mode = 1;
        a.mma_warps = plan.warps;
        a.mma_groups = plan.groups;
        a.mma_slabs = plan.slabs;
        a.mma_spb = plan.spb;
        a.mma_qfrag = reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(workspace) +
                                                   plan.partial_bytes);
    }
    return cuda_status(launch_decode(rot, kcb, vcb, a, stream), "decode launch");
}

}  // extern "C"
