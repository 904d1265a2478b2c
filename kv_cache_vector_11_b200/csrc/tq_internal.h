// Internal declarations shared by the host code and the CUDA kernels of the
// TurboQuant library.  Not part of the public ABI (include/tq.h is).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <string>
#include <vector>

#include "../../include/tq.h"

struct tq_rotation {
    int32_t kind = 0;
    int32_t rows = 0;
    int32_t cols = 0;
    uint64_t seed = 0;
    std::vector<double> host;   // dense float64 matrix, row-major
    // WHT: sign bits of D1 and D2 (bit i set <=> sign_i = -1), head_dim <= 256.
    uint32_t d1_bits[8] = {0};
    uint32_t d2_bits[8] = {0};
    // HAAR / GAUSS: device copies (row-major rows x cols).
    float * dev_f32 = nullptr;
    uint16_t * dev_hi = nullptr;  // bf16 bits of fp32 value rounded to bf16
    uint16_t * dev_lo = nullptr;  // bf16 bits of (value - hi)
    int device = -1;
};

namespace tq {

// Thread-local error detail; returns `s` for convenient `return fail(...)`.
tq_status fail(tq_status s, const std::string & why);
const char * last_error_cstr();

// Host generators (tq_host.cpp).
void splitmix64_fill(uint64_t seed, uint64_t * out, int64_t n);
void signs_fill(uint64_t seed, double * out, int64_t n);
void gaussians_fill(uint64_t seed, double * out, int64_t n);
bool generate_matrix(int32_t kind, int32_t rows, int32_t cols, uint64_t seed, double * out,
                     std::string * why);
bool lloyd_max(int32_t bits, int32_t block, std::vector<double> * centroids,
               std::string * why);

// Number of context splits per (batch, kv head) used by decode; depends on
// the current device's SM count.
int32_t decode_splits(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                      int32_t head_dim);
int32_t device_sm_count();

// Raise `func`'s dynamic shared-memory limit on the current device to at least
// `bytes`.  The largest value set per (kernel, device) is remembered under a
// lock, so calls from several host threads (e.g. one per device) are safe and
// the attribute is set at most once per size increase.  Returns a cudaError_t.
int ensure_dynamic_smem(const void * func, int bytes);

// Kernel-side parameter blocks ------------------------------------------------

constexpr int kBlock = 32;       // coordinates per norm block
constexpr int kMaxLevels = 16;   // 2^4 centroids

struct CodebookParams {
    float centroid[kMaxLevels];        // ascending, 2^bits valid
    float pos_boundary[kMaxLevels / 2];  // boundaries > 0, ascending, 2^(bits-1) - 1 valid
};

// Uniform-grid search table for the quantizer.  Cells of width w (a power of
// two below the smallest gap between boundaries) tile [-1 - w/2, 1 + w/2]; the
// cell of u is read straight from the bits of y = fmaf(u, scale, offset):
// the offset is an exact integer in [2^23, 2^24), so the FMA's one rounding
// puts 128 * (cell index) + (sub-cell fraction) in the mantissa and
// bits(y) & mask is the byte offset of the cell's 128-byte table row (one
// copy of the entry per lane slot).  code(u) = base[c] + (u >= t[c]) with
// t[c] the one boundary inside the cell (+inf if none).  Entry 0 covers
// u < -1 - w/2 and NaN (whose bits mask to 0).
constexpr int kSearchMax = 128;
struct SearchTable {
    float scale;      // 128 / w
    float offset;     // 2^23 + 128 (1/w + 1) + 64
    uint32_t mask;    // (table size - 1) << 7
    uint32_t size;
    float t[kSearchMax];
    int32_t base[kSearchMax];
};
bool build_search_table(int bits, const float * boundaries, SearchTable * out, std::string * why);

struct WhtParams {
    uint32_t d1_bits[8];
    uint32_t d2_bits[8];
};

struct QuantizeArgs {
    const void * x;
    int64_t n_rows;
    uint32_t * codes;
    uint16_t * norms;
    uint32_t * qjl_signs;
    uint16_t * qjl_rnorm;
    uint32_t * status;
    const float * rot_f32;      // HAAR
    const uint16_t * rot_hi;    // HAAR bf16 split
    const uint16_t * rot_lo;
    const float * qjl_f32;      // GAUSS m x d
    const uint16_t * qjl_hi;
    const uint16_t * qjl_lo;
    int32_t qjl_m;
    float inv_sqrt_d;
    // format variants (register kernels only): norm block size in
    // coordinates, fp32 norms, norm correction with the squared centroids
    int32_t norm_block;
    int32_t norm_f32;
    int32_t norm_corr;
    float centroid_sq[16];
    float boundary[16];         // ascending decision boundaries (variants' binary search)
    int32_t grouped;            // codes in the lane-grouped row order (tensor-core kernel, d = 128)
};

struct AttnArgs {
    const void * q;
    int32_t q_bf16;
    int32_t batch, n_q_heads, n_kv_heads, head_dim;
    int64_t ctx;
    const uint32_t * k_codes;
    const uint16_t * k_norms;
    const uint32_t * qjl_signs;
    const uint16_t * qjl_rnorm;
    const uint32_t * v_codes;
    const uint16_t * v_norms;
    int32_t v_grouped;          // value codes in the lane-grouped row order (d = 128)
    int32_t k_bits, v_bits;
    int32_t rot_kind;
    const float * rot_f32;      // HAAR (d x d)
    const float * qjl_f32;      // GAUSS (m x d)
    int32_t qjl_m;
    float scale;
    float * logits;
    float * out;
    void * workspace;
    int32_t n_splits;
    // warp-range decode (tensor-core path): the partial slots of a query head
    // are the warps whose slab ranges meet its (batch, kv head, group)
    int32_t mma_mode;
    int32_t mma_warps;          // warps of the persistent grid
    int32_t mma_groups;         // head groups of four per kv head
    int64_t mma_slabs;          // 16-token slabs over all (batch, kv head, group)
    int64_t mma_spb;            // slabs per (batch, kv head, group)
    uint32_t * mma_qfrag;       // rotated-query fragments, inside the workspace
    int32_t mma_qwords;         // fragment words per lane and group
    int32_t mma_lut_off;        // dynamic shared offset of the pair tables
    int32_t mma_ring_a;         // warps whose staging ring sits below the tables
    int32_t norm_block;         // coordinates per stored norm (32, 64, 128)
    int32_t norm_f32;           // norms stored as fp32
    // paged cache (tensor-core decode): 0 = flat [b][hk][ctx] rows; else
    // pages of page_size = 2^page_shift tokens, rows [page][kv head][token],
    // block_table[b * max_pages + j] = page of tokens [j P, (j + 1) P)
    int32_t page_size, page_shift, max_pages, n_pages;
    const int32_t * block_table;
    int32_t mma_wait_first;     // the prep kernel writes rows the decode reads
};

// Decode-time append (prep kernel of the tensor-core decode): quantize the
// new token's K and V rows of every (batch, kv head) and store them at token
// ctx - 1 of the cache before attention reads it.
struct AppendParams {
    int32_t enabled;
    int32_t kv_bf16;            // new rows are bf16 (else fp32)
    const void * k_new;         // [batch][n_kv_heads][head_dim]
    const void * v_new;
    uint32_t * k_codes;         // the cache the decode reads (writable)
    uint16_t * k_norms;
    uint32_t * v_codes;
    uint16_t * v_norms;
    uint32_t * status;          // TQ_STATUS_* (may be NULL)
    float k_bound[kMaxLevels];  // ascending decision boundaries (2^bits - 1)
    float v_bound[kMaxLevels];
};

// 2-D tiled tensor map (TMA) over `base` with `inner` elements of `dtype` per
// row, `outer` rows `stride` bytes apart, boxes of box_inner x box_outer;
// false if the driver entry point is unavailable or rejects the map.
bool encode_tensor_map_2d(CUtensorMap * map, CUtensorMapDataType dtype, const void * base,
                          uint64_t inner, uint64_t outer, uint64_t stride, uint32_t box_inner,
                          uint32_t box_outer, CUtensorMapSwizzle swizzle);

// Warp-range decode plan (tq_attention.cu): whether the tensor-core path
// applies, its grid and the partial slots per query head.
// Workspace: [partials (rounded to 256 B)][query fragments].
struct MmaDecodePlan {
    bool ok;
    int32_t ctas, warps_per_cta, warps, groups, slots, qfrag_words;
    int64_t slabs, spb;
    size_t smem_bytes, partial_bytes, qfrag_bytes;
};
// qjl_m = 0 for keys without QJL signs.
MmaDecodePlan plan_mma_decode(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                              int32_t head_dim, int32_t k_bits, int32_t v_bits, int32_t qjl_m,
                              bool paged = false);

// Launchers (tq_quantize.cu, tq_attention.cu).  Return cudaError_t as int.
int launch_quantize(const tq_rotation * rot, const tq_rotation * qjl, int bits, bool bf16,
                    int head_dim, const CodebookParams & cb, const SearchTable & tab,
                    const QuantizeArgs & a, void * stream);
int launch_logits(const tq_rotation * rot, const CodebookParams & kcb, const AttnArgs & a,
                  void * stream);
int launch_decode(const tq_rotation * rot, const CodebookParams & kcb,
                  const CodebookParams & vcb, const AttnArgs & a, void * stream,
                  const AppendParams * ap = nullptr);
size_t decode_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t n_splits,
                              int32_t head_dim);
// Workspace bytes tq_decode_attention needs for exactly these bit widths and
// key kind on the current device (tq_decode_workspace_size is the maximum
// over bit widths); qjl_m = -1 for formats only the CUDA-core path reads.
size_t decode_need_bytes(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                         int32_t head_dim, int32_t k_bits, int32_t v_bits, int32_t qjl_m);
size_t qrot_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t head_dim, int32_t qjl_m);

// Inner-product search (tq_attention.cu): workspace bytes and launch.  `a`
// carries the queries (n_q_heads of them, batch = n_kv_heads = 1), the
// database (k_codes / k_norms, ctx rows), k_bits, the rotation and the
// workspace.
size_t search_workspace_bytes(int32_t n_queries, int64_t n_db, int32_t head_dim, int32_t k);
int launch_search(const tq_rotation * rot, const CodebookParams & kcb, const AttnArgs & a,
                  int32_t k, float * top_scores, int32_t * top_rows, void * stream);

}  // namespace tq
