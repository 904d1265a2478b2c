// Attention over the packed cache (sm_100a): raw logits and split-context
// decode with a combine step.
//
// "TurboQuant+ upstream guide", sec. 5.3: the rotation is fixed and shared,
// so <q, R^T c[idx]> = <R q, c[idx]> -- each CTA rotates its query heads once
// and scores the packed keys in the rotated frame with a centroid lookup times
// the block norm; the value sum is accumulated in the rotated frame and
// rotated back once (sec. 6.1, the inverse-rotation fix).  "Google TurboQuant
// deep dive", sec. 4.3: softmax(Q K^T / sqrt(d)) V; sec. 2.2: the QJL term
// sqrt(pi/2)/m * rho * sum_i (S q)_i (2 s_i - 1) estimates the residual's
// contribution with a full-precision query.
//
// Decode decomposition: grid = (context splits, batch * kv heads).  Each CTA
// streams one contiguous token range of one (batch, kv head), keeps an online
// softmax (running max and sum, base-2 exponentials) for the G query heads of
// the group, and writes a partial (max, sum, unnormalised rotated output).  A
// second launch merges the splits and applies R^T.

#include <cuda_runtime.h>
#include <math_constants.h>

#include "tq_device.cuh"

namespace tq {

namespace {

constexpr int kThreads = 128;
constexpr int kMaxGroup = 8;
constexpr int kMaxDim = 256;
constexpr int kMaxQjl = 256;
constexpr int kLogitTokensPerCta = 2048;
constexpr float kLog2e = 1.4426950408889634f;

struct RotParams {
    uint32_t d1_bits[8];
    uint32_t d2_bits[8];
};

__device__ __forceinline__ float sign_of(const uint32_t * bits, int i) {
    return ((bits[i >> 5] >> (i & 31)) & 1u) ? -1.0f : 1.0f;
}

// In-place unnormalised Walsh-Hadamard transform of `n` vectors of length d
// stored back to back in shared memory (natural order).
__device__ void smem_fwht(float * v, int d, int n) {
    for (int h = 1; h < d; h <<= 1) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * d / 2; idx += blockDim.x) {
            const int vec = idx / (d / 2);
            const int k = idx % (d / 2);
            const int i = (k / h) * 2 * h + (k % h);
            float * base = v + vec * d;
            const float a = base[i], b = base[i + h];
            base[i] = a + b;
            base[i + h] = a - b;
        }
    }
    __syncthreads();
}

// q_rot[g][:] = R q[b][h0 + g][:] for g < G, into shared memory (fp32).
__device__ void rotate_queries(const AttnArgs & a, const RotParams & rp, int b, int h0, int G,
                               float * q_rot) {
    const int d = a.head_dim;
    for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
        const int g = idx / d, i = idx % d;
        const int64_t off = ((int64_t)b * a.n_q_heads + h0 + g) * d + i;
        float v = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.q)[off])
                           : static_cast<const float *>(a.q)[off];
        if (a.rot_kind == TQ_ROT_WHT) v *= sign_of(rp.d2_bits, i);
        q_rot[idx] = v;
    }
    if (a.rot_kind == TQ_ROT_WHT) {
        smem_fwht(q_rot, d, G);
        const float sc = rsqrtf((float)d);
        for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x)
            q_rot[idx] *= sc * sign_of(rp.d1_bits, idx % d);
        __syncthreads();
    } else {
        // dense: stage the raw queries, then q_rot = P q
        __shared__ float q_raw[kMaxGroup * kMaxDim];
        __syncthreads();
        for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) q_raw[idx] = q_rot[idx];
        __syncthreads();
        for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
            const int g = idx / d, e = idx % d;
            const float * pr = a.rot_f32 + (int64_t)e * d;
            float acc = 0.0f;
            for (int i = 0; i < d; ++i) acc = fmaf(pr[i], q_raw[g * d + i], acc);
            q_rot[idx] = acc;
        }
        __syncthreads();
    }
}

// w[g][i] = (S q_rot[g])_i for the QJL projection S (m x d, fp32 in global).
__device__ void project_queries(const AttnArgs & a, int G, const float * q_rot, float * w) {
    const int d = a.head_dim, m = a.qjl_m;
    for (int idx = threadIdx.x; idx < G * m; idx += blockDim.x) {
        const int g = idx / m, i = idx % m;
        const float * sr = a.qjl_f32 + (int64_t)i * d;
        float acc = 0.0f;
        for (int j = 0; j < d; ++j) acc = fmaf(sr[j], q_rot[g * d + j], acc);
        w[idx] = acc;
    }
    __syncthreads();
}

// Raw score of token row `row` for the G heads: sum_k gamma_k sum_j q_j c[idx_j]
// (+ QJL term).  Generic in BITS through extract_code.
template <int BITS>
__device__ __forceinline__ void score_row(const AttnArgs & a, int64_t row, int G,
                                          const float * q_rot, const float * lut,
                                          const float * w_qjl, float * s) {
    const int d = a.head_dim;
    const int nb = d / 32;
    const uint32_t * cw = a.k_codes + row * (int64_t)(nb * BITS);
    const uint16_t * nw = a.k_norms + row * nb;
    for (int g = 0; g < G; ++g) s[g] = 0.0f;
    for (int k = 0; k < nb; ++k) {
        uint32_t words[BITS];
#pragma unroll
        for (int i = 0; i < BITS; ++i) words[i] = cw[k * BITS + i];
        float part[kMaxGroup];
        for (int g = 0; g < G; ++g) part[g] = 0.0f;
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
            const float c = lut[extract_code<BITS>(words, j)];
            for (int g = 0; g < G; ++g) part[g] = fmaf(q_rot[g * d + k * 32 + j], c, part[g]);
        }
        const float gam = half_bits_to_float(nw[k]);
        for (int g = 0; g < G; ++g) s[g] = fmaf(gam, part[g], s[g]);
    }
    if (a.qjl_signs != nullptr) {
        const int m = a.qjl_m;
        const uint32_t * sw = a.qjl_signs + row * (int64_t)(m / 32);
        const float rho = half_bits_to_float(a.qjl_rnorm[row]);
        const float coef = 1.2533141373155003f / (float)m * rho;  // sqrt(pi/2)/m * rho
        for (int g = 0; g < G; ++g) {
            float acc = 0.0f;
            for (int wi = 0; wi < m / 32; ++wi) {
                const uint32_t bits = sw[wi];
                for (int i = 0; i < 32; ++i) {
                    const float wv = w_qjl[g * m + wi * 32 + i];
                    acc += ((bits >> i) & 1u) ? wv : -wv;
                }
            }
            s[g] = fmaf(coef, acc, s[g]);
        }
    }
}

template <int KBITS>
__global__ void __launch_bounds__(kThreads)
logits_simple_kernel(const AttnArgs a, const CodebookParams kcb, const RotParams rp) {
    __shared__ float q_rot[kMaxGroup * kMaxDim];
    __shared__ float w_qjl[kMaxGroup * kMaxQjl];
    __shared__ float lut[16];
    const int G = a.n_q_heads / a.n_kv_heads;
    const int bh = blockIdx.y;
    const int b = bh / a.n_kv_heads, hk = bh % a.n_kv_heads;
    if (threadIdx.x < (1 << KBITS)) lut[threadIdx.x] = kcb.centroid[threadIdx.x];
    rotate_queries(a, rp, b, hk * G, G, q_rot);
    if (a.qjl_signs != nullptr) project_queries(a, G, q_rot, w_qjl);
    const int64_t t0 = (int64_t)blockIdx.x * kLogitTokensPerCta;
    const int64_t t1 = min(a.ctx, t0 + kLogitTokensPerCta);
    for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int64_t row = (int64_t)bh * a.ctx + t;
        float s[kMaxGroup];
        score_row<KBITS>(a, row, G, q_rot, lut, w_qjl, s);
        for (int g = 0; g < G; ++g)
            a.logits[((int64_t)b * a.n_q_heads + hk * G + g) * a.ctx + t] = s[g];
    }
}

__device__ __forceinline__ float block_max(float v, float * red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    return r;
}

__device__ __forceinline__ float block_sum(float v, float * red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += red[w];
    return r;
}

// Partial workspace layout (floats): o[(b*Hq + h) * S + s][d], then
// ml[(b*Hq + h) * S + s][2] = (max in log2 units, sum).
template <int KBITS, int VBITS>
__global__ void __launch_bounds__(kThreads)
decode_split_simple_kernel(const AttnArgs a, const CodebookParams kcb, const CodebookParams vcb,
                           const RotParams rp) {
    __shared__ float q_rot[kMaxGroup * kMaxDim];
    __shared__ float w_qjl[kMaxGroup * kMaxQjl];
    __shared__ float klut[16], vlut[16];
    __shared__ float p_s[kMaxGroup][kThreads];
    __shared__ float red[kThreads / 32];
    const int G = a.n_q_heads / a.n_kv_heads;
    const int d = a.head_dim, nb = d / 32;
    const int S = a.n_splits;
    const int split = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / a.n_kv_heads, hk = bh % a.n_kv_heads;
    if (threadIdx.x < 16) {
        klut[threadIdx.x] = kcb.centroid[threadIdx.x];
        vlut[threadIdx.x] = vcb.centroid[threadIdx.x];
    }
    rotate_queries(a, rp, b, hk * G, G, q_rot);
    if (a.qjl_signs != nullptr) project_queries(a, G, q_rot, w_qjl);

    const int64_t chunk = ((a.ctx + S - 1) / S + kThreads - 1) / kThreads * kThreads;
    const int64_t t0 = (int64_t)split * chunk;
    const int64_t t1 = min(a.ctx, t0 + chunk);
    const float sl2 = a.scale * kLog2e;

    float m_run[kMaxGroup], l_run[kMaxGroup];
    float o[kMaxGroup][kMaxDim / kThreads];
    for (int g = 0; g < kMaxGroup; ++g) {
        m_run[g] = -CUDART_INF_F;
        l_run[g] = 0.0f;
        for (int k = 0; k < kMaxDim / kThreads; ++k) o[g][k] = 0.0f;
    }
    for (int64_t tb = t0; tb < t1; tb += kThreads) {
        const int64_t t = tb + threadIdx.x;
        const bool valid = t < t1;
        float s[kMaxGroup];
        if (valid) {
            score_row<KBITS>(a, (int64_t)bh * a.ctx + t, G, q_rot, klut, w_qjl, s);
            for (int g = 0; g < G; ++g) s[g] *= sl2;
        } else {
            for (int g = 0; g < G; ++g) s[g] = -CUDART_INF_F;
        }
        for (int g = 0; g < G; ++g) {
            const float mt = block_max(s[g], red);
            const float m_new = fmaxf(m_run[g], mt);
            const float alpha = exp2f(m_run[g] - m_new);   // 0 when m_run = -inf
            const float p = valid ? exp2f(s[g] - m_new) : 0.0f;
            p_s[g][threadIdx.x] = p;
            const float ps = block_sum(p, red);
            l_run[g] = l_run[g] * alpha + ps;
            m_run[g] = m_new;
            for (int k = 0; k < kMaxDim / kThreads; ++k) o[g][k] *= alpha;
        }
        __syncthreads();
        const int n_tok = (int)min((int64_t)kThreads, t1 - tb);
        for (int k = 0; k * kThreads < d; ++k) {
            const int j = k * kThreads + threadIdx.x;
            if (j >= d) break;
            const int blk = j >> 5, jj = j & 31;
            for (int i = 0; i < n_tok; ++i) {
                const int64_t row = (int64_t)bh * a.ctx + tb + i;
                const uint32_t * vw = a.v_codes + row * (int64_t)(nb * VBITS) + blk * VBITS;
                const float c = vlut[extract_code<VBITS>(vw, jj)];
                const float vg = half_bits_to_float(a.v_norms[row * nb + blk]) * c;
                for (int g = 0; g < G; ++g) o[g][k] = fmaf(p_s[g][i], vg, o[g][k]);
            }
        }
        __syncthreads();
    }
    float * ws = static_cast<float *>(a.workspace);
    const int64_t n_part = (int64_t)a.batch * a.n_q_heads * S;
    for (int g = 0; g < G; ++g) {
        const int64_t pidx = ((int64_t)b * a.n_q_heads + hk * G + g) * S + split;
        for (int k = 0; k * kThreads < d; ++k) {
            const int j = k * kThreads + threadIdx.x;
            if (j < d) ws[pidx * d + j] = o[g][k];
        }
        if (threadIdx.x == 0) {
            ws[n_part * d + 2 * pidx] = m_run[g];
            ws[n_part * d + 2 * pidx + 1] = l_run[g];
        }
    }
}

__global__ void __launch_bounds__(kThreads)
decode_combine_kernel(const AttnArgs a, const RotParams rp) {
    __shared__ float o_s[kMaxDim];
    __shared__ float o_raw[kMaxDim];
    const int d = a.head_dim;
    const int S = a.n_splits;
    const int64_t bhq = blockIdx.x;  // b * Hq + h
    const float * ws = static_cast<const float *>(a.workspace);
    const int64_t n_part = (int64_t)a.batch * a.n_q_heads * S;
    const float * ml = ws + n_part * d;
    float M = -CUDART_INF_F;
    for (int s = 0; s < S; ++s) M = fmaxf(M, ml[2 * (bhq * S + s)]);
    float L = 0.0f;
    for (int s = 0; s < S; ++s) {
        const float ms = ml[2 * (bhq * S + s)];
        if (ms != -CUDART_INF_F) L += exp2f(ms - M) * ml[2 * (bhq * S + s) + 1];
    }
    const float inv_l = 1.0f / L;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        float acc = 0.0f;
        for (int s = 0; s < S; ++s) {
            const float ms = ml[2 * (bhq * S + s)];
            if (ms != -CUDART_INF_F) acc = fmaf(exp2f(ms - M), ws[(bhq * S + s) * d + j], acc);
        }
        o_s[j] = acc * inv_l;
    }
    __syncthreads();
    if (a.rot_kind == TQ_ROT_WHT) {
        // R^T = d^-1/2 D2 H D1
        for (int j = threadIdx.x; j < d; j += blockDim.x) o_s[j] *= sign_of(rp.d1_bits, j);
        smem_fwht(o_s, d, 1);
        const float sc = rsqrtf((float)d);
        for (int j = threadIdx.x; j < d; j += blockDim.x)
            a.out[bhq * d + j] = o_s[j] * sc * sign_of(rp.d2_bits, j);
    } else {
        for (int j = threadIdx.x; j < d; j += blockDim.x) o_raw[j] = o_s[j];
        __syncthreads();
        for (int i = threadIdx.x; i < d; i += blockDim.x) {
            float acc = 0.0f;
            for (int e = 0; e < d; ++e) acc = fmaf(a.rot_f32[(int64_t)e * d + i], o_raw[e], acc);
            a.out[bhq * d + i] = acc;
        }
    }
}

// ---------------------------------------------------------------------------
// Fast split decode (CUDA cores).  One CTA = 8 warps streams 128-token tiles
// of one (batch, kv head) for four query heads (a group of up to four of the
// G heads that share the kv head; missing heads are zero queries).
//
//  * staging: cp.async copies each tile's K codes, K norms, V codes and V
//    norms into shared memory, double buffered.  K codes are stored block
//    major ([block][token][words]) so that the 32 lanes of a warp, which read
//    one block of 32 consecutive tokens, hit distinct banks.
//  * logits: a thread scores TL tokens on one 32-coordinate block; code
//    pairs index a pair table {c[lo], c[hi]} and feed f32x2 FMAs against the
//    rotated query pairs of the four heads (shared-memory broadcast).  The
//    pair tables hold one copy per lane of a half warp, laid out so that
//    every lane reads its own banks: lookups never conflict.
//  * softmax: one thread per token sums the block partials (each already
//    scaled by its fp16 block norm), the CTA keeps a running max per head
//    (base-2 exponentials) and the per-token weights p * norm_V are staged for
//    the value pass.
//  * values: warp w owns block w mod NB; a lane owns 8 coordinates of it for
//    the four heads (32 fp32 accumulators, as f32x2 pairs) and walks one
//    token of every 8; pair lookups again feed f32x2 FMAs.
// ---------------------------------------------------------------------------

constexpr int kFastThreads = 256;
constexpr int kFastWarps = kFastThreads / 32;
constexpr int kTile = 128;
constexpr int kQH = 4;        // query heads per CTA
constexpr int kCopies = 16;   // pair-table copies (lanes of a half warp)

template <int D, int KB, int VB>
struct Fast {
    static constexpr int NB = D / 32;
    static constexpr int KW = NB * KB;               // K code words per row
    static constexpr int VW = NB * VB;               // V code words per row
    static constexpr int SLOTS = kFastThreads / NB;  // logit token slots
    static constexpr int TL = kTile / SLOTS;         // tokens per thread (logits)
    static constexpr int KLUT = 1 << (2 * KB);
    static constexpr int VLUT = 1 << (2 * VB);
    static constexpr int WPB = kFastWarps / NB;      // warps per block (values)
    static constexpr int VTOK = kTile / WPB;         // tokens per warp (values)
    static constexpr int VSTEP = VTOK / 8;
    static constexpr int WSTRIDE = NB * 8 + 4;       // floats per token in wbuf (padded)
    // shared memory layout, byte offsets (all multiples of 16)
    static constexpr int OFF_KLUT = 0;                          // {hi, lo} half2 x 16 copies
    static constexpr int OFF_VLUT = OFF_KLUT + KLUT * kCopies * 8;
    static constexpr int OFF_Q = OFF_VLUT + VLUT * kCopies * 8;
    static constexpr int SZ_KC = kTile * KW * 4;                // row-major (KB = 4: swizzled)
    static constexpr int SZ_KN = kTile * NB * 2;
    static constexpr int SZ_VC = kTile * VW * 4;
    static constexpr int SZ_VN = kTile * NB * 2;
    static constexpr int SZ_STAGE = SZ_KC + SZ_KN + SZ_VC + SZ_VN;
    static constexpr int OFF_STAGE = OFF_Q + D * 16;
    static constexpr int OFF_PART = OFF_STAGE + 2 * SZ_STAGE;
    static constexpr int OFF_W = OFF_PART + kTile * 16;
    static constexpr int SZ_W = kTile * WSTRIDE * 4;
    static constexpr int OFF_RED = OFF_W + (SZ_W > WPB * kQH * D * 4 ? SZ_W : WPB * kQH * D * 4);
    static constexpr int SMEM = OFF_RED + kFastWarps * kQH * 4 + 16;
    static_assert(SZ_KC % 16 == 0 && SZ_KN % 16 == 0 && SZ_VC % 16 == 0 && SZ_VN % 16 == 0, "align");
    static_assert(TL >= 1 && VSTEP >= 1, "tile");
};

template <int W>
__device__ __forceinline__ uint32_t bits_at(const uint32_t * words, int p) {
    // W-bit field starting at bit p of a little-endian word stream
    const int wi = p >> 5, sh = p & 31;
    uint32_t v = words[wi] >> sh;
    if (sh + W > 32) v |= words[wi + 1] << (32 - sh);
    return v & ((1u << W) - 1u);
}

__device__ __forceinline__ void cp_async(void * smem_dst, const void * gmem_src, int bytes) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    if (bytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src));
    else if (bytes == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(gmem_src));
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gmem_src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

// Chunk swizzle for 4-bit K code rows (NB 16-byte chunks per row).
template <int NB>
__device__ __forceinline__ int kswz(int t) {
    return (t / (8 / NB)) & (NB - 1);
}

// Issue the copies of one tile (tokens [t0, t0 + n) of row block `row0`).
template <int D, int KB, int VB>
__device__ __forceinline__ void stage_tile(const AttnArgs & a, unsigned char * st, int64_t row0,
                                           int n) {
    using F = Fast<D, KB, VB>;
    constexpr int NB = F::NB;
    uint32_t * kc = reinterpret_cast<uint32_t *>(st);
    uint16_t * kn = reinterpret_cast<uint16_t *>(st + F::SZ_KC);
    uint32_t * vc = reinterpret_cast<uint32_t *>(st + F::SZ_KC + F::SZ_KN);
    uint16_t * vn = reinterpret_cast<uint16_t *>(st + F::SZ_KC + F::SZ_KN + F::SZ_VC);
    const int tid = threadIdx.x;
    // K codes, row major in 16-byte chunks.  For 4-bit codes a chunk is one
    // block; chunk blk of token t is stored at chunk blk ^ kswz(t) so that
    // the tensor-core fragment loads (8 tokens x 4 words) hit distinct banks.
    constexpr int KCB = (F::KW * 4) % 16 == 0 ? 16 : ((F::KW * 4) % 8 == 0 ? 8 : 4);
    constexpr int KCH = F::KW * 4 / KCB;
    for (int idx = tid; idx < KCH * kTile; idx += kFastThreads) {
        const int t = idx / KCH, ch = idx % KCH;
        const int slot = (KB == 4) ? (ch ^ kswz<NB>(t)) : ch;
        if (t < n)
            cp_async(reinterpret_cast<unsigned char *>(kc) + t * F::KW * 4 + slot * KCB,
                     reinterpret_cast<const unsigned char *>(a.k_codes + (row0 + t) * F::KW) + ch * KCB,
                     KCB);
    }
    // V codes, row major, in the largest chunk the row size allows.
    constexpr int VCB = (F::VW * 4) % 16 == 0 ? 16 : ((F::VW * 4) % 8 == 0 ? 8 : 4);
    constexpr int VCH = F::VW * 4 / VCB;
    for (int idx = tid; idx < VCH * kTile; idx += kFastThreads) {
        const int t = idx / VCH, ch = idx % VCH;
        if (t < n)
            cp_async(reinterpret_cast<unsigned char *>(vc) + t * F::VW * 4 + ch * VCB,
                     reinterpret_cast<const unsigned char *>(a.v_codes + (row0 + t) * F::VW) + ch * VCB, VCB);
    }
    // norms: NB halves per token (4, 8 or 16 bytes)
    for (int idx = tid; idx < 2 * kTile; idx += kFastThreads) {
        const int t = idx % kTile;
        if (t >= n) continue;
        if (idx < kTile)
            cp_async(kn + t * NB, a.k_norms + (row0 + t) * NB, NB * 2);
        else
            cp_async(vn + t * NB, a.v_norms + (row0 + t) * NB, NB * 2);
    }
}


// Shared-window byte address of table entry `e` for this lane's copy
// (entries are 16 float2 = 128 bytes apart; `lane_base` already holds the
// table's shared address plus 8 * (lane & 15)).
__device__ __forceinline__ uint32_t lut_addr(uint32_t e, uint32_t lane_base) {
    return e * 128u + lane_base;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}

// Pair field p (two W-bit codes, 2W bits) of a block's little-endian words.
// Byte-aligned fields (W = 4) come out with one byte permute.
template <int W>
__device__ __forceinline__ uint32_t pair_field(const uint32_t * words, int p) {
    if constexpr (W == 4) {
        return __byte_perm(words[p >> 2], 0u, 0x4440u | (uint32_t)(p & 3));
    } else {
        return bits_at<2 * W>(words, 2 * W * p);
    }
}

template <int D, int KB, int VB>
__global__ void __launch_bounds__(kFastThreads, 2)
decode_split_fast_kernel(const __grid_constant__ AttnArgs a,
                         const __grid_constant__ CodebookParams kcb,
                         const __grid_constant__ CodebookParams vcb,
                         const __grid_constant__ RotParams rp) {
    using F = Fast<D, KB, VB>;
    constexpr int NB = F::NB;
    extern __shared__ __align__(16) unsigned char smem[];
    uint2 * klut = reinterpret_cast<uint2 *>(smem + F::OFF_KLUT);   // {hi, lo} half2, 16 copies
    float2 * vlut = reinterpret_cast<float2 *>(smem + F::OFF_VLUT);
    float4 * part = reinterpret_cast<float4 *>(smem + F::OFF_PART);
    float * wbuf = reinterpret_cast<float *>(smem + F::OFF_W);
    float * red = reinterpret_cast<float *>(smem + F::OFF_RED);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int HG = (G + kQH - 1) / kQH;
    const int split = blockIdx.x;
    const int bhg = blockIdx.y;
    const int hg = bhg % HG;
    const int bh = bhg / HG;
    const int b = bh / a.n_kv_heads, hk = bh % a.n_kv_heads;
    const int h0 = hk * G + hg * kQH;               // first query head of this CTA
    const int nh = min(kQH, G - hg * kQH);          // real heads here

    // K pair table for the tensor cores: each centroid as an fp16 high part
    // and an fp16 low part (c - hi), so that hi + lo carries ~22 bits; entry
    // e, copy c at uint2 index e * 16 + c = {hi pair, lo pair}.  V pair table
    // as fp32 pairs: entry e, copy c at float2 index e * 16 + c.
    for (int i = tid; i < F::KLUT * kCopies; i += kFastThreads) {
        const int e = i / kCopies;
        const float c0 = kcb.centroid[e & ((1 << KB) - 1)], c1 = kcb.centroid[e >> KB];
        const __half2 hi = __floats2half2_rn(c0, c1);
        const __half2 lo = __floats2half2_rn(c0 - __low2float(hi), c1 - __high2float(hi));
        klut[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&hi),
                             *reinterpret_cast<const uint32_t *>(&lo));
    }
    for (int i = tid; i < F::VLUT * kCopies; i += kFastThreads) {
        const int e = i / kCopies;
        vlut[i] = make_float2(vcb.centroid[e & ((1 << VB) - 1)], vcb.centroid[e >> VB]);
    }
    // rotated queries (scratch in the wbuf region), then B fragments
    uint32_t qb[NB][2][2];
    {
        float * qr = wbuf;   // [kQH][D]
        for (int idx = tid; idx < kQH * D; idx += kFastThreads) {
            const int g = idx / D, i = idx % D;
            float v = 0.0f;
            if (g < nh) {
                const int64_t off = ((int64_t)b * a.n_q_heads + h0 + g) * D + i;
                v = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.q)[off])
                             : static_cast<const float *>(a.q)[off];
                if (a.rot_kind == TQ_ROT_WHT) v *= sign_of(rp.d2_bits, i);
            }
            qr[idx] = v;
        }
        if (a.rot_kind == TQ_ROT_WHT) {
            smem_fwht(qr, D, kQH);
            const float sc = rsqrtf((float)D);
            for (int idx = tid; idx < kQH * D; idx += kFastThreads) qr[idx] *= sc * sign_of(rp.d1_bits, idx % D);
            __syncthreads();
        } else {
            float * qd = wbuf + kQH * D;   // dense: q_rot = P q
            for (int idx = tid; idx < kQH * D; idx += kFastThreads) {
                const int g = idx / D, e = idx % D;
                const float * pr = a.rot_f32 + (int64_t)e * D;
                float acc = 0.0f;
                for (int i = 0; i < D; ++i) acc = fmaf(pr[i], qr[g * D + i], acc);
                qd[idx] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < kQH * D; idx += kFastThreads) qr[idx] = qd[idx];
            __syncthreads();
        }
        // Tensor-core B fragments of the rotated query (m16n8k16, column n =
        // lane / 4 is head n % 4, fp16 high part for n < 4, low part for
        // n >= 4).  Block blk, k-step s: the thread's k slots (2c, 2c + 1) and
        // (2c + 8, 2c + 9) hold dims 32 blk + 8c + 4s + {0, 1} and {2, 3}.
        {
            const int n = lane >> 2, c = lane & 3;
            const float * qh = qr + (n & 3) * D;
#pragma unroll
            for (int blk = 0; blk < NB; ++blk)
#pragma unroll
                for (int st2 = 0; st2 < 2; ++st2)
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int dim = 32 * blk + 8 * c + 4 * st2 + 2 * r;
                        const float x0 = qh[dim], x1 = qh[dim + 1];
                        const __half2 hi = __floats2half2_rn(x0, x1);
                        __half2 v = hi;
                        if (n >= 4) v = __floats2half2_rn(x0 - __low2float(hi), x1 - __high2float(hi));
                        qb[blk][st2][r] = *reinterpret_cast<const uint32_t *>(&v);
                    }
        }
        __syncthreads();
    }

    // token range of this split
    const int64_t chunk = ((a.ctx + a.n_splits - 1) / a.n_splits + kTile - 1) / kTile * kTile;
    const int64_t t_begin = (int64_t)split * chunk;
    const int64_t t_end = min(a.ctx, t_begin + chunk);
    const int n_tiles = t_end > t_begin ? (int)((t_end - t_begin + kTile - 1) / kTile) : 0;
    const int64_t row_base = (int64_t)bh * a.ctx;
    const float sl2 = a.scale * kLog2e;

    // per-thread state
    float m_run[kQH], l_tok[kQH];
#pragma unroll
    for (int h = 0; h < kQH; ++h) { m_run[h] = -CUDART_INF_F; l_tok[h] = 0.0f; }
    float2 acc_v[kQH][4];
#pragma unroll
    for (int h = 0; h < kQH; ++h)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc_v[h][k] = make_float2(0.0f, 0.0f);

    // lane roles
    const int lam = lane & 15;
    const uint32_t klut_lane = (uint32_t)__cvta_generic_to_shared(klut) + 8u * (uint32_t)lam;
    const uint32_t vlut_lane = (uint32_t)__cvta_generic_to_shared(vlut) + 8u * (uint32_t)lam;
    const int kg = lane >> 2, kcq = lane & 3;                    // logits (mma fragment)
    const int vblk = warp % NB, vtq = warp / NB;                  // values
    const int vgrp = lane >> 2, vc = lane & 3;

    if (n_tiles > 0) {
        stage_tile<D, KB, VB>(a, smem + F::OFF_STAGE, row_base + t_begin,
                              (int)min((int64_t)kTile, t_end - t_begin));
    }
    cp_async_commit();
    for (int it = 0; it < n_tiles; ++it) {
        const int64_t t0 = t_begin + (int64_t)it * kTile;
        const int n = (int)min((int64_t)kTile, t_end - t0);
        if (it + 1 < n_tiles) {
            const int64_t t1 = t0 + kTile;
            stage_tile<D, KB, VB>(a, smem + F::OFF_STAGE + ((it + 1) & 1) * F::SZ_STAGE,
                                  row_base + t1, (int)min((int64_t)kTile, t_end - t1));
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        unsigned char * st = smem + F::OFF_STAGE + (it & 1) * F::SZ_STAGE;
        const uint32_t * kc = reinterpret_cast<const uint32_t *>(st);
        const uint16_t * kn = reinterpret_cast<const uint16_t *>(st + F::SZ_KC);
        const uint32_t * vcw = reinterpret_cast<const uint32_t *>(st + F::SZ_KC + F::SZ_KN);
        const uint16_t * vn = reinterpret_cast<const uint16_t *>(st + F::SZ_KC + F::SZ_KN + F::SZ_VC);

        // ---- logits on tensor cores: warp w scores tokens 16w .. 16w + 15 ----
        {
            const int t0 = 16 * warp + kg, t1 = t0 + 8;
            float tot[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            // fp16 block norms of both rows
            float g0[NB], g1[NB];
#pragma unroll
            for (int blk = 0; blk < NB; ++blk) {
                g0[blk] = half_bits_to_float(kn[t0 * NB + blk]);
                g1[blk] = half_bits_to_float(kn[t1 * NB + blk]);
            }
#pragma unroll
            for (int blk = 0; blk < NB; ++blk) {
                // the thread's 8 codes of this block (codes 8c .. 8c + 7) for both rows
                uint32_t w0, w1;
                if constexpr (KB == 4) {
                    w0 = kc[t0 * F::KW + 4 * (blk ^ kswz<NB>(t0)) + kcq];
                    w1 = kc[t1 * F::KW + 4 * (blk ^ kswz<NB>(t1)) + kcq];
                } else {
                    const int bo = 8 * KB * kcq;
                    const uint32_t * r0p = kc + t0 * F::KW + blk * KB;
                    const uint32_t * r1p = kc + t1 * F::KW + blk * KB;
                    const int wl = bo >> 5, sh = bo & 31;
                    w0 = __funnelshift_r(r0p[wl], (wl + 1 < KB) ? r0p[wl + 1] : 0u, sh);
                    w1 = __funnelshift_r(r1p[wl], (wl + 1 < KB) ? r1p[wl + 1] : 0u, sh);
                }
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int st2 = 0; st2 < 2; ++st2) {
                    // pair fields 2 st2 and 2 st2 + 1 of the 8 codes
                    uint32_t e[4];
                    if constexpr (KB == 4) {
                        e[0] = __byte_perm(w0, 0u, 0x4440u | (uint32_t)(2 * st2));
                        e[1] = __byte_perm(w1, 0u, 0x4440u | (uint32_t)(2 * st2));
                        e[2] = __byte_perm(w0, 0u, 0x4440u | (uint32_t)(2 * st2 + 1));
                        e[3] = __byte_perm(w1, 0u, 0x4440u | (uint32_t)(2 * st2 + 1));
                    } else {
                        constexpr uint32_t PM = (1u << (2 * KB)) - 1u;
                        e[0] = (w0 >> (2 * KB * (2 * st2))) & PM;
                        e[1] = (w1 >> (2 * KB * (2 * st2))) & PM;
                        e[2] = (w0 >> (2 * KB * (2 * st2 + 1))) & PM;
                        e[3] = (w1 >> (2 * KB * (2 * st2 + 1))) & PM;
                    }
                    uint32_t ah[4], al[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t addr = e[i] * 128u + klut_lane;
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(ah[i]), "=r"(al[i]) : "r"(addr));
                    }
                    asm volatile(
                        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
                        : "r"(ah[0]), "r"(ah[1]), "r"(ah[2]), "r"(ah[3]),
                          "r"(qb[blk][st2][0]), "r"(qb[blk][st2][1]));
                    asm volatile(
                        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
                        : "r"(al[0]), "r"(al[1]), "r"(al[2]), "r"(al[3]),
                          "r"(qb[blk][st2][0]), "r"(qb[blk][st2][1]));
                }
                tot[0] = fmaf(g0[blk], acc[0], tot[0]);
                tot[1] = fmaf(g0[blk], acc[1], tot[1]);
                tot[2] = fmaf(g1[blk], acc[2], tot[2]);
                tot[3] = fmaf(g1[blk], acc[3], tot[3]);
            }
            // columns 2c, 2c+1: heads (2c, 2c+1) high parts for c < 2, low parts
            // for c >= 2; add the partner lane (c ^ 2) to get full scores
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[i] += __shfl_xor_sync(0xffffffffu, tot[i], 2);
            if (kcq < 2) {
                float * pt = reinterpret_cast<float *>(part);
                *reinterpret_cast<float2 *>(pt + t0 * 4 + 2 * kcq) = make_float2(tot[0], tot[1]);
                *reinterpret_cast<float2 *>(pt + t1 * 4 + 2 * kcq) = make_float2(tot[2], tot[3]);
            }
        }
        __syncthreads();

        // ---- softmax: one thread per token ----
        float alpha[kQH];
        {
            const int t = tid;
            const bool valid = t < n;
            float s[kQH];
#pragma unroll
            for (int h = 0; h < kQH; ++h) s[h] = -CUDART_INF_F;
            if (valid) {
                const float4 sum = part[t];
                s[0] = sum.x * sl2; s[1] = sum.y * sl2; s[2] = sum.z * sl2; s[3] = sum.w * sl2;
            }
#pragma unroll
            for (int h = 0; h < kQH; ++h) {
                float v = s[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (lane == 0) red[warp * kQH + h] = v;
            }
            __syncthreads();
            float p[kQH];
#pragma unroll
            for (int h = 0; h < kQH; ++h) {
                float mt = red[h];
#pragma unroll
                for (int w = 1; w < kFastWarps; ++w) mt = fmaxf(mt, red[w * kQH + h]);
                const float m_new = fmaxf(m_run[h], mt);
                alpha[h] = exp2f(m_run[h] - m_new);
                m_run[h] = m_new;
                p[h] = valid ? exp2f(s[h] - m_new) : 0.0f;
                l_tok[h] = l_tok[h] * alpha[h] + p[h];
            }
            if (t < kTile) {
                float * wt = wbuf + t * F::WSTRIDE;
#pragma unroll
                for (int blk = 0; blk < NB; ++blk) {
                    const float gv = valid ? half_bits_to_float(vn[t * NB + blk]) : 0.0f;
                    const float w0 = p[0] * gv, w1 = p[1] * gv, w2 = p[2] * gv, w3 = p[3] * gv;
                    reinterpret_cast<float4 *>(wt + blk * 8)[0] = make_float4(w0, w0, w1, w1);
                    reinterpret_cast<float4 *>(wt + blk * 8)[1] = make_float4(w2, w2, w3, w3);
                }
            }
        }
        __syncthreads();

        // ---- values: warp owns block vblk, lane owns 8 coordinates ----
        {
#pragma unroll
            for (int h = 0; h < kQH; ++h) {
                const float2 al = make_float2(alpha[h], alpha[h]);
#pragma unroll
                for (int k = 0; k < 4; ++k) acc_v[h][k] = __fmul2_rn(acc_v[h][k], al);
            }
            const int bitoff = 8 * VB * vc;             // lane's first code bit in the block
            const int w_lo = bitoff >> 5, sh = bitoff & 31;
#pragma unroll 2
            for (int i = 0; i < F::VSTEP; ++i) {
                const int t = vtq * F::VTOK + vgrp + 8 * i;
                if (t >= n) break;
                const uint32_t * row = vcw + t * F::VW + vblk * VB;
                uint32_t lo = row[w_lo];
                uint32_t hi = (w_lo + 1 < VB) ? row[w_lo + 1] : 0u;
                const uint32_t chunk = __funnelshift_r(lo, hi, sh);    // lane's 8 codes
                const float * wt = wbuf + t * F::WSTRIDE + vblk * 8;
                const float4 wa = reinterpret_cast<const float4 *>(wt)[0];
                const float4 wb = reinterpret_cast<const float4 *>(wt)[1];
                const float2 w0 = make_float2(wa.x, wa.y), w1 = make_float2(wa.z, wa.w);
                const float2 w2 = make_float2(wb.x, wb.y), w3 = make_float2(wb.z, wb.w);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t e = VB == 4 ? __byte_perm(chunk, 0u, 0x4440u | (uint32_t)k)
                                               : (chunk >> (2 * VB * k)) & ((1u << (2 * VB)) - 1u);
                    const float2 vv = lds_f2(lut_addr(e, vlut_lane));
                    acc_v[0][k] = __ffma2_rn(vv, w0, acc_v[0][k]);
                    acc_v[1][k] = __ffma2_rn(vv, w1, acc_v[1][k]);
                    acc_v[2][k] = __ffma2_rn(vv, w2, acc_v[2][k]);
                    acc_v[3][k] = __ffma2_rn(vv, w3, acc_v[3][k]);
                }
            }
        }
        __syncthreads();   // the stage buffer and wbuf are rewritten next
    }
    cp_async_wait<0>();

    // ---- finalize: CTA sums ----
    // running sums: per-token partials -> per head
    float L[kQH];
#pragma unroll
    for (int h = 0; h < kQH; ++h) {
        float v = l_tok[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp * kQH + h] = v;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kQH; ++h) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kFastWarps; ++w) v += red[w * kQH + h];
        L[h] = v;
    }
    // value accumulators: sum the 8 token groups of a warp (lanes with equal vc)
#pragma unroll
    for (int h = 0; h < kQH; ++h)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 v = acc_v[h][k];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
                v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
            }
            acc_v[h][k] = v;
        }
    float * obuf = wbuf;   // [WPB][kQH][D]
    if (vgrp == 0) {
#pragma unroll
        for (int h = 0; h < kQH; ++h)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = vblk * 32 + 8 * vc + 2 * k;
                obuf[(vtq * kQH + h) * D + j] = acc_v[h][k].x;
                obuf[(vtq * kQH + h) * D + j + 1] = acc_v[h][k].y;
            }
    }
    __syncthreads();
    float * ws = static_cast<float *>(a.workspace);
    const int S = a.n_splits;
    const int64_t n_part = (int64_t)a.batch * a.n_q_heads * S;
    for (int idx = tid; idx < nh * D; idx += kFastThreads) {
        const int h = idx / D, j = idx % D;
        float v = 0.0f;
#pragma unroll
        for (int q = 0; q < F::WPB; ++q) v += obuf[(q * kQH + h) * D + j];
        const int64_t pidx = ((int64_t)b * a.n_q_heads + h0 + h) * S + split;
        ws[pidx * D + j] = v;
    }
    if (tid < nh) {
        const int64_t pidx = ((int64_t)b * a.n_q_heads + h0 + tid) * S + split;
        float mh = m_run[0], lh = L[0];
#pragma unroll
        for (int h = 1; h < kQH; ++h) if (tid == h) { mh = m_run[h]; lh = L[h]; }
        ws[n_part * D + 2 * pidx] = n_tiles > 0 ? mh : -CUDART_INF_F;
        ws[n_part * D + 2 * pidx + 1] = n_tiles > 0 ? lh : 0.0f;
    }
}

template <int D, int KB, int VB>
int launch_fast_t(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
                  const RotParams & rp, cudaStream_t st) {
    using F = Fast<D, KB, VB>;
    auto k = decode_split_fast_kernel<D, KB, VB>;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
        if (e != cudaSuccess) return (int)e;
        attr_set[dev] = true;
    }
    const int G = a.n_q_heads / a.n_kv_heads;
    const int HG = (G + kQH - 1) / kQH;
    dim3 grid((unsigned)a.n_splits, (unsigned)(a.batch * a.n_kv_heads * HG));
    k<<<grid, kFastThreads, F::SMEM, st>>>(a, kcb, vcb, rp);
    return (int)cudaGetLastError();
}

template <int D, int KB>
int fast_vb(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
            const RotParams & rp, cudaStream_t st) {
    switch (a.v_bits) {
        case 2: return launch_fast_t<D, KB, 2>(a, kcb, vcb, rp, st);
        case 3: return launch_fast_t<D, KB, 3>(a, kcb, vcb, rp, st);
        case 4: return launch_fast_t<D, KB, 4>(a, kcb, vcb, rp, st);
    }
    return (int)cudaErrorInvalidValue;
}

template <int D>
int fast_kb(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
            const RotParams & rp, cudaStream_t st) {
    switch (a.k_bits) {
        case 2: return fast_vb<D, 2>(a, kcb, vcb, rp, st);
        case 3: return fast_vb<D, 3>(a, kcb, vcb, rp, st);
        case 4: return fast_vb<D, 4>(a, kcb, vcb, rp, st);
    }
    return (int)cudaErrorInvalidValue;
}

RotParams rot_params(const tq_rotation * rot) {
    RotParams rp{};
    for (int i = 0; i < 8; ++i) {
        rp.d1_bits[i] = rot->d1_bits[i];
        rp.d2_bits[i] = rot->d2_bits[i];
    }
    return rp;
}

}  // namespace

int launch_logits(const tq_rotation * rot, const CodebookParams & kcb, const AttnArgs & a,
                  void * stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RotParams rp = rot_params(rot);
    dim3 grid((unsigned)((a.ctx + kLogitTokensPerCta - 1) / kLogitTokensPerCta),
              (unsigned)(a.batch * a.n_kv_heads));
    switch (a.k_bits) {
        case 2: logits_simple_kernel<2><<<grid, kThreads, 0, st>>>(a, kcb, rp); break;
        case 3: logits_simple_kernel<3><<<grid, kThreads, 0, st>>>(a, kcb, rp); break;
        case 4: logits_simple_kernel<4><<<grid, kThreads, 0, st>>>(a, kcb, rp); break;
        default: return (int)cudaErrorInvalidValue;
    }
    return (int)cudaGetLastError();
}

template <int KB>
static int launch_split_k(const AttnArgs & a, const CodebookParams & kcb,
                          const CodebookParams & vcb, const RotParams & rp, dim3 grid,
                          cudaStream_t st) {
    switch (a.v_bits) {
        case 2: decode_split_simple_kernel<KB, 2><<<grid, kThreads, 0, st>>>(a, kcb, vcb, rp); break;
        case 3: decode_split_simple_kernel<KB, 3><<<grid, kThreads, 0, st>>>(a, kcb, vcb, rp); break;
        case 4: decode_split_simple_kernel<KB, 4><<<grid, kThreads, 0, st>>>(a, kcb, vcb, rp); break;
        default: return (int)cudaErrorInvalidValue;
    }
    return (int)cudaGetLastError();
}

int launch_decode(const tq_rotation * rot, const CodebookParams & kcb,
                  const CodebookParams & vcb, const AttnArgs & a, void * stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RotParams rp = rot_params(rot);
    if (a.qjl_signs == nullptr) {
        int err;
        switch (a.head_dim) {
            case 64: err = fast_kb<64>(a, kcb, vcb, rp, st); break;
            case 128: err = fast_kb<128>(a, kcb, vcb, rp, st); break;
            case 256: err = fast_kb<256>(a, kcb, vcb, rp, st); break;
            default: return (int)cudaErrorInvalidValue;
        }
        if (err) return err;
        decode_combine_kernel<<<(unsigned)(a.batch * a.n_q_heads), kThreads, 0, st>>>(a, rp);
        return (int)cudaGetLastError();
    }
    dim3 grid((unsigned)a.n_splits, (unsigned)(a.batch * a.n_kv_heads));
    int err;
    switch (a.k_bits) {
        case 2: err = launch_split_k<2>(a, kcb, vcb, rp, grid, st); break;
        case 3: err = launch_split_k<3>(a, kcb, vcb, rp, grid, st); break;
        case 4: err = launch_split_k<4>(a, kcb, vcb, rp, grid, st); break;
        default: return (int)cudaErrorInvalidValue;
    }
    if (err) return err;
    decode_combine_kernel<<<(unsigned)(a.batch * a.n_q_heads), kThreads, 0, st>>>(a, rp);
    return (int)cudaGetLastError();
}

size_t decode_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t n_splits,
                              int32_t head_dim) {
    const size_t parts = (size_t)batch * n_q_heads * n_splits;
    return parts * ((size_t)head_dim + 2) * sizeof(float);
}

size_t qrot_workspace_bytes(int32_t, int32_t, int32_t, int32_t) { return 0; }

}  // namespace tq
