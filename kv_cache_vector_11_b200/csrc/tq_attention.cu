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

#include <algorithm>
#include <type_traits>
#include <utility>

#include <cuda_runtime.h>
#include <math_constants.h>

#include "tq_device.cuh"
#include "tq_tc.cuh"

namespace tq {

namespace {

constexpr int kThreads = 128;
constexpr int kMaxGroup = 8;
constexpr int kMaxDim = 256;
constexpr int kMaxQjl = 256;
constexpr int kLogitTokensPerCta = 2048;
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ __forceinline__ int64_t warp_of_slab(int64_t s, int64_t n_slabs,
                                                         int64_t n_warps) {
    // the warp w whose range [w T / W, (w + 1) T / W) holds slab s
    return ((s + 1) * n_warps - 1) / n_slabs;
}

struct RotParams {
    uint32_t d1_bits[8];
    uint32_t d2_bits[8];
};

// Programmatic dependent launch: let the next kernel of the stream start its
// prologue now / wait here until the previous kernel's results are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
        // q_rot[g][e] = sum_i P[e][i] q_raw[g][i]: warp w takes rows e = w, w +
        // (warps), ...; its lanes read the row coalesced and the G sums meet by
        // shuffles
        const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
        for (int e = wi; e < d; e += nw) {
            float acc[kMaxGroup];
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g) acc[g] = 0.0f;
            for (int i = lane; i < d; i += 32) {
                const float pv = a.rot_f32[(int64_t)e * d + i];
#pragma unroll
                for (int g = 0; g < kMaxGroup; ++g)
                    if (g < G) acc[g] = fmaf(pv, q_raw[g * d + i], acc[g]);
            }
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g) {
                if (g < G) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o);
                    if (lane == 0) q_rot[g * d + e] = acc[g];
                }
            }
        }
        __syncthreads();
    }
}

// w[g][i] = (S q_rot[g])_i for the QJL projection S (m x d, fp32 in global).
// Warp w takes rows i = w, w + (warps), ...; its lanes read the row
// coalesced and the G sums meet by shuffles.
__device__ void project_queries(const AttnArgs & a, int G, const float * q_rot, float * w) {
    const int d = a.head_dim, m = a.qjl_m;
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
    for (int i = wi; i < m; i += nw) {
        float acc[kMaxGroup];
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) acc[g] = 0.0f;
        for (int j = lane; j < d; j += 32) {
            const float sv = a.qjl_f32[(int64_t)i * d + j];
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g)
                if (g < G) acc[g] = fmaf(sv, q_rot[g * d + j], acc[g]);
        }
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g < G) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o);
                if (lane == 0) w[g * m + i] = acc[g];
            }
        }
    }
    __syncthreads();
}

// Stored norm of the 32-coordinate piece k of cache row `row`: norms hold
// head_dim / norm_block values per row, fp16 bits or fp32.
__device__ __forceinline__ float piece_norm(const AttnArgs & a, const uint16_t * norms,
                                            int64_t row, int k) {
    const int nbk = a.head_dim / a.norm_block;
    const int64_t i = row * nbk + (k * 32) / a.norm_block;
    return a.norm_f32 ? reinterpret_cast<const float *>(norms)[i] : half_bits_to_float(norms[i]);
}

// Raw score of token row `row` for the G heads: sum_k gamma_k sum_j q_j c[idx_j]
// (+ QJL term).  Generic in BITS through extract_code; codes have the same
// layout for every norm block size.
template <int BITS>
__device__ __forceinline__ void score_row(const AttnArgs & a, int64_t row, int G,
                                          const float * q_rot, const float * lut,
                                          const float * w_qjl, float * s) {
    const int d = a.head_dim;
    const int nb = d / 32;
    const uint32_t * cw = a.k_codes + row * (int64_t)(nb * BITS);
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
        const float gam = piece_norm(a, a.k_norms, row, k);
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
                // code index of (block blk, coordinate jj) in the row's stream:
                // blocks one after the other, or lane-grouped (4 (nb (jj / 4) +
                // blk) + jj % 4)
                const uint32_t * vr = a.v_codes + row * (int64_t)(nb * VBITS);
                const int ci = a.v_grouped ? 4 * (nb * (jj >> 2) + blk) + (jj & 3) : 32 * blk + jj;
                const float c = vlut[extract_code<VBITS>(vr, ci)];
                const float vg = piece_norm(a, a.v_norms, row, blk) * c;
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

// One CTA per (batch, q head): merge the head's partial slots -- one per warp
// range on the tensor-core path, one per context split on the CUDA-core path
// -- and apply R^T.  The slots are spread over the CTA: thread t owns four
// consecutive dims (4 (t mod d/4) ..) of the slots s = t div (d/4) (mod P,
// P = 4 * 256 / d parts), and loads the first kCombinePre of them (partial
// and (m, l)) before anything else, so that their latency overlaps the
// block-wide maximum; the parts meet in shared memory.  Launched as the
// decode's programmatic dependent: it waits for the decode grid first.
constexpr int kCombineThreads = 256;
constexpr int kCombinePre = 8;

__global__ void __launch_bounds__(kCombineThreads)
decode_combine_kernel(const AttnArgs a, const RotParams rp) {
    __shared__ __align__(16) float o_s[kMaxDim];
    __shared__ float o_raw[kMaxDim];
    __shared__ __align__(16) float part_s[4 * kCombineThreads];
    __shared__ float red[kCombineThreads / 32];
    pdl_wait();
    const int d = a.head_dim;
    const int S = a.n_splits;
    const int64_t bhq = blockIdx.x;  // b * Hq + h
    const float * ws = static_cast<const float *>(a.workspace);
    const int64_t n_part = (int64_t)a.batch * a.n_q_heads * S;
    const float * ml = ws + n_part * d;
    int S_act = S;
    if (a.mma_mode) {
        // slots of this head = the warps whose slab ranges meet its group
        const int G = a.n_q_heads / a.n_kv_heads;
        const int64_t b = bhq / a.n_q_heads;
        const int h = (int)(bhq % a.n_q_heads);
        const int64_t bhg = (b * a.n_kv_heads + h / G) * a.mma_groups + (h % G) / 4;
        S_act = (int)(warp_of_slab((bhg + 1) * a.mma_spb - 1, a.mma_slabs, a.mma_warps) -
                      warp_of_slab(bhg * a.mma_spb, a.mma_slabs, a.mma_warps) + 1);
    }
    const float2 * mls = reinterpret_cast<const float2 *>(ml) + bhq * S;
    const float * wsh = ws + bhq * S * d;
    const int Q = d / 4;                          // threads per slot (4 dims each)
    const int P = kCombineThreads / Q;            // slot parts
    const int j4 = 4 * (threadIdx.x % Q), part = threadIdx.x / Q;
    // early loads: the first kCombinePre slots of this thread's part
    float4 o4[kCombinePre];
    float2 mlv[kCombinePre];
#pragma unroll
    for (int i = 0; i < kCombinePre; ++i) {
        const int s = part + P * i;
        if (s < S_act) {
            o4[i] = *reinterpret_cast<const float4 *>(wsh + (int64_t)s * d + j4);
            mlv[i] = mls[s];
        } else {
            o4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            mlv[i] = make_float2(-CUDART_INF_F, 0.0f);
        }
    }
    // M = max_s m_s and L = sum_s 2^(m_s - M) l_s (a slot that saw no token
    // has m = -inf and weight 0)
    float m = -CUDART_INF_F;
    for (int s = threadIdx.x; s < S_act; s += blockDim.x) m = fmaxf(m, mls[s].x);
    const float M = block_max(m, red);
    float l = 0.0f;
    for (int s = threadIdx.x; s < S_act; s += blockDim.x) {
        const float2 m_l = mls[s];
        if (m_l.x != -CUDART_INF_F) l = fmaf(exp2f(m_l.x - M), m_l.y, l);
    }
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    auto add = [&](const float2 m_l, const float4 o) {
        const float w = m_l.x == -CUDART_INF_F ? 0.0f : exp2f(m_l.x - M);
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
    };
#pragma unroll
    for (int i = 0; i < kCombinePre; ++i) add(mlv[i], o4[i]);
#pragma unroll 4
    for (int s = part + P * kCombinePre; s < S_act; s += P)
        add(mls[s], *reinterpret_cast<const float4 *>(wsh + (int64_t)s * d + j4));
    const float L = block_sum(l, red);
    *reinterpret_cast<float4 *>(part_s + 4 * threadIdx.x) = acc;
    __syncthreads();
    for (int jj = threadIdx.x; jj < d; jj += blockDim.x) {
        float t = 0.0f;
        for (int p = 0; p < P; ++p) t += part_s[4 * (p * Q + jj / 4) + (jj & 3)];
        o_s[jj] = t / L;
    }
    __syncthreads();
    if (a.rot_kind == TQ_ROT_WHT) {
        // R^T = d^-1/2 D2 H D1
        for (int jj = threadIdx.x; jj < d; jj += blockDim.x) o_s[jj] *= sign_of(rp.d1_bits, jj);
        smem_fwht(o_s, d, 1);
        const float sc = rsqrtf((float)d);
        for (int jj = threadIdx.x; jj < d; jj += blockDim.x)
            a.out[bhq * d + jj] = o_s[jj] * sc * sign_of(rp.d2_bits, jj);
    } else {
        for (int jj = threadIdx.x; jj < d; jj += blockDim.x) o_raw[jj] = o_s[jj];
        __syncthreads();
        for (int i = threadIdx.x; i < d; i += blockDim.x) {
            float t = 0.0f;
            for (int e = 0; e < d; ++e) t = fmaf(a.rot_f32[(int64_t)e * d + i], o_raw[e], t);
            a.out[bhq * d + i] = t;
        }
    }
}

// Launch the combine; with `pdl` as the previous kernel's programmatic
// dependent (its CTAs start as soon as that grid lets them and wait inside).
int launch_combine(const AttnArgs & a, const RotParams & rp, cudaStream_t st, bool pdl) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(a.batch * a.n_q_heads));
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_combine_kernel, a, rp);
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
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
    if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), F::SMEM)) return e;
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

// ---------------------------------------------------------------------------
// Warp-streamed decode on tensor cores (keys without the QJL stage).
//
// The tokens of every (batch, kv head, group of four query heads) are cut into
// 16-token slabs; the slabs of all of them, back to back, are cut into one
// contiguous range per warp of a persistent grid (one CTA of up to 16 warps
// per SM), so every warp streams the same number of slabs and no two warps
// ever wait on each other.  A warp stages its slabs with cp.async into a
// private 3-deep ring and keeps its own online softmax (base-2, the scale and
// log2 e folded into the query); where its range enters the next (batch, kv
// head, group) it writes a partial (max, sum, unnormalised rotated output)
// into the slot of that query head and starts over.  The combine launch merges
// the slots and applies R^T.
//
//  * logits: mma.sync m16n8k16, A = 16 tokens x 16 coordinates of fp16
//    centroids (exact: the stored table is fp16), B = the rotated query of the
//    four heads split into fp16 high and low parts, column 2 h + part, so a
//    thread's column pair sums to one head's score.  One accumulator per
//    32-coordinate block, scaled by the block's fp16 norm.  Centroid pairs
//    come from a pair table with one copy per lane: entry e of lane l sits at
//    byte e * 256 + 4 l, so one byte permute turns a byte of 4-bit codes into
//    the address.  K code chunks are XOR-swizzled per token so that the eight
//    tokens of a fragment load hit distinct banks.
//  * softmax: a head's 16 scores sit on the 8 lanes that share its column;
//    the running state is rescaled only when a head's maximum grows.
//  * values: mma.sync, A = 16 coordinates x 16 tokens of fp16 centroids (a
//    lane owns four consecutive coordinates of a block: a funnel shift, two
//    pair lookups per token, one byte permute per two tokens), B = p * ||v||
//    of the block in fp16 for the four heads, moved out of the logit layout
//    with two shuffles.
// ---------------------------------------------------------------------------
constexpr int kSlab = 16;
constexpr int kStages = 3;
constexpr int kLutBytes = 65536;
constexpr int kMmaMaxM = 128;       // QJL projection rows on the tensor-core decode

template <int D, bool QJL>
struct MmaCfg {
    // warps per CTA (register budget: 16 x 128 registers, or 12 x 168 with
    // the QJL fragments)
    static constexpr int WPC = QJL ? 12 : (D <= 128 ? 16 : 8);
};

template <int D, int KB, int VB, bool QJL>
struct SlabCfg {
    static constexpr int NB = D / 32;
    static constexpr int KW = NB * KB;                 // K code words per token
    static constexpr int VW = NB * VB;
    static constexpr int SZ_KC = kSlab * KW * 4;
    static constexpr int SZ_KN = kSlab * NB * 2;
    static constexpr int SZ_VC = kSlab * VW * 4;
    static constexpr int SZ_VN = kSlab * NB * 2;
    static constexpr int SZ_SG = QJL ? kSlab * (kMmaMaxM / 32) * 4 : 0;   // sign words
    static constexpr int SZ_RN = QJL ? kSlab * 2 : 0;                     // residual norms
    static constexpr int OFF_KN = SZ_KC;
    static constexpr int OFF_VC = OFF_KN + SZ_KN;
    static constexpr int OFF_VN = OFF_VC + SZ_VC;
    static constexpr int OFF_SG = OFF_VN + SZ_VN;
    static constexpr int OFF_RN = OFF_SG + SZ_SG;
    static constexpr int BYTES = OFF_RN + SZ_RN;
    static constexpr int RING = kStages * BYTES;
    static_assert(SZ_KC % 16 == 0 && SZ_KN % 16 == 0 && SZ_VC % 16 == 0 && SZ_VN % 16 == 0 &&
                      SZ_SG % 16 == 0 && SZ_RN % 16 == 0,
                  "slab sections must be whole 16-byte chunks");
};


// 2^x with the hardware approximation (relative error below 2^-22; -inf -> 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t h2_bits(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a),
                              *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}

__device__ __forceinline__ void mma16816(float * d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Pair-table byte offset of code pair p (codes 2p, 2p+1 of the 8 codes in
// `w`) for a lane whose copy starts at `lane_off` (< 256, bits 8..15 zero).
template <int B>
__device__ __forceinline__ uint32_t pair_offset(uint32_t w, int p, uint32_t lane_off) {
    if constexpr (B == 4) {
        return __byte_perm(w, lane_off, 0x7604u | ((uint32_t)p << 4));
    } else {
        constexpr uint32_t PM = ((1u << (2 * B)) - 1u) << 8;
        const int sh = 2 * B * p - 8;     // move the field to bit 8
        const uint32_t x = sh >= 0 ? (w >> sh) : (w << (-sh));
        return (x & PM) | lane_off;
    }
}

// +-1 fp16 pairs from two sign bits: bit set -> +1, clear -> -1.  One multiply
// sends bit 0 to bits 15 and 30 and bit 1 to bits 16 and 31 (bits 8, 9 alike
// with the shifted constant); the mask keeps 15 and 31, the XOR turns them
// into fp16 +1 / -1.
__device__ __forceinline__ uint32_t signs_lo_pair(uint32_t x) {
    return (((x & 3u) * 0x40008000u) & 0x80008000u) ^ 0xBC00BC00u;
}
__device__ __forceinline__ uint32_t signs_hi_pair(uint32_t x) {
    return (((x & 0x300u) * 0x00400080u) & 0x80008000u) ^ 0xBC00BC00u;
}


// Quantize one new cache row exactly as tq_quantize_kv defines it -- y = R x,
// per-32-block norm ||y_blk|| (fp32, stored fp16 round-to-nearest, saturating
// at 65504), code = #{i : u >= t_i} with u = y_blk / ||y_blk|| (a zero block
// stores 2^(b-1)), b-bit little-endian packing -- and store it at cache row
// `row`.  Run by all threads of the CTA; y and xr are D floats of shared memory.
template <int D>
__device__ void append_row(const void * src, bool bf16, int64_t off, int bits, const float * bound,
                           const AttnArgs & a, const RotParams & rp, float * y, float * xr,
                           uint32_t * codes, uint16_t * norms, int64_t row, uint32_t & status) {
    constexpr int NB = D / 32;
    const bool wht = a.rot_kind == TQ_ROT_WHT;
    __syncthreads();
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        float v = bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(src)[off + i])
                       : static_cast<const float *>(src)[off + i];
        if (wht) v *= sign_of(rp.d2_bits, i);
        (wht ? y : xr)[i] = v;
    }
    if (wht) {
        smem_fwht(y, D, 1);
        const float sc = rsqrtf((float)D);
        for (int i = threadIdx.x; i < D; i += blockDim.x) y[i] *= sc * sign_of(rp.d1_bits, i);
    } else {
        __syncthreads();
        for (int e = threadIdx.x; e < D; e += blockDim.x) {
            const float * pr = a.rot_f32 + (int64_t)e * D;
            float acc = 0.0f;
            for (int i = 0; i < D; ++i) acc = fmaf(pr[i], xr[i], acc);
            y[e] = acc;
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int levels = (1 << bits) - 1;
    for (int blk = w; blk < NB; blk += nw) {
        const float v = y[32 * blk + lane];
        float ss = v * v;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float gam = sqrtf(ss);
        uint32_t code = 1u << (bits - 1);
        if (gam > 0.0f) {
            const float u = v / gam;
            code = 0u;
            for (int i = 0; i < levels; ++i) code += u >= bound[i] ? 1u : 0u;
        }
        const int p = lane * bits;
        for (int k = 0; k < bits; ++k) {
            const int lo = p - 32 * k;
            uint32_t part = 0u;
            if (lo >= 0 && lo < 32) part = code << lo;
            else if (lo < 0 && lo + bits > 0) part = code >> (-lo);
            const uint32_t word = __reduce_or_sync(0xffffffffu, part);
            if (lane == k) codes[row * (NB * bits) + blk * bits + k] = word;
        }
        if (lane == 0) {
            if (!isfinite(ss)) status |= TQ_STATUS_NONFINITE;
            bool sat;
            norms[row * NB + blk] = norm_to_half_bits(gam, &sat);
            if (sat) status |= TQ_STATUS_NORM_SATURATED;
        }
    }
}

// Rotated, scaled query fragments of one (batch, kv head, group): for lane l
// (B column n = l / 4: head n / 2, fp16 high part if n is even, low part if
// odd; t = l % 4), block b and k step s, the words (b * 2 + s) * 2 + {0, 1}
// hold dims 32 b + 8 t + 4 s + {0, 1} and {2, 3}.  With QJL keys, words
// NB * 4 + 2 c + {0, 1} hold the B fragment of projection rows 16 c + 2 t +
// {0, 1} and 16 c + 2 t + 8 + {0, 1} of sqrt(pi/2) / m * (S q~).  Every value
// carries the softmax scale times log2 e.
// (256 threads: one CTA per group has little work but a long chain of
// dependent steps; more warps shorten the QJL projection's share)
constexpr int kPrepThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPrepThreads)
decode_mma_prep_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ RotParams rp,
                       const __grid_constant__ AppendParams ap) {
    constexpr int NB = D / 32;
    __shared__ float q_rot[kQH * D];
    __shared__ float w_s[kQH * kMmaMaxM];
    __shared__ float y_s[D], x_s[D];
    pdl_launch_dependents();
    const int64_t bhg = blockIdx.x;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int hg = (int)(bhg % a.mma_groups);
    const int64_t bh = bhg / a.mma_groups;
    const int b = (int)(bh / a.n_kv_heads), hk = (int)(bh % a.n_kv_heads);
    const int h0 = hk * G + hg * kQH;
    const int nh = min(kQH, G - hg * kQH);
    const bool qjl = a.qjl_signs != nullptr;
    const int m = qjl ? a.qjl_m : 0;
    for (int i = threadIdx.x; i < kQH * D; i += blockDim.x) q_rot[i] = 0.0f;
    for (int i = threadIdx.x; i < kQH * kMmaMaxM; i += blockDim.x) w_s[i] = 0.0f;
    __syncthreads();
    rotate_queries(a, rp, b, h0, nh, q_rot);
    if (ap.enabled && hg == 0) {
        // decode-time append: the new token of (b, hk) goes to position ctx - 1
        const int64_t t = a.ctx - 1;
        int64_t row = bh * a.ctx + t;
        if (a.page_size != 0) {
            const int64_t page = min(max(a.block_table[(int64_t)b * a.max_pages + (t >> a.page_shift)], 0),
                                     a.n_pages - 1);
            row = ((page * a.n_kv_heads + hk) << a.page_shift) + (t & (a.page_size - 1));
        }
        uint32_t status = 0u;
        const int64_t off = bh * D;
        append_row<D>(ap.k_new, ap.kv_bf16 != 0, off, a.k_bits, ap.k_bound, a, rp, y_s, x_s,
                      ap.k_codes, ap.k_norms, row, status);
        append_row<D>(ap.v_new, ap.kv_bf16 != 0, off, a.v_bits, ap.v_bound, a, rp, y_s, x_s,
                      ap.v_codes, ap.v_norms, row, status);
        if (status != 0u && ap.status != nullptr) atomicOr(ap.status, status);
    }
    if (qjl) {
        // w_s[h][i] = (S q~_h)_i: warp w takes rows w, w + (warps), ..., its lanes
        // read a row coalesced (eight rows' loads in flight) and the partial
        // sums of the group's heads meet by shuffles
        const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
        constexpr int JW = D / 32;
#pragma unroll 8
        for (int r = wi; r < m; r += nw) {
            float sv[JW];
#pragma unroll
            for (int jj = 0; jj < JW; ++jj) sv[jj] = a.qjl_f32[(int64_t)r * D + lane + 32 * jj];
            float acc[kQH];
#pragma unroll
            for (int h = 0; h < kQH; ++h) acc[h] = 0.0f;
#pragma unroll
            for (int jj = 0; jj < JW; ++jj)
#pragma unroll
                for (int h = 0; h < kQH; ++h) acc[h] = fmaf(sv[jj], q_rot[h * D + lane + 32 * jj], acc[h]);
#pragma unroll
            for (int h = 0; h < kQH; ++h) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
            }
            if (lane == 0)
                for (int h = 0; h < nh; ++h) w_s[h * kMmaMaxM + r] = acc[h];
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x, n = lane >> 2, t = lane & 3;
        const int head = n >> 1;
        const bool lo_part = (n & 1) != 0;
        const float sl2 = a.scale * kLog2e;
        auto frag = [&](float x0, float x1) {
            const __half2 hi = __floats2half2_rn(x0, x1);
            const uint32_t v = *reinterpret_cast<const uint32_t *>(&hi);
            return lo_part ? h2_bits(x0 - __low2float(hi), x1 - __high2float(hi)) : v;
        };
        uint32_t * dst = a.mma_qfrag + (bhg * 32 + lane) * a.mma_qwords;
        for (int blk = 0; blk < NB; ++blk)
            for (int s = 0; s < 2; ++s)
                for (int r = 0; r < 2; ++r) {
                    const int dim = 32 * blk + 8 * t + 4 * s + 2 * r;
                    const float x0 = head < nh ? q_rot[head * D + dim] * sl2 : 0.0f;
                    const float x1 = head < nh ? q_rot[head * D + dim + 1] * sl2 : 0.0f;
                    dst[(blk * 2 + s) * 2 + r] = frag(x0, x1);
                }
        if (qjl) {
            const float coef = 1.2533141373155003f / (float)m * sl2;   // sqrt(pi/2) / m
            for (int c = 0; c < kMmaMaxM / 16; ++c)
                for (int r = 0; r < 2; ++r) {
                    const int i0 = 16 * c + 2 * t + 8 * r;
                    const bool live = head < nh && i0 < m;
                    const float x0 = live ? coef * w_s[head * kMmaMaxM + i0] : 0.0f;
                    const float x1 = live ? coef * w_s[head * kMmaMaxM + i0 + 1] : 0.0f;
                    dst[NB * 4 + 2 * c + r] = frag(x0, x1);
                }
        }
    }
}

// f(integral_constant<int, 0>) ... f(integral_constant<int, N - 1>): an
// unrolled loop whose index can be a template argument (load offsets).
template <typename F, int... I>
__device__ __forceinline__ void static_for_seq(F & f, std::integer_sequence<int, I...>) {
    (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F && f) {
    static_for_seq(f, std::make_integer_sequence<int, N>{});
}

// Shared-memory loads by 32-bit window address (the offset is an immediate).
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(addr), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ void cp_async16_s(uint32_t dst, const void * src) {
    asm volatile("cp.async.cg.shared.global [%0+%2], [%1], 16;" ::"r"(dst), "l"(src), "n"(OFF) : "memory");
}
template <int OFF = 0>
__device__ __forceinline__ void cp_async16_zfill_s(uint32_t dst, const void * src, int n) {
    const int sz = n <= 0 ? 0 : (n >= 16 ? 16 : n);
    asm volatile("cp.async.cg.shared.global [%0+%3], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz), "n"(OFF)
                 : "memory");
}

template <int D, int KB, int VB, bool QJL, bool PAGED, bool VG = false>
__global__ void __launch_bounds__(32 * MmaCfg<D, QJL>::WPC, 1)
decode_mma_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CodebookParams kcb,
                  const __grid_constant__ CodebookParams vcb) {
    using S = SlabCfg<D, KB, VB, QJL>;
    constexpr int NB = S::NB;
    constexpr int NK = 1 << (2 * KB), NV = 1 << (2 * VB);
    extern __shared__ __align__(16) unsigned char smem[];
    // the combine grid may be launched now; it waits for this grid's results
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    // The pair tables sit at a window address with zero low 16 bits, so that
    // (entry << 8) | (lane offset) -- one byte permute or multiply-add -- is
    // the full load address.
    const uint32_t lut_w = (uint32_t)__cvta_generic_to_shared(smem) + (uint32_t)a.mma_lut_off;
    const bool lut_ok = (lut_w & 0xFFFFu) == 0u;

    if (lut_ok) {
        uint32_t * lw = reinterpret_cast<uint32_t *>(smem + a.mma_lut_off);
        for (int i = threadIdx.x; i < (NK + NV) * 32; i += blockDim.x) {
            const int e = i >> 5, l = i & 31;
            if (e < NK) {
                lw[e * 64 + l] = h2_bits(kcb.centroid[e & ((1 << KB) - 1)], kcb.centroid[e >> KB]);
            } else {
                const int ev = e - NK;
                lw[ev * 64 + 32 + l] = h2_bits(vcb.centroid[ev & ((1 << VB) - 1)], vcb.centroid[ev >> VB]);
            }
        }
    }
    __syncthreads();

    const int64_t T = a.mma_slabs, W = a.mma_warps, spb = a.mma_spb;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + wi;
    if (gw >= W) return;                      // W <= T: every live warp owns >= 1 slab
    const int64_t s_begin = gw * T / W, s_end = (gw + 1) * T / W;
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(smem) +
                          (uint32_t)(wi < a.mma_ring_a ? wi * S::RING
                                                       : a.mma_lut_off + kLutBytes + (wi - a.mma_ring_a) * S::RING);
    const int G = a.n_q_heads / a.n_kv_heads;
    const int m = QJL ? a.qjl_m : 0;

    // slab cursor: (batch, kv head, group) index, first token, first cache row
    // of the (batch, kv head); advanced without divisions
    // (all in 32 bits: the plan keeps rows and groups below 2^31)
    struct Cursor {
        int32_t bhg, ts, hg, row0, rowbase;   // group, first token, head group, first row, bh row
        int32_t b, hk;                        // sequence and kv head (paged cache)
    };
    auto cursor_at = [&](int64_t s) {
        Cursor c;
        const int64_t bhg = s / spb;
        c.bhg = (int32_t)bhg;
        c.ts = (int32_t)((s - bhg * spb) * kSlab);
        c.hg = (int32_t)(bhg % a.mma_groups);
        const int64_t bh = bhg / a.mma_groups;
        c.rowbase = (int32_t)(bh * a.ctx);
        c.row0 = c.rowbase + c.ts;
        c.b = (int32_t)(bh / a.n_kv_heads);
        c.hk = (int32_t)(bh % a.n_kv_heads);
        return c;
    };
    const int32_t ctx32 = (int32_t)a.ctx;
    auto advance = [&](Cursor & c) {
        c.ts += kSlab;
        c.row0 += kSlab;
        if (c.ts >= ctx32) {
            c.ts = 0;
            ++c.bhg;
            if (++c.hg == a.mma_groups) {
                c.hg = 0;
                c.rowbase += ctx32;
                if (++c.hk == a.n_kv_heads) {
                    c.hk = 0;
                    ++c.b;
                }
            }
            c.row0 = c.rowbase;
        }
    };
    // first row of a slab: [b][hk][ctx] rows, or through the block table of a
    // paged cache (pages of 2^page_shift tokens, [page][kv head][token] rows;
    // a slab never straddles two pages)
    auto slab_row = [&](const Cursor & c) -> uint32_t {
        if constexpr (!PAGED) return (uint32_t)c.row0;
        // (an entry outside [0, n_pages) reads the nearest valid page instead
        // of memory beyond the page storage)
        const int32_t page = min(max(__ldg(a.block_table + (int64_t)c.b * a.max_pages + (c.ts >> a.page_shift)), 0),
                                 a.n_pages - 1);
        return (uint32_t)((page * a.n_kv_heads + c.hk) << a.page_shift) +
               (uint32_t)(c.ts & (a.page_size - 1));
    };

    // per-lane destination offsets of the 16-byte chunks this lane copies
    constexpr int NKC = S::SZ_KC / 16, NVC = S::SZ_VC / 16, NKN = S::SZ_KN / 16;
    constexpr int KCL = (NKC + 31) / 32, VCL = (NVC + 31) / 32;
    uint32_t kdst[KCL];
#pragma unroll
    for (int j = 0; j < KCL; ++j) {
        const int c = lane + 32 * j;
        int off = 16 * c;
        if constexpr (KB == 4) {
            const int r = c / NB, cc = c % NB;
            off = r * NB * 16 + 16 * (cc ^ kswz<NB>(r));
        }
        kdst[j] = (uint32_t)off;
    }
    // the small sections (K norms, V norms and, with QJL keys, sign words and
    // residual norms): chunk list [K norms | V norms | signs | rnorms], chunk
    // lane + 32 j for this lane
    constexpr int NMISC_MAX = 2 * NKN + (QJL ? (kSlab * kMmaMaxM / 8) / 16 + 2 : 0);
    constexpr int MCL = (NMISC_MAX + 31) / 32;
    const int nsg = QJL ? m / 8 : 0;                 // sign chunks per slab: 16 tokens x m/8 bytes
    const int nmisc = 2 * NKN + (QJL ? nsg + 2 : 0);
    const unsigned char * msrc[MCL];
    uint32_t mdst[MCL];
    int mrow[MCL], mchunk[MCL];
#pragma unroll
    for (int j = 0; j < MCL; ++j) {
        const int c = lane + 32 * j;
        int sec = 0, ci = c;
        if (ci >= NKN) { ci -= NKN; sec = 1; }
        if (sec == 1 && ci >= NKN) { ci -= NKN; sec = 2; }
        if (sec == 2 && ci >= nsg) { ci -= nsg; sec = 3; }
        const unsigned char * base =
            sec == 0 ? reinterpret_cast<const unsigned char *>(a.k_norms)
          : sec == 1 ? reinterpret_cast<const unsigned char *>(a.v_norms)
          : sec == 2 ? reinterpret_cast<const unsigned char *>(a.qjl_signs)
                     : reinterpret_cast<const unsigned char *>(a.qjl_rnorm);
        mrow[j] = (!QJL || sec <= 1) ? NB * 2 : sec == 2 ? m / 8 : 2;
        mchunk[j] = c < nmisc ? ci : -1;
        msrc[j] = base + 16 * ci;
        mdst[j] = (uint32_t)((sec == 0 ? S::OFF_KN : sec == 1 ? S::OFF_VN : sec == 2 ? S::OFF_SG : S::OFF_RN) +
                             16 * ci);
    }

    // per-lane source bases: a lane always copies the same chunks of a slab
    constexpr int KROW = S::KW * 4, VROW = S::VW * 4;
    const unsigned char * kc_l = reinterpret_cast<const unsigned char *>(a.k_codes) + 16 * lane;
    const unsigned char * vc_l = reinterpret_cast<const unsigned char *>(a.v_codes) + 16 * lane;
    // destinations as window addresses in stage 0 of this warp's ring (the
    // stage offset is an immediate of each copy)
#pragma unroll
    for (int j = 0; j < KCL; ++j) kdst[j] += ring;
    const uint32_t vdst = ring + (uint32_t)(S::OFF_VC + 16 * lane);
#pragma unroll
    for (int j = 0; j < MCL; ++j) mdst[j] += ring;

    // copies of one slab into the stage at byte offset FB of the ring
    auto stage = [&](const Cursor & cu, auto FBC) {
        constexpr int FB = decltype(FBC)::value;
        const uint32_t r0 = slab_row(cu);
        if (cu.ts + kSlab <= ctx32) {
            const unsigned char * ks = kc_l + (size_t)r0 * KROW;
            const unsigned char * vs = vc_l + (size_t)r0 * VROW;
#pragma unroll
            for (int j = 0; j < KCL; ++j)
                if (NKC % 32 == 0 || lane + 32 * j < NKC) cp_async16_s<FB>(kdst[j], ks + 512 * j);
            static_for<VCL>([&](auto J) {
                constexpr int j = decltype(J)::value;
                if (NVC % 32 == 0 || lane + 32 * j < NVC) cp_async16_s<FB + 512 * j>(vdst, vs + 512 * j);
            });
#pragma unroll
            for (int j = 0; j < MCL; ++j)
                if (mchunk[j] >= 0)
                    cp_async16_s<FB>(mdst[j], msrc[j] + (size_t)r0 * (QJL ? mrow[j] : NB * 2));
        } else {
            // ragged last slab: copy the valid bytes, zero the rest
            const int nvalid = ctx32 - cu.ts;
            const unsigned char * kc = reinterpret_cast<const unsigned char *>(a.k_codes) + (size_t)r0 * KROW;
            const unsigned char * vc = reinterpret_cast<const unsigned char *>(a.v_codes) + (size_t)r0 * VROW;
#pragma unroll
            for (int j = 0; j < KCL; ++j) {
                const int c = lane + 32 * j;
                if (NKC % 32 == 0 || c < NKC) {
                    const int n = nvalid * KROW - 16 * c;
                    cp_async16_zfill_s<FB>(kdst[j], n > 0 ? kc + 16 * c : kc, n);
                }
            }
            static_for<VCL>([&](auto J) {
                constexpr int j = decltype(J)::value;
                const int c = lane + 32 * j;
                if (NVC % 32 == 0 || c < NVC) {
                    const int n = nvalid * VROW - 16 * c;
                    cp_async16_zfill_s<FB + 512 * j>(vdst, n > 0 ? vc + 16 * c : vc, n);
                }
            });
#pragma unroll
            for (int j = 0; j < MCL; ++j)
                if (mchunk[j] >= 0) {
                    const unsigned char * sec0 = msrc[j] - 16 * mchunk[j] + (size_t)r0 * mrow[j];
                    const int n = nvalid * mrow[j] - 16 * mchunk[j];
                    cp_async16_zfill_s<FB>(mdst[j], n > 0 ? sec0 + 16 * mchunk[j] : sec0, n);
                }
        }
    };

    // per-lane constants
    const uint32_t klane = lut_w + 4u * (uint32_t)lane;          // byte 1 clear: entry goes there
    const uint32_t vlane = lut_w + 128u + 4u * (uint32_t)lane;
    constexpr int QBITS = 4 * VB;                                  // a lane's 4 value codes
    // the lane's field of a block starts at bit QBITS * g of the block's
    // words; the 64-bit window read for it starts at word vq_w (one word
    // early for g = 0) so that the field sits 8 bits above the shift
    const int vq_w = ((QBITS * g + 24) >> 5) - 1;
    const int vq_sh = QBITS * g - 8 - 32 * vq_w;
    // K words of rows g and g + 8 (same swizzle: kswz depends on row / (8 / NB) mod NB)
    // (window addresses in stage 0 of the ring; the stage offset is an
    // immediate of each load)
    uint32_t kb_r[NB];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
        if constexpr (KB == 4) kb_r[blk] = ring + (uint32_t)(g * S::KW * 4 + 16 * (blk ^ kswz<NB>(g)) + 4 * t4);
        else kb_r[blk] = ring + (uint32_t)(g * S::KW * 4 + 4 * (KB * blk + ((8 * KB * t4) >> 5)));
    }
    const int ksh = (8 * KB * t4) & 31;
    const uint32_t va_r = ring + (uint32_t)(S::OFF_VC + 4 * (t4 * S::VW + vq_w));   // OFF_VC > 0
    // lane-grouped value rows (d = 128): the lane's codes of all four blocks
    // of a token are one field of 16 VB bits at bit 16 VB g of the row -- word
    // g (2-bit), words 2 g .. 2 g + 1 (4-bit), or for 3-bit codes 48 bits from
    // word 3 (g / 2) + g % 2, bit 16 (g % 2).  Block b's 4 VB bits are moved to
    // bit 8 by one funnel shift or rotation with a per-lane amount.
    static_assert(!VG || NB == 4, "lane-grouped value rows: d = 128");
    const uint32_t vg_r = ring + (uint32_t)(S::OFF_VC + 4 * (t4 * S::VW +
                                 (VB == 3 ? 3 * (g >> 1) + (g & 1) : (VB == 4 ? 2 * g : g))));
    const bool godd = (g & 1) != 0;
    const uint32_t gs0 = godd ? 8u : 24u, gs1 = godd ? 20u : 4u, gs2 = godd ? 32u : 16u,
                   gs3 = godd ? 12u : 28u;
    const uint32_t kn_r = ring + (uint32_t)(S::OFF_KN + g * NB * 2);
    const uint32_t vn_r = ring + (uint32_t)(S::OFF_VN + t4 * NB * 2);
    const int mw = m / 32;                                       // sign words per token
    const uint32_t sg_r = ring + (uint32_t)(S::OFF_SG + g * mw * 4);
    const uint32_t rn_r = ring + (uint32_t)(S::OFF_RN + 4 * (g >> 1));
    const int mchunks = m / 16;

    float m_run = -CUDART_INF_F, l_run = 0.0f;
    float accv[NB][2][4];
    uint32_t qb[NB][2][2];
    uint32_t wq[QJL ? kMmaMaxM / 16 : 1][2];
    int64_t cur = -1;

    auto reset = [&]() {
        m_run = -CUDART_INF_F;
        l_run = 0.0f;
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int k = 0; k < 4; ++k) accv[b][h][k] = 0.0f;
    };
    auto load_q = [&](int64_t bhg) {
        const uint4 * src = reinterpret_cast<const uint4 *>(a.mma_qfrag + (bhg * 32 + lane) * a.mma_qwords);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const uint4 v = src[b];
            qb[b][0][0] = v.x; qb[b][0][1] = v.y; qb[b][1][0] = v.z; qb[b][1][1] = v.w;
        }
        if constexpr (QJL) {
#pragma unroll
            for (int c = 0; c < kMmaMaxM / 32; ++c) {
                const uint4 v = src[NB + c];
                wq[2 * c][0] = v.x; wq[2 * c][1] = v.y; wq[2 * c + 1][0] = v.z; wq[2 * c + 1][1] = v.w;
            }
        }
    };
    // write this warp's partial of group bhg into its slot
    auto flush = [&](int64_t bhg) {
        float L = l_run;
        L += __shfl_xor_sync(0xffffffffu, L, 4);
        L += __shfl_xor_sync(0xffffffffu, L, 8);
        L += __shfl_xor_sync(0xffffffffu, L, 16);
        const int hg = (int)(bhg % a.mma_groups);
        const int64_t bh = bhg / a.mma_groups;
        const int b = (int)(bh / a.n_kv_heads), hk = (int)(bh % a.n_kv_heads);
        const int h0 = hk * G + hg * kQH;
        const int nh = min(kQH, G - hg * kQH);
        const int64_t first = warp_of_slab(bhg * spb, T, W);
        const int64_t slot = gw - first;
        const int Sm = a.n_splits;
        float * ws = static_cast<float *>(a.workspace);
        const int64_t n_part = (int64_t)a.batch * a.n_q_heads * Sm;
        const float bad = lut_ok ? 0.0f : CUDART_NAN_F;    // unusable layout: poison the output
        if (g == 0 && t4 < nh) {
            const int64_t pidx = ((int64_t)b * a.n_q_heads + h0 + t4) * Sm + slot;
            ws[n_part * D + 2 * pidx] = lut_ok ? m_run : 0.0f;
            ws[n_part * D + 2 * pidx + 1] = lut_ok ? L : 1.0f;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int head = 2 * t4 + hh;
            if (t4 < 2 && head < nh) {
                const int64_t pidx = ((int64_t)b * a.n_q_heads + h0 + head) * Sm + slot;
                float * o = ws + pidx * D;
#pragma unroll
                for (int blk = 0; blk < NB; ++blk)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = 32 * blk + 4 * g + 2 * h;
                        *reinterpret_cast<float2 *>(o + c) =
                            make_float2(accv[blk][h][hh] + bad, accv[blk][h][2 + hh] + bad);
                    }
            }
        }
    };

    Cursor fc = cursor_at(s_begin);
    Cursor uc = fc;
    int32_t n_left = lut_ok ? (int32_t)(s_end - s_begin) : 0;
    int32_t n_fetch = n_left;
    // the first kStages - 1 slabs go to stages 0 .. kStages - 2
    static_for<kStages - 1>([&](auto I) {
        constexpr int i = decltype(I)::value;
        if (n_fetch > 0) {
            // the prep kernel appends the new token when asked to: a slab
            // that holds token ctx - 1 is copied only after it is written
            if (PAGED && a.mma_wait_first && fc.ts + kSlab >= ctx32) pdl_wait();
            stage(fc, std::integral_constant<int, i * S::BYTES>{});
            advance(fc);
        }
        cp_async_commit();
        --n_fetch;
    });
    // the query fragments and the partial slots belong to the prep kernel's
    // grid (launched as this grid's programmatic predecessor): wait for it
    // before touching them
    pdl_wait();
    reset();
    // one slab: consume stage ST, refill stage ST - 1 (mod kStages); the loop
    // below unrolls kStages of these so that every stage offset is an
    // immediate of the loads and copies
    auto step = [&](auto STC) {
        constexpr int ST = decltype(STC)::value;
        constexpr int SB = ST * S::BYTES;
        constexpr int FB = ((ST + kStages - 1) % kStages) * S::BYTES;
        if (n_fetch > 0) {
            stage(fc, std::integral_constant<int, FB>{});
            advance(fc);
        }
        cp_async_commit();
        --n_fetch;
        cp_async_wait<kStages - 1>();
        __syncwarp();

        const int64_t bhg = uc.bhg;
        if (bhg != cur) {
            if (cur >= 0) {
                flush(cur);
                reset();
            }
            load_q(bhg);
            cur = bhg;
        }
        const int nvalid = min(kSlab, ctx32 - uc.ts);
        advance(uc);

        // ---- logits ----
        float tot[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        {
            uint32_t kn0[(NB + 1) / 2], kn1[(NB + 1) / 2];
            {
                if constexpr (NB == 2) {
                    kn0[0] = lds32<SB>(kn_r);
                    kn1[0] = lds32<SB + 8 * NB * 2>(kn_r);
                } else {
                    static_for<NB / 4>([&](auto K2) {
                        constexpr int k = 2 * decltype(K2)::value;
                        const uint2 x0 = lds64<SB + 4 * k>(kn_r);
                        const uint2 x1 = lds64<SB + 8 * NB * 2 + 4 * k>(kn_r);
                        kn0[k] = x0.x; kn0[k + 1] = x0.y;
                        kn1[k] = x1.x; kn1[k + 1] = x1.y;
                    });
                }
            }
#pragma unroll
            for (int blk = 0; blk < NB; ++blk) {
                const uint32_t ka = kb_r[blk];
                uint32_t w0, w1;
                if constexpr (KB == 4) {
                    w0 = lds32<SB>(ka);
                    w1 = lds32<SB + 8 * S::KW * 4>(ka);
                } else {
                    w0 = __funnelshift_r(lds32<SB>(ka), lds32<SB + 4>(ka), ksh);
                    w1 = __funnelshift_r(lds32<SB + 8 * S::KW * 4>(ka), lds32<SB + 8 * S::KW * 4 + 4>(ka), ksh);
                }
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const uint32_t a0 = lds32(pair_offset<KB>(w0, 2 * s2, klane));
                    const uint32_t a1 = lds32(pair_offset<KB>(w1, 2 * s2, klane));
                    const uint32_t a2 = lds32(pair_offset<KB>(w0, 2 * s2 + 1, klane));
                    const uint32_t a3 = lds32(pair_offset<KB>(w1, 2 * s2 + 1, klane));
                    mma16816(acc, a0, a1, a2, a3, qb[blk][s2][0], qb[blk][s2][1]);
                }
                const float g0 = __half2float(__ushort_as_half(
                    (unsigned short)(kn0[blk >> 1] >> (16 * (blk & 1)))));
                const float g1 = __half2float(__ushort_as_half(
                    (unsigned short)(kn1[blk >> 1] >> (16 * (blk & 1)))));
                tot[0] = fmaf(g0, acc[0], tot[0]);
                tot[1] = fmaf(g0, acc[1], tot[1]);
                tot[2] = fmaf(g1, acc[2], tot[2]);
                tot[3] = fmaf(g1, acc[3], tot[3]);
            }
        }
        float s0 = tot[0] + tot[1], s1 = tot[2] + tot[3];
        if constexpr (QJL) {
            // QJL term: A = 16 tokens x 16 projection rows of +-1 from the sign
            // bits, B = the scaled projected query (hi/lo); times the token's
            // fp16 residual norm
            float qa[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            uint32_t sw0[kMmaMaxM / 32], sw1[kMmaMaxM / 32];
            if (mw == 4) {
                const uint4 v0 = lds128<SB>(sg_r), v1 = lds128<SB + 8 * 16>(sg_r);
                sw0[0] = v0.x; sw0[1] = v0.y; sw0[2] = v0.z; sw0[3] = v0.w;
                sw1[0] = v1.x; sw1[1] = v1.y; sw1[2] = v1.z; sw1[3] = v1.w;
            } else {
                static_for<kMmaMaxM / 32>([&](auto K) {
                    constexpr int k = decltype(K)::value;
                    sw0[k] = k < mw ? lds32<SB + 4 * k>(sg_r) : 0u;
                    sw1[k] = k < mw ? lds32<SB + 4 * k>(sg_r + 8 * mw * 4) : 0u;
                });
            }
#pragma unroll
            for (int c = 0; c < kMmaMaxM / 16; ++c) {
                if (c < mchunks) {
                    const int sh = 16 * (c & 1) + 2 * t4;
                    const uint32_t x0 = sw0[c >> 1] >> sh;      // token g
                    const uint32_t x1 = sw1[c >> 1] >> sh;      // token g + 8
                    mma16816(qa, signs_lo_pair(x0), signs_lo_pair(x1), signs_hi_pair(x0),
                             signs_hi_pair(x1), wq[c][0], wq[c][1]);
                }
            }
            const uint32_t rr = lds32<SB>(rn_r);
            const uint32_t rr8 = lds32<SB + 16>(rn_r);
            const float rho0 = __half2float(__ushort_as_half((unsigned short)(rr >> (16 * (g & 1)))));
            const float rho1 = __half2float(__ushort_as_half((unsigned short)(rr8 >> (16 * (g & 1)))));
            s0 = fmaf(rho0, qa[0] + qa[1], s0);
            s1 = fmaf(rho1, qa[2] + qa[3], s1);
        }
        s0 = g < nvalid ? s0 : -CUDART_INF_F;
        s1 = g + 8 < nvalid ? s1 : -CUDART_INF_F;

        // ---- softmax (head t4) ----
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run, mx);
        if (__any_sync(0xffffffffu, m_new > m_run)) {
            const float alpha = ex2_approx(m_run - m_new);
            l_run *= alpha;
            const float a_lo = __shfl_sync(0xffffffffu, alpha, (lane & ~3) | ((2 * t4) & 3));
            const float a_hi = __shfl_sync(0xffffffffu, alpha, (lane & ~3) | ((2 * t4 + 1) & 3));
#pragma unroll
            for (int blk = 0; blk < NB; ++blk)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    accv[blk][h][0] *= a_lo;
                    accv[blk][h][2] *= a_lo;
                    accv[blk][h][1] *= a_hi;
                    accv[blk][h][3] *= a_hi;
                }
            m_run = m_new;
        }
        const float p0 = ex2_approx(s0 - m_run), p1 = ex2_approx(s1 - m_run);
        l_run += p0 + p1;

        // ---- value weights: B[k][n] = p(head n, token kappa(k)) * ||v_blk||,
        // kappa(2t) = t, kappa(2t+1) = t + 4, kappa(2t+8) = t + 8, kappa(2t+9) = t + 12;
        // columns n >= 4 repeat heads n - 4 and their outputs are never read
        uint32_t wb0[NB], wb1[NB];
        {
            const uint32_t pk = h2_bits(p0, p1);                 // tokens g, g + 8 of head t4
            const uint32_t x = __shfl_sync(0xffffffffu, pk, 4 * t4 + (g & 3));
            const uint32_t y = __shfl_sync(0xffffffffu, pk, 4 * t4 + 16 + (g & 3));
            const uint32_t pb0 = __byte_perm(x, y, 0x5410u);     // tokens t4, t4 + 4
            const uint32_t pb1 = __byte_perm(x, y, 0x7632u);     // tokens t4 + 8, t4 + 12
            constexpr int NW = NB / 2;                           // norm words per token
            uint32_t n0[NW], n1[NW], n2[NW], n3[NW];
            constexpr int TS = 4 * NB * 2;                       // bytes between tokens t and t + 4
            if constexpr (NW == 2) {
                // one 8-byte load per token (the norm rows are 8-byte aligned)
                const uint2 x0 = lds64<SB>(vn_r), x1 = lds64<SB + TS>(vn_r),
                            x2 = lds64<SB + 2 * TS>(vn_r), x3 = lds64<SB + 3 * TS>(vn_r);
                n0[0] = x0.x; n0[1] = x0.y;
                n1[0] = x1.x; n1[1] = x1.y;
                n2[0] = x2.x; n2[1] = x2.y;
                n3[0] = x3.x; n3[1] = x3.y;
            } else {
                static_for<NW>([&](auto K) {
                    constexpr int k = decltype(K)::value;
                    n0[k] = lds32<SB + 4 * k>(vn_r);
                    n1[k] = lds32<SB + TS + 4 * k>(vn_r);
                    n2[k] = lds32<SB + 2 * TS + 4 * k>(vn_r);
                    n3[k] = lds32<SB + 3 * TS + 4 * k>(vn_r);
                });
            }
#pragma unroll
            for (int blk = 0; blk < NB; ++blk) {
                const uint32_t sel = (blk & 1) ? 0x7632u : 0x5410u;
                wb0[blk] = hmul2_bits(pb0, __byte_perm(n0[blk >> 1], n1[blk >> 1], sel));
                wb1[blk] = hmul2_bits(pb1, __byte_perm(n2[blk >> 1], n3[blk >> 1], sel));
            }
        }

        // ---- values ----
        {
            constexpr int TB = 4 * 4 * S::VW;                    // bytes between tokens t and t + 4
            constexpr uint32_t EM = ((1u << (2 * VB)) - 1u) << 8; // a pair entry at bit 8
            uint32_t gw0[4], gw1[4];             // lane-grouped rows: the lane's words per token
            if constexpr (VG) {
                static_for<4>([&](auto I) {
                    constexpr int i = decltype(I)::value;
                    if constexpr (VB == 4) {
                        const uint2 w = lds64<SB + i * TB>(vg_r);
                        gw0[i] = w.x;
                        gw1[i] = w.y;
                    } else {
                        gw0[i] = lds32<SB + i * TB>(vg_r);
                        gw1[i] = VB == 3 ? lds32<SB + i * TB + 4>(vg_r) : 0u;
                    }
                });
            }
            static_for<NB>([&](auto BLK) {
                constexpr int blk = decltype(BLK)::value;
                uint32_t L0[4], L1[4];
                static_for<4>([&](auto I) {
                    constexpr int i = decltype(I)::value;
                    constexpr int off = SB + i * TB + 4 * VB * blk;
                    // the lane's 4 codes land at bits 8.. of q, so that one
                    // mask-or with the lane address is the first pair's address
                    uint32_t q;
                    if constexpr (VG && VB == 3) {
                        if constexpr (blk == 0) q = __funnelshift_r(gw0[i], gw0[i], gs0);
                        else if constexpr (blk == 1) q = __funnelshift_r(gw0[i], gw1[i], gs1);
                        else if constexpr (blk == 2) q = __funnelshift_rc(gw0[i], gw1[i], gs2);
                        else q = __funnelshift_r(gw1[i], gw1[i], gs3);
                    } else if constexpr (VG && VB == 4) {
                        const uint32_t w = blk < 2 ? gw0[i] : gw1[i];
                        q = __funnelshift_r(w, w, (blk & 1) ? 8u : 24u);
                    } else if constexpr (VG) {
                        q = __funnelshift_r(gw0[i], gw0[i], (uint32_t)((8 * blk + 24) & 31));
                    } else {
                        q = __funnelshift_r(lds32<off>(va_r), lds32<off + 4>(va_r), vq_sh);
                    }
                    L0[i] = lds32((q & EM) | vlane);
                    L1[i] = lds32(((q >> (2 * VB)) & EM) | vlane);
                });
                mma16816(accv[blk][0], __byte_perm(L0[0], L0[1], 0x5410u), __byte_perm(L0[0], L0[1], 0x7632u),
                         __byte_perm(L0[2], L0[3], 0x5410u), __byte_perm(L0[2], L0[3], 0x7632u),
                         wb0[blk], wb1[blk]);
                mma16816(accv[blk][1], __byte_perm(L1[0], L1[1], 0x5410u), __byte_perm(L1[0], L1[1], 0x7632u),
                         __byte_perm(L1[2], L1[3], 0x5410u), __byte_perm(L1[2], L1[3], 0x7632u),
                         wb0[blk], wb1[blk]);
            });
        }
        __syncwarp();
    };
    static_assert(kStages == 3, "the slab loop below unrolls three stages");
    while (n_left > 0) {
        step(std::integral_constant<int, 0>{});
        if (--n_left == 0) break;
        step(std::integral_constant<int, 1>{});
        if (--n_left == 0) break;
        step(std::integral_constant<int, 2>{});
        --n_left;
    }
    cp_async_wait<0>();
    if (!lut_ok) {
        // poison every group this warp owns so that the combine outputs NaN
        reset();
        Cursor c = cursor_at(s_begin);
        for (int64_t n = s_end - s_begin; n > 0; --n) {
            if (c.bhg != cur) {
                if (cur >= 0) flush(cur);
                cur = c.bhg;
            }
            advance(c);
        }
    }
    if (cur >= 0) flush(cur);
}

// ---------------------------------------------------------------------------
// Raw logits on the tensor cores (tq_attn_logits for d = 64/128, up to 128 QJL
// rows).  The 16-token slabs of all (batch, kv head, group of 4 q heads) are
// cut into one contiguous range per CTA, and each CTA's range into one range
// per warp.  A CTA first rotates (and projects) the queries of the at most
// kLgMaxBhg groups its range meets into fragment tables in shared memory;
// then every warp stages its slabs (K codes, K norms, QJL sign words and
// residual norms) with cp.async and runs the decode's score MMAs:
//  * codes: A = 16 tokens x 16 coordinates of fp16 centroid pairs from the
//    per-lane pair table, B = the rotated query in fp16 hi/lo, one
//    accumulator per 32-coordinate block scaled by its fp16 norm;
//  * QJL: A = 16 tokens x 16 projection rows of +-1 (fp16) built from the
//    sign bits, B = sqrt(pi/2)/m (S q~) in fp16 hi/lo; the sum is scaled by
//    the token's fp16 residual norm.
// Lane (g, t) ends with the scores of tokens g and g + 8 for head t.
// ---------------------------------------------------------------------------
constexpr int kLgMaxBhg = 3;
constexpr int kLgMaxM = 128;
constexpr int kLgWarps = 16;

template <int D, int KB>
struct LgCfg {
    // a slab of 16 keys is quick to score, so more of them are kept in flight
    static constexpr int STAGES = KB == 4 ? 5 : 6;
    static constexpr int NB = D / 32;
    static constexpr int KW = NB * KB;
    static constexpr int SZ_KC = kSlab * KW * 4;
    static constexpr int SZ_KN = kSlab * NB * 2;
    static constexpr int SZ_SG = kSlab * (kLgMaxM / 32) * 4;
    static constexpr int SZ_RN = kSlab * 2;
    static constexpr int OFF_KN = SZ_KC;
    static constexpr int OFF_SG = OFF_KN + SZ_KN;
    static constexpr int OFF_RN = OFF_SG + SZ_SG;
    static constexpr int BYTES = OFF_RN + SZ_RN;
    static constexpr int RING = STAGES * BYTES;
    static constexpr int QF = NB * 4;                      // query fragment words per lane
    static constexpr int WF = (kLgMaxM / 16) * 2;          // QJL fragment words per lane
    static_assert(SZ_KC % 16 == 0 && SZ_KN % 16 == 0 && SZ_SG % 16 == 0 && SZ_RN % 16 == 0,
                  "slab sections must be whole 16-byte chunks");
};

template <int D, int KB>
__global__ void __launch_bounds__(32 * kLgWarps, 1)
logits_mma_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CodebookParams kcb,
                  const __grid_constant__ RotParams rp) {
    using S = LgCfg<D, KB>;
    constexpr int NB = S::NB;
    constexpr int NK = 1 << (2 * KB);
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float q_rot[kQH * D];
    __shared__ float w_s[kQH * kLgMaxM];
    __shared__ __align__(16) uint32_t s_qf[kLgMaxBhg][32][S::QF];
    __shared__ __align__(16) uint32_t s_wf[kLgMaxBhg][32][S::WF];
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    // the pair tables go to the first window address with zero low 16 bits;
    // the staging rings fill the space below and after them (the launch
    // provides 64 KiB + tables + all rings)
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t lut_w = (sbase + 0xFFFFu) & ~0xFFFFu;
    const int lut_off = (int)(lut_w - sbase);
    const int ring_a = min(kLgWarps, lut_off / S::RING);
    uint32_t dyn_bytes;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
    if ((uint32_t)(lut_off + kLutBytes + (kLgWarps - ring_a) * S::RING) > dyn_bytes) {
        // the launch sized shared memory for another placement (never
        // expected): poison this CTA's scores instead of overrunning it
        const int64_t T0 = a.mma_slabs, sp0 = a.mma_spb;
        const int G0 = a.n_q_heads / a.n_kv_heads;
        const int64_t c0 = (int64_t)blockIdx.x * T0 / gridDim.x, c1 = ((int64_t)blockIdx.x + 1) * T0 / gridDim.x;
        for (int64_t e = (int64_t)threadIdx.x; e < (c1 - c0) * kQH * kSlab; e += blockDim.x) {
            const int64_t sl = c0 + e / (kQH * kSlab);
            const int hh = (int)((e / kSlab) % kQH);
            const int64_t bhg = sl / sp0, t = (sl - bhg * sp0) * kSlab + e % kSlab;
            const int hg = (int)(bhg % a.mma_groups);
            const int64_t bh = bhg / a.mma_groups;
            if (hg * kQH + hh < G0 && t < a.ctx)
                a.logits[((bh / a.n_kv_heads) * a.n_q_heads + (bh % a.n_kv_heads) * G0 + hg * kQH + hh) * a.ctx + t] =
                    CUDART_NAN_F;
        }
        return;
    }
    {
        uint32_t * lw = reinterpret_cast<uint32_t *>(smem + lut_off);
        for (int i = threadIdx.x; i < NK * 32; i += blockDim.x) {
            const int e = i >> 5, l = i & 31;
            lw[e * 64 + l] = h2_bits(kcb.centroid[e & ((1 << KB) - 1)], kcb.centroid[e >> KB]);
        }
    }
    const bool qjl = a.qjl_signs != nullptr;
    const int m = qjl ? a.qjl_m : 0;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int64_t T = a.mma_slabs, spb = a.mma_spb;
    const int64_t cs = (int64_t)blockIdx.x * T / gridDim.x, ce = ((int64_t)blockIdx.x + 1) * T / gridDim.x;
    const int64_t bhg0 = cs / spb;
    // the launch sizes the CTA ranges so that this is at most kLgMaxBhg
    const int nbhg = ce > cs ? min((int)((ce - 1) / spb - bhg0 + 1), kLgMaxBhg) : 0;

    // ---- this warp's slab range ----
    const int64_t ws0 = cs + (int64_t)wi * (ce - cs) / kLgWarps;
    const int64_t ws1 = cs + ((int64_t)wi + 1) * (ce - cs) / kLgWarps;
    // a range that meets a group beyond the table (never, by the launch's sizing) is skipped
    const bool idle = ws1 <= ws0 || (ws1 - 1) / spb - bhg0 >= kLgMaxBhg;
    const uint32_t ring = sbase + (uint32_t)(wi < ring_a ? wi * S::RING
                                                         : lut_off + kLutBytes + (wi - ring_a) * S::RING);
    const int32_t ctx32 = (int32_t)a.ctx;
    struct Cursor {
        int32_t bhg, ts, hg, row0, rowbase;
    };
    auto cursor_at = [&](int64_t sl) {
        Cursor c;
        const int64_t bhg = sl / spb;
        c.bhg = (int32_t)bhg;
        c.ts = (int32_t)((sl - bhg * spb) * kSlab);
        c.hg = (int32_t)(bhg % a.mma_groups);
        c.rowbase = (int32_t)((bhg / a.mma_groups) * a.ctx);
        c.row0 = c.rowbase + c.ts;
        return c;
    };
    auto advance = [&](Cursor & c) {
        c.ts += kSlab;
        c.row0 += kSlab;
        if (c.ts >= ctx32) {
            c.ts = 0;
            ++c.bhg;
            if (++c.hg == a.mma_groups) {
                c.hg = 0;
                c.rowbase += ctx32;
            }
            c.row0 = c.rowbase;
        }
    };

    // per-lane copy assignment: K code chunks (KB = 4: XOR-swizzled per token),
    // then one chunk of the norm / sign / residual-norm sections
    constexpr int NKC = S::SZ_KC / 16, NKN = S::SZ_KN / 16;
    constexpr int KCL = (NKC + 31) / 32;
    uint32_t kdst[KCL];
#pragma unroll
    for (int j = 0; j < KCL; ++j) {
        const int c = lane + 32 * j;
        int off = 16 * c;
        if constexpr (KB == 4) {
            const int r = c / NB, cc = c % NB;
            off = r * NB * 16 + 16 * (cc ^ kswz<NB>(r));
        }
        kdst[j] = (uint32_t)off;
    }
    const int nsg = qjl ? m / 8 : 0;                        // sign chunks per slab (16 tokens x m/8 bytes / 16)
    const int nrn = qjl ? 2 : 0;
    const int misc = lane < NKN ? 0 : lane < NKN + nsg ? 1 : lane < NKN + nsg + nrn ? 2 : 3;
    const int mc = misc == 0 ? lane : misc == 1 ? lane - NKN : lane - NKN - nsg;
    const int64_t mrow_bytes = misc == 0 ? NB * 2 : misc == 1 ? m / 8 : 2;
    const unsigned char * msrc = misc == 0 ? reinterpret_cast<const unsigned char *>(a.k_norms)
                               : misc == 1 ? reinterpret_cast<const unsigned char *>(a.qjl_signs)
                                           : reinterpret_cast<const unsigned char *>(a.qjl_rnorm);
    const uint32_t mdst = (uint32_t)((misc == 0 ? S::OFF_KN : misc == 1 ? S::OFF_SG : S::OFF_RN) + 16 * mc);
    constexpr int KROW = S::KW * 4;
    auto stage = [&](const Cursor & cu, int st) {
        const uint32_t dst = ring + (uint32_t)(st * S::BYTES);
        const int64_t r0 = cu.row0;
        const int nvalid = min(kSlab, ctx32 - cu.ts);
        const unsigned char * kc = reinterpret_cast<const unsigned char *>(a.k_codes) + r0 * KROW;
#pragma unroll
        for (int j = 0; j < KCL; ++j) {
            const int c = lane + 32 * j;
            if (NKC % 32 == 0 || c < NKC) {
                const int n = nvalid * KROW - 16 * c;
                if (n >= 16) cp_async16_s(dst + kdst[j], kc + 16 * c);
                else cp_async16_zfill_s(dst + kdst[j], n > 0 ? kc + 16 * c : kc, n);
            }
        }
        if (misc < 3) {
            const unsigned char * src = msrc + r0 * mrow_bytes;
            const int n = (int)(nvalid * mrow_bytes) - 16 * mc;
            if (n >= 16) cp_async16_s(dst + mdst, src + 16 * mc);
            else cp_async16_zfill_s(dst + mdst, n > 0 ? src + 16 * mc : src, n);
        }
    };

    // the first copies go out before the fragment tables are built
    Cursor fc = cursor_at(ws0), uc = fc;
    int64_t n_fetch = idle ? 0 : ws1 - ws0;
    int st_fetch = 0;
#pragma unroll
    for (int i = 0; i < S::STAGES - 1; ++i) {
        if (n_fetch > 0) {
            stage(fc, st_fetch);
            advance(fc);
        }
        cp_async_commit();
        --n_fetch;
        st_fetch = st_fetch + 1 == S::STAGES ? 0 : st_fetch + 1;
    }
    // ---- fragment tables of the groups this CTA meets ----
    for (int i = 0; i < nbhg; ++i) {
        const int64_t bhg = bhg0 + i;
        const int hg = (int)(bhg % a.mma_groups);
        const int64_t bh = bhg / a.mma_groups;
        const int b = (int)(bh / a.n_kv_heads), hk = (int)(bh % a.n_kv_heads);
        const int h0 = hk * G + hg * kQH;
        const int nh = min(kQH, G - hg * kQH);
        __syncthreads();
        for (int k = threadIdx.x; k < kQH * D; k += blockDim.x) q_rot[k] = 0.0f;
        for (int k = threadIdx.x; k < kQH * kLgMaxM; k += blockDim.x) w_s[k] = 0.0f;
        __syncthreads();
        rotate_queries(a, rp, b, h0, nh, q_rot);
        if (qjl) {
            // w_s[h][i] = (S q~_h)_i: warp wi takes rows wi, wi + 16, ..., its lanes
            // read the row coalesced and the partial sums meet by shuffles
            // all of this warp's loads first (one round trip), then the sums
            constexpr int RW = kLgMaxM / kLgWarps, JW = D / 32;
            float sv[RW][JW];
#pragma unroll
            for (int k = 0; k < RW; ++k)
#pragma unroll
                for (int jj = 0; jj < JW; ++jj) {
                    const int r = wi + kLgWarps * k;
                    sv[k][jj] = r < m ? a.qjl_f32[(int64_t)r * D + lane + 32 * jj] : 0.0f;
                }
#pragma unroll
            for (int k = 0; k < RW; ++k) {
                const int r = wi + kLgWarps * k;
                float acc[kQH] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int jj = 0; jj < JW; ++jj)
#pragma unroll
                    for (int h = 0; h < kQH; ++h) acc[h] = fmaf(sv[k][jj], q_rot[h * D + lane + 32 * jj], acc[h]);
#pragma unroll
                for (int h = 0; h < kQH; ++h) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
                }
                if (lane == 0 && r < m)
                    for (int h = 0; h < nh; ++h) w_s[h * m + r] = acc[h];
            }
            __syncthreads();
        }
        if (threadIdx.x < 32) {
            const int n = lane >> 2, t = lane & 3, head = n >> 1;
            const bool lo_part = (n & 1) != 0;
            auto frag = [&](float x0, float x1) {
                const __half2 h = __floats2half2_rn(x0, x1);
                const uint32_t v = *reinterpret_cast<const uint32_t *>(&h);
                return lo_part ? h2_bits(x0 - __low2float(h), x1 - __high2float(h)) : v;
            };
            for (int blk = 0; blk < NB; ++blk)
                for (int s2 = 0; s2 < 2; ++s2)
                    for (int r = 0; r < 2; ++r) {
                        const int dim = 32 * blk + 8 * t + 4 * s2 + 2 * r;
                        const float x0 = head < nh ? q_rot[head * D + dim] : 0.0f;
                        const float x1 = head < nh ? q_rot[head * D + dim + 1] : 0.0f;
                        s_qf[i][lane][(blk * 2 + s2) * 2 + r] = frag(x0, x1);
                    }
            // QJL: B[k][n] of chunk c = coef * w[head][16 c + k]; b0 holds k = 2t, 2t + 1,
            // b1 holds k = 2t + 8, 2t + 9
            const float coef = qjl ? 1.2533141373155003f / (float)m : 0.0f;   // sqrt(pi/2) / m
            for (int c = 0; c < kLgMaxM / 16; ++c)
                for (int r = 0; r < 2; ++r) {
                    const int i0 = 16 * c + 2 * t + 8 * r;
                    const bool live = head < nh && i0 < m;
                    const float x0 = live ? coef * w_s[head * m + i0] : 0.0f;
                    const float x1 = live ? coef * w_s[head * m + i0 + 1] : 0.0f;
                    s_wf[i][lane][2 * c + r] = frag(x0, x1);
                }
        }
    }
    __syncthreads();

    if (idle) return;
    const uint32_t klane = lut_w + 4u * (uint32_t)lane;
    uint32_t koff[NB];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
        if constexpr (KB == 4) koff[blk] = (uint32_t)(g * S::KW * 4 + 16 * (blk ^ kswz<NB>(g)) + 4 * t4);
        else koff[blk] = (uint32_t)(g * S::KW * 4 + 4 * (KB * blk + ((8 * KB * t4) >> 5)));
    }
    const int ksh = (8 * KB * t4) & 31;
    const uint32_t kn_off = (uint32_t)(S::OFF_KN + g * NB * 2);
    const int mw = m / 32;                                  // sign words per token
    const uint32_t sg_off = (uint32_t)(S::OFF_SG + g * mw * 4);
    const uint32_t rn_off = (uint32_t)(S::OFF_RN + g * 2);
    const int mchunks = m / 16;

    uint32_t qb[NB][2][2];
    uint32_t wq[kLgMaxM / 16][2];
    int64_t cur = -1;
    auto load_frags = [&](int64_t bhg) {
        const int i = (int)(bhg - bhg0);
        const uint32_t * qf = s_qf[i][lane];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            qb[b][0][0] = qf[4 * b]; qb[b][0][1] = qf[4 * b + 1];
            qb[b][1][0] = qf[4 * b + 2]; qb[b][1][1] = qf[4 * b + 3];
        }
        const uint32_t * wf = s_wf[i][lane];
#pragma unroll
        for (int c = 0; c < kLgMaxM / 16; ++c) { wq[c][0] = wf[2 * c]; wq[c][1] = wf[2 * c + 1]; }
    };

    int st_use = 0;
    for (int64_t n_left = ws1 - ws0; n_left > 0; --n_left) {
        if (n_fetch > 0) {
            stage(fc, st_fetch);
            advance(fc);
        }
        cp_async_commit();
        --n_fetch;
        st_fetch = st_fetch + 1 == S::STAGES ? 0 : st_fetch + 1;
        cp_async_wait<S::STAGES - 1>();
        __syncwarp();
        if (uc.bhg != cur) {
            load_frags(uc.bhg);
            cur = uc.bhg;
        }
        const Cursor cu = uc;
        advance(uc);
        const uint32_t sb = ring + (uint32_t)(st_use * S::BYTES);
        st_use = st_use + 1 == S::STAGES ? 0 : st_use + 1;

        float tot[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        {
            uint32_t kn0[(NB + 1) / 2], kn1[(NB + 1) / 2];
#pragma unroll
            for (int k = 0; k < (NB + 1) / 2; ++k) {
                kn0[k] = lds32(sb + kn_off + 4 * k);
                kn1[k] = lds32(sb + kn_off + 8 * NB * 2 + 4 * k);
            }
#pragma unroll
            for (int blk = 0; blk < NB; ++blk) {
                const uint32_t ka = sb + koff[blk];
                uint32_t w0, w1;
                if constexpr (KB == 4) {
                    w0 = lds32<0>(ka);
                    w1 = lds32<8 * S::KW * 4>(ka);
                } else {
                    w0 = __funnelshift_r(lds32<0>(ka), lds32<4>(ka), ksh);
                    w1 = __funnelshift_r(lds32<8 * S::KW * 4>(ka), lds32<8 * S::KW * 4 + 4>(ka), ksh);
                }
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const uint32_t a0 = lds32(pair_offset<KB>(w0, 2 * s2, klane));
                    const uint32_t a1 = lds32(pair_offset<KB>(w1, 2 * s2, klane));
                    const uint32_t a2 = lds32(pair_offset<KB>(w0, 2 * s2 + 1, klane));
                    const uint32_t a3 = lds32(pair_offset<KB>(w1, 2 * s2 + 1, klane));
                    mma16816(acc, a0, a1, a2, a3, qb[blk][s2][0], qb[blk][s2][1]);
                }
                const float g0 = __half2float(__ushort_as_half((unsigned short)(kn0[blk >> 1] >> (16 * (blk & 1)))));
                const float g1 = __half2float(__ushort_as_half((unsigned short)(kn1[blk >> 1] >> (16 * (blk & 1)))));
                tot[0] = fmaf(g0, acc[0], tot[0]);
                tot[1] = fmaf(g0, acc[1], tot[1]);
                tot[2] = fmaf(g1, acc[2], tot[2]);
                tot[3] = fmaf(g1, acc[3], tot[3]);
            }
        }
        float s0 = tot[0] + tot[1], s1 = tot[2] + tot[3];
        if (qjl) {
            // +-1 pairs from sign bits: bit i -> +1 (set) or -1, as fp16 halves
            float qa[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const uint32_t sa = sb + sg_off;
            // the sign words of tokens g and g + 8 (m / 32 of each)
            uint32_t sw0[kLgMaxM / 32], sw1[kLgMaxM / 32];
            if (mw == 4) {
                uint4 v0, v1;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v0.x), "=r"(v0.y), "=r"(v0.z), "=r"(v0.w) : "r"(sa));
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v1.x), "=r"(v1.y), "=r"(v1.z), "=r"(v1.w) : "r"(sa + 8u * 16u));
                sw0[0] = v0.x; sw0[1] = v0.y; sw0[2] = v0.z; sw0[3] = v0.w;
                sw1[0] = v1.x; sw1[1] = v1.y; sw1[2] = v1.z; sw1[3] = v1.w;
            } else {
#pragma unroll
                for (int k = 0; k < kLgMaxM / 32; ++k) {
                    sw0[k] = k < mw ? lds32(sa + 4 * k) : 0u;
                    sw1[k] = k < mw ? lds32(sa + 8 * mw * 4 + 4 * k) : 0u;
                }
            }
#pragma unroll
            for (int c = 0; c < kLgMaxM / 16; ++c) {
                if (c < mchunks) {
                    const int sh = 16 * (c & 1) + 2 * t4;
                    const uint32_t x0 = sw0[c >> 1] >> sh;      // token g
                    const uint32_t x1 = sw1[c >> 1] >> sh;      // token g + 8
                    // one multiply sends bit 0 to bits 15 and 30 and bit 1 to bits 16 and
                    // 31 (bits 8, 9 likewise with the shifted constant); the mask keeps
                    // 15 and 31, the XOR turns them into fp16 +1 / -1
                    const uint32_t a0 = (((x0 & 3u) * 0x40008000u) & 0x80008000u) ^ 0xBC00BC00u;
                    const uint32_t a1 = (((x1 & 3u) * 0x40008000u) & 0x80008000u) ^ 0xBC00BC00u;
                    const uint32_t a2 = (((x0 & 0x300u) * 0x00400080u) & 0x80008000u) ^ 0xBC00BC00u;
                    const uint32_t a3 = (((x1 & 0x300u) * 0x00400080u) & 0x80008000u) ^ 0xBC00BC00u;
                    mma16816(qa, a0, a1, a2, a3, wq[c][0], wq[c][1]);
                }
            }
            const uint32_t rr = lds32(sb + S::OFF_RN + 4 * (g >> 1));
            const uint32_t rr8 = lds32(sb + S::OFF_RN + 16 + 4 * (g >> 1));
            const float rho0 = __half2float(__ushort_as_half((unsigned short)(rr >> (16 * (g & 1)))));
            const float rho1 = __half2float(__ushort_as_half((unsigned short)(rr8 >> (16 * (g & 1)))));
            s0 = fmaf(rho0, qa[0] + qa[1], s0);
            s1 = fmaf(rho1, qa[2] + qa[3], s1);
        }
        // lane (g, t4): tokens g and g + 8 of head t4
        {
            const int hg = cu.hg;
            const int64_t bh = (int64_t)cu.bhg / a.mma_groups;
            const int b = (int)(bh / a.n_kv_heads), hk = (int)(bh % a.n_kv_heads);
            const int head = hk * G + hg * kQH + t4;
            if (t4 < min(kQH, G - hg * kQH)) {
                float * o = a.logits + ((int64_t)b * a.n_q_heads + head) * a.ctx + cu.ts;
                if (cu.ts + g < ctx32) o[g] = s0;
                if (cu.ts + g + 8 < ctx32) o[g + 8] = s1;
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

template <int D, int KB>
int launch_logits_mma_t(const AttnArgs & a, const CodebookParams & kcb, const RotParams & rp,
                        int64_t ctas, cudaStream_t st) {
    using S = LgCfg<D, KB>;
    auto k = logits_mma_kernel<D, KB>;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
    // dynamic shared memory starts after the reserved area and the static
    // tables; the kernel puts the pair tables at the next window address with
    // zero low 16 bits, rings below them as far as they fit and the rest after
    int reserved = 0;
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, k) != cudaSuccess) return (int)cudaErrorInvalidDeviceFunction;
    const int base = reserved + (int)fa.sharedSizeBytes;
    if (base < 0 || base > 65536) return (int)cudaErrorInvalidConfiguration;
    const int lut_off = (65536 - base) & 0xFFFF;
    const int ring_a = std::min(kLgWarps, lut_off / S::RING);
    const int smem = lut_off + kLutBytes + (kLgWarps - ring_a) * S::RING;
    if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return e;
    k<<<(unsigned)ctas, 32 * kLgWarps, smem, st>>>(a, kcb, rp);
    return (int)cudaGetLastError();
}

template <int D, int KB, int VB, bool QJL, bool PAGED, bool VG = false>
int launch_mma_t(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
                 const RotParams & rp, cudaStream_t st) {
    if constexpr (!VG) {
        // lane-grouped value rows: d = 128 without paging (the paged entry
        // point reads the default order)
        if (a.v_grouped) {
            if constexpr (D == 128 && !PAGED)
                return launch_mma_t<D, KB, VB, QJL, PAGED, true>(a, kcb, vcb, rp, st);
            return (int)cudaErrorInvalidValue;
        }
    }
    using S = SlabCfg<D, KB, VB, QJL>;
    constexpr int WPC = MmaCfg<D, QJL>::WPC;
    // Dynamic shared memory starts right after the per-block reserved area;
    // the pair tables go to the first window address with zero low 16 bits,
    // the warps' staging rings fill the space below and after them.
    int dev = 0;
    cudaGetDevice(&dev);
    int reserved = 0;
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (reserved < 0 || reserved > 65536) return (int)cudaErrorInvalidConfiguration;
    AttnArgs b = a;
    b.mma_lut_off = 65536 - reserved;
    b.mma_ring_a = std::min(WPC, b.mma_lut_off / S::RING);
    const int smem = b.mma_lut_off + kLutBytes + (WPC - b.mma_ring_a) * S::RING;
    auto k = decode_mma_kernel<D, KB, VB, QJL, PAGED, VG>;
    if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return e;
    // programmatic dependent launch: the CTAs start (pair tables, first slab
    // copies) while the prep kernel is still running and wait for its results
    // inside (griddepcontrol.wait)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((a.mma_warps + WPC - 1) / WPC));
    cfg.blockDim = dim3(WPC * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k, b, kcb, vcb);
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
}

template <int D, int KB, bool QJL, bool PAGED>
int mma_vb(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
           const RotParams & rp, cudaStream_t st) {
    switch (a.v_bits) {
        case 2: return launch_mma_t<D, KB, 2, QJL, PAGED>(a, kcb, vcb, rp, st);
        case 3: return launch_mma_t<D, KB, 3, QJL, PAGED>(a, kcb, vcb, rp, st);
        case 4: return launch_mma_t<D, KB, 4, QJL, PAGED>(a, kcb, vcb, rp, st);
    }
    return (int)cudaErrorInvalidValue;
}

template <int D, bool QJL, bool PAGED>
int mma_kb(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
           const RotParams & rp, cudaStream_t st) {
    switch (a.k_bits) {
        case 2: return mma_vb<D, 2, QJL, PAGED>(a, kcb, vcb, rp, st);
        case 3: return mma_vb<D, 3, QJL, PAGED>(a, kcb, vcb, rp, st);
        case 4: return mma_vb<D, 4, QJL, PAGED>(a, kcb, vcb, rp, st);
    }
    return (int)cudaErrorInvalidValue;
}

template <int D>
int launch_mma_decode(const AttnArgs & a, const CodebookParams & kcb, const CodebookParams & vcb,
                      const RotParams & rp, const AppendParams & ap, cudaStream_t st) {
    const int64_t n_bhg = (int64_t)a.batch * a.n_kv_heads * a.mma_groups;
    decode_mma_prep_kernel<D><<<(unsigned)n_bhg, kPrepThreads, 0, st>>>(a, rp, ap);
    int err = (int)cudaGetLastError();
    if (err) return err;
    if (a.qjl_signs != nullptr) {
        if (a.page_size != 0) return (int)cudaErrorInvalidValue;
        if constexpr (D <= 128) return mma_kb<D, true, false>(a, kcb, vcb, rp, st);
        return (int)cudaErrorInvalidValue;
    }
    if (a.page_size != 0) return mma_kb<D, false, true>(a, kcb, vcb, rp, st);
    return mma_kb<D, false, false>(a, kcb, vcb, rp, st);
}

template <int D>
size_t mma_smem_bytes(int kb, int vb, bool qjl) {
    // upper bound (tables placed at the next 64 KiB window boundary)
    const int NB = D / 32;
    const int slab = kSlab * (NB * kb * 4 + NB * 2 + NB * vb * 4 + NB * 2 +
                              (qjl ? kMmaMaxM / 8 + 2 : 0));
    const int wpc = qjl ? MmaCfg<D, true>::WPC : MmaCfg<D, false>::WPC;
    return (size_t)65536 + kLutBytes + (size_t)wpc * kStages * slab;
}

RotParams rot_params(const tq_rotation * rot) {
    RotParams rp{};
    for (int i = 0; i < 8; ++i) {
        rp.d1_bits[i] = rot->d1_bits[i];
        rp.d2_bits[i] = rot->d2_bits[i];
    }
    return rp;
}

// ---------------------------------------------------------------------------
// Maximum-inner-product search over packed rows ("Google TurboQuant deep
// dive", sec. 3.4: the codes serve vector search).  Scores are the decode's
// raw logits, <R q, x_hat_j> (upstream guide sec. 5.3), for up to eight
// queries per warp: B = the rotated queries in fp16 (one column per query),
// A = 16 rows x 16 coordinates of fp16 centroid pairs from the per-lane pair
// table, one accumulator per 32-coordinate block scaled by its fp16 norm.
// The database is cut into 16-row slabs; every warp streams one contiguous
// slab range (cp.async ring, as in the decode) for one group of eight
// queries, and writes its scores to the score matrix [n_queries][n_db].  A
// second kernel keeps the k largest of every query's row.
// ---------------------------------------------------------------------------
constexpr int kSearchWarps = 16;
constexpr int kSearchQ = 8;           // queries per warp (the MMA's N)
constexpr int kTopkChunk = 2048;      // keys sorted per CTA in the top-k passes
constexpr int kTopkThreads = 512;

// Order-preserving 64-bit key of (score, row): larger key = larger score,
// and for equal scores the smaller row.  NaN sorts below every number.
__device__ __forceinline__ uint64_t topk_key(float s, uint32_t row) {
    uint32_t u = __float_as_uint(s);
    if (s != s) u = 0u;                                         // NaN -> smallest
    else u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - row);
}
__device__ __forceinline__ float topk_score(uint64_t key) {
    uint32_t u = (uint32_t)(key >> 32);
    u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
    return __uint_as_float(u);
}
__device__ __forceinline__ int32_t topk_row(uint64_t key) {
    return (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

template <int D, int KB>
struct SearchCfg {
    static constexpr int NB = D / 32;
    static constexpr int KW = NB * KB;
    static constexpr int SZ_KC = kSlab * KW * 4;
    static constexpr int SZ_KN = kSlab * NB * 2;
    static constexpr int OFF_KN = SZ_KC;
    static constexpr int BYTES = SZ_KC + SZ_KN;
    static constexpr int RING = kStages * BYTES;
    static_assert(SZ_KC % 16 == 0 && SZ_KN % 16 == 0, "slab sections must be whole 16-byte chunks");
};

// fp16 B fragments of the rotated queries of group qg (eight queries, column
// n = query qg * 8 + n): for lane l (n = l / 4, t = l % 4), block b and k step
// s, words (b * 2 + s) * 2 + {0, 1} hold dims 32 b + 8 t + 4 s + {0, 1} and
// {2, 3}.  Missing queries are zero columns.
template <int D>
__global__ void __launch_bounds__(kThreads)
search_prep_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ RotParams rp) {
    constexpr int NB = D / 32;
    __shared__ float q_rot[kSearchQ * D];
    const int qg = blockIdx.x;
    const int q0 = qg * kSearchQ;
    const int nq = min(kSearchQ, a.n_q_heads - q0);
    for (int i = threadIdx.x; i < kSearchQ * D; i += blockDim.x) q_rot[i] = 0.0f;
    __syncthreads();
    rotate_queries(a, rp, 0, q0, nq, q_rot);
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x, n = lane >> 2, t = lane & 3;
        uint32_t * dst = a.mma_qfrag + ((int64_t)qg * 32 + lane) * (NB * 4);
        for (int blk = 0; blk < NB; ++blk)
            for (int s = 0; s < 2; ++s)
                for (int r = 0; r < 2; ++r) {
                    const int dim = 32 * blk + 8 * t + 4 * s + 2 * r;
                    dst[(blk * 2 + s) * 2 + r] = h2_bits(q_rot[n * D + dim], q_rot[n * D + dim + 1]);
                }
    }
}

// TOPK (k <= kSearchHeapK): instead of writing the score matrix, every warp
// keeps the k largest keys of each of its 8 queries as a descending list
// spread over its lanes (lane i holds the i-th key, in a register); a score
// is a candidate only above the list's last key, so insertions (one ballot
// for the position and one shuffle to shift the tail) are rare once the lists
// have filled.  At the end the warp writes its lists to cand_keys[q][warp][k];
// the top-k passes then reduce the candidates.
constexpr int kSearchHeapK = 32;

template <int D, int KB, bool TOPK>
__global__ void __launch_bounds__(32 * kSearchWarps, 1)
search_scores_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CodebookParams kcb,
                     int32_t topk, uint64_t * __restrict__ cand_keys) {
    using S = SearchCfg<D, KB>;
    constexpr int NB = S::NB;
    constexpr int NK = 1 << (2 * KB);
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const uint32_t lut_w = (uint32_t)__cvta_generic_to_shared(smem) + (uint32_t)a.mma_lut_off;
    const bool lut_ok = (lut_w & 0xFFFFu) == 0u;
    if (lut_ok) {
        uint32_t * lw = reinterpret_cast<uint32_t *>(smem + a.mma_lut_off);
        for (int i = threadIdx.x; i < NK * 32; i += blockDim.x) {
            const int e = i >> 5, l = i & 31;
            lw[e * 64 + l] = h2_bits(kcb.centroid[e & ((1 << KB) - 1)], kcb.centroid[e >> KB]);
        }
    }
    __syncthreads();
    const int qg = blockIdx.y;
    const int64_t n_db = a.ctx;
    const int64_t T = (n_db + kSlab - 1) / kSlab;
    const int64_t W = (int64_t)gridDim.x * kSearchWarps;
    const int64_t gw = (int64_t)blockIdx.x * kSearchWarps + wi;
    const int64_t s_begin = gw * T / W, s_end = (gw + 1) * T / W;
    // per query jq of the group: lane i < topk holds the i-th largest key so
    // far in list_s[jq * 32 + i] (0 = empty, below every real key); the lists
    // of every warp sit after the rings
    uint64_t * list_s = reinterpret_cast<uint64_t *>(
        smem + a.mma_lut_off + kLutBytes + (kSearchWarps - a.mma_ring_a) * S::RING) +
        (int64_t)wi * kSearchQ * 32;
    // the last kept key of this lane's two queries 2 t4 and 2 t4 + 1
    uint64_t thr[2] = {0ull, 0ull};
    if constexpr (TOPK) {
        for (int i = lane; i < kSearchQ * 32; i += 32) list_s[i] = 0ull;
        __syncwarp();
    } else {
        if (s_end <= s_begin) return;
    }
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(smem) +
                          (uint32_t)(wi < a.mma_ring_a ? wi * S::RING
                                                       : a.mma_lut_off + kLutBytes + (wi - a.mma_ring_a) * S::RING);
    // query fragments of this group
    uint32_t qb[NB][2][2];
    {
        const uint4 * src = reinterpret_cast<const uint4 *>(a.mma_qfrag + ((int64_t)qg * 32 + lane) * (NB * 4));
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const uint4 v = src[b];
            qb[b][0][0] = v.x; qb[b][0][1] = v.y; qb[b][1][0] = v.z; qb[b][1][1] = v.w;
        }
    }
    constexpr int NKC = S::SZ_KC / 16, NKN = S::SZ_KN / 16;
    constexpr int KCL = (NKC + 31) / 32;
    constexpr int KROW = S::KW * 4, NROW = NB * 2;
    uint32_t kdst[KCL];
#pragma unroll
    for (int j = 0; j < KCL; ++j) {
        const int c = lane + 32 * j;
        int off = 16 * c;
        if constexpr (KB == 4) {
            const int r = c / NB, cc = c % NB;
            off = r * NB * 16 + 16 * (cc ^ kswz<NB>(r));
        }
        kdst[j] = (uint32_t)off;
    }
    // per-lane source bases; destinations as window addresses in stage 0 of
    // the ring (the stage offset is an immediate of each copy and load)
    const unsigned char * kc_l = reinterpret_cast<const unsigned char *>(a.k_codes) + 16 * lane;
    const unsigned char * ns_l = reinterpret_cast<const unsigned char *>(a.k_norms) + 16 * lane;
#pragma unroll
    for (int j = 0; j < KCL; ++j) kdst[j] += ring;
    const uint32_t ndst = ring + (uint32_t)(S::OFF_KN + 16 * lane);
    // copies of slab sl into the stage at byte offset fb of the ring
    auto stage = [&](int64_t sl, uint32_t fb) {
        const int64_t r0 = sl * kSlab;
        if (r0 + kSlab <= n_db) {
            const unsigned char * ks = kc_l + r0 * KROW;
#pragma unroll
            for (int j = 0; j < KCL; ++j)
                if (NKC % 32 == 0 || lane + 32 * j < NKC) cp_async16_s(kdst[j] + fb, ks + 512 * j);
            if (lane < NKN) cp_async16_s(ndst + fb, ns_l + r0 * NROW);
        } else {
            // ragged last slab: copy the valid bytes, zero the rest
            const int nvalid = (int)(n_db - r0);
            const unsigned char * kc = reinterpret_cast<const unsigned char *>(a.k_codes) + r0 * KROW;
#pragma unroll
            for (int j = 0; j < KCL; ++j) {
                const int c = lane + 32 * j;
                if (NKC % 32 == 0 || c < NKC) {
                    const int n = nvalid * KROW - 16 * c;
                    cp_async16_zfill_s(kdst[j] + fb, n > 0 ? kc + 16 * c : kc, n);
                }
            }
            if (lane < NKN) {
                const unsigned char * ns = reinterpret_cast<const unsigned char *>(a.k_norms) + r0 * NROW;
                const int n = nvalid * NROW - 16 * lane;
                cp_async16_zfill_s(ndst + fb, n > 0 ? ns + 16 * lane : ns, n);
            }
        }
    };
    const uint32_t klane = lut_w + 4u * (uint32_t)lane;
    uint32_t kb_r[NB];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
        if constexpr (KB == 4) kb_r[blk] = ring + (uint32_t)(g * S::KW * 4 + 16 * (blk ^ kswz<NB>(g)) + 4 * t4);
        else kb_r[blk] = ring + (uint32_t)(g * S::KW * 4 + 4 * (KB * blk + ((8 * KB * t4) >> 5)));
    }
    const int ksh = (8 * KB * t4) & 31;
    const uint32_t kn_r = ring + (uint32_t)(S::OFF_KN + g * NB * 2);
    const int q0 = qg * kSearchQ + 2 * t4;            // this lane's two queries
    float * out0 = a.logits + (int64_t)q0 * n_db;
    float * out1 = out0 + n_db;
    const bool live0 = q0 < a.n_q_heads, live1 = q0 + 1 < a.n_q_heads;
    const float bad = lut_ok ? 0.0f : CUDART_NAN_F;
    // score of each query's last kept key: a score below it cannot enter (an
    // unfilled list's last key decodes as NaN, which lets every score through)
    float thr_s[2] = {CUDART_NAN_F, CUDART_NAN_F};

    int64_t fetch = s_begin;
    const bool copy = lut_ok;                // an unusable table layout copies nothing (output NaN)
    uint32_t fb = 0;
    for (int i = 0; i < kStages - 1; ++i) {
        if (copy && fetch < s_end) stage(fetch++, fb);
        cp_async_commit();
        fb = fb + S::BYTES == (uint32_t)S::RING ? 0u : fb + S::BYTES;
    }
    uint32_t sb = 0;
    // (a plain loop: the candidate path below is long, and three unrolled
    // copies of it overflow the instruction cache)
    for (int64_t sl = s_begin; sl < s_end; ++sl) {
        if (copy && fetch < s_end) stage(fetch++, fb);
        cp_async_commit();
        fb = fb + S::BYTES == (uint32_t)S::RING ? 0u : fb + S::BYTES;
        cp_async_wait<kStages - 1>();
        __syncwarp();
        float tot[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        {
            uint32_t kn0[(NB + 1) / 2], kn1[(NB + 1) / 2];
#pragma unroll
            for (int k = 0; k < (NB + 1) / 2; ++k) {
                kn0[k] = lds32(kn_r + sb + 4 * k);
                kn1[k] = lds32(kn_r + sb + 8 * NB * 2 + 4 * k);
            }
#pragma unroll
            for (int blk = 0; blk < NB; ++blk) {
                const uint32_t ka = kb_r[blk] + sb;
                uint32_t w0, w1;
                if constexpr (KB == 4) {
                    w0 = lds32<0>(ka);
                    w1 = lds32<8 * S::KW * 4>(ka);
                } else {
                    w0 = __funnelshift_r(lds32<0>(ka), lds32<4>(ka), ksh);
                    w1 = __funnelshift_r(lds32<8 * S::KW * 4>(ka), lds32<8 * S::KW * 4 + 4>(ka), ksh);
                }
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const uint32_t a0 = lds32(pair_offset<KB>(w0, 2 * s2, klane));
                    const uint32_t a1 = lds32(pair_offset<KB>(w1, 2 * s2, klane));
                    const uint32_t a2 = lds32(pair_offset<KB>(w0, 2 * s2 + 1, klane));
                    const uint32_t a3 = lds32(pair_offset<KB>(w1, 2 * s2 + 1, klane));
                    mma16816(acc, a0, a1, a2, a3, qb[blk][s2][0], qb[blk][s2][1]);
                }
                const float g0 = __half2float(__ushort_as_half((unsigned short)(kn0[blk >> 1] >> (16 * (blk & 1)))));
                const float g1 = __half2float(__ushort_as_half((unsigned short)(kn1[blk >> 1] >> (16 * (blk & 1)))));
                tot[0] = fmaf(g0, acc[0], tot[0]);
                tot[1] = fmaf(g0, acc[1], tot[1]);
                tot[2] = fmaf(g1, acc[2], tot[2]);
                tot[3] = fmaf(g1, acc[3], tot[3]);
            }
        }
        sb = sb + S::BYTES == (uint32_t)S::RING ? 0u : sb + S::BYTES;
        // lane (g, t4): rows g and g + 8 for queries q0 and q0 + 1
        const int64_t r = sl * kSlab + g;
        if constexpr (TOPK) {
            bool cand[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool live = (e & 1 ? live1 : live0) && r + 8 * (e >> 1) < n_db;
                cand[e] = live && !(tot[e] + bad < thr_s[e & 1]);
            }
            if (__any_sync(0xffffffffu, cand[0] || cand[1] || cand[2] || cand[3])) {
                uint64_t key[4];
                uint32_t lm = 0u;                // bit 2 jq + h: a candidate of query jq, row g + 8 h
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    key[e] = topk_key(tot[e] + bad, (uint32_t)(r + 8 * (e >> 1)));
                    if (cand[e] && key[e] > thr[e & 1]) lm |= 1u << (2 * (2 * t4 + (e & 1)) + (e >> 1));
                }
                uint32_t qm = __reduce_or_sync(0xffffffffu, lm);
                while (qm != 0u) {
                    const int idx = __ffs(qm) - 1;
                    qm &= qm - 1u;
                    const int jq = idx >> 1, e = (jq & 1) + 2 * (idx & 1);
                    const uint64_t ke = e == 0 ? key[0] : e == 1 ? key[1] : e == 2 ? key[2] : key[3];
                    uint64_t * L = list_s + jq * 32;
                    uint64_t cur = L[lane];
                    uint64_t last = __shfl_sync(0xffffffffu, cur, topk - 1);
                    bool cnd = ((lm >> idx) & 1u) && ke > last;
                    uint32_t m = __ballot_sync(0xffffffffu, cnd);
                    while (m != 0u) {
                        const int src = __ffs(m) - 1;
                        const uint64_t c = __shfl_sync(0xffffffffu, ke, src);
                        // position = number of kept keys above c
                        const int pos = __popc(__ballot_sync(0xffffffffu, lane < topk && cur > c));
                        const uint64_t up = __shfl_up_sync(0xffffffffu, cur, 1);
                        if (lane > pos) cur = up;
                        if (lane == pos) cur = c;
                        last = __shfl_sync(0xffffffffu, cur, topk - 1);
                        cnd = cnd && lane != src && ke > last;
                        m = __ballot_sync(0xffffffffu, cnd);
                    }
                    L[lane] = cur;
                    if (t4 == (jq >> 1)) {
                        if (jq & 1) {
                            thr[1] = last;
                            thr_s[1] = topk_score(last);
                        } else {
                            thr[0] = last;
                            thr_s[0] = topk_score(last);
                        }
                    }
                }
                __syncwarp();
            }
        } else {
            if (r < n_db) {
                if (live0) out0[r] = tot[0] + bad;
                if (live1) out1[r] = tot[1] + bad;
            }
            if (r + 8 < n_db) {
                if (live0) out0[r + 8] = tot[2] + bad;
                if (live1) out1[r + 8] = tot[3] + bad;
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if constexpr (TOPK) {
        // this warp's candidates: cand_keys[(q * W + gw) * topk + i]
        for (int jq = 0; jq < kSearchQ; ++jq) {
            const int q = qg * kSearchQ + jq;
            if (q < a.n_q_heads && lane < topk) cand_keys[((int64_t)q * W + gw) * topk + lane] = list_s[jq * 32 + lane];
        }
    }
}

// ---------------------------------------------------------------------------
// Top-k search on the tensor cores (d = 64 / 128, k <= kStMaxK).  The scores of
// up to 128 queries against a tile of 128 database rows are one tcgen05 GEMM,
// D[m][n] = sum_j q_j B[n][j], with B the tile dequantized once into shared
// memory for every query: B[n][j] = c[idx_j] * (gamma_blk / s_n) in fp16, s_n
// the row's largest block norm (every product stays in [-1, 1] times a
// centroid, so no block underflows against the others); the score is s_n D.
// One CTA walks the tiles x, x + gridDim.x, ... of the database with
// specialised warps that hand tiles on through mbarriers:
//  * a copying warp: codes and norms by bulk copies (no tensor map, no
//    multicast) into a ring of kStStages stages, each stage refilled as soon
//    as the dequantization warps release it, completing on an mbarrier per
//    stage;
//  * 4 dequantization warps per 32-coordinate block (16 at d = 128): every
//    thread turns one block of a row into the 128-byte swizzled K-major
//    operand layout (per-lane fp16 pair tables, as the decode) in one of two
//    B buffers;
//  * an issuing warp: the tile's MMAs into one of two TMEM accumulators once
//    its B buffer is written and the accumulator has been read (the copy and
//    MMA instructions hold their thread about as long as the hardware takes
//    to carry them out, so each kind has a warp of its own);
//  * 8 scan warps, two per TMEM lane quarter: the thread of lane m and half h
//    reads half of lane m's columns (query m, or with at most 64 queries,
//    held twice in the operand, query m % 64 over a quarter of the columns),
//    scales by s_n and keeps its k best keys in shared memory; at the end the
//    two halves of a lane merge into one list.  A score enters
//    a list only if it is not below the larger of the list's k-th score and a
//    per-query bound in global memory: the k-th largest column maximum of a
//    sample pass, raised by every list's k-th score as the lists fill (k keys
//    at or above the bound exist, so a lower score cannot be among the k).
// Every wait is bounded; a CTA that gives up writes empty lists (key 0: row
// -1, score NaN).
// ---------------------------------------------------------------------------
constexpr int kStRows = 128;        // database rows per tile (the MMA's N)
constexpr int kStQ = 128;           // rows of the query operand (the MMA's M)
constexpr int kStScanWarps = 8;
constexpr int kStScanThreads = 32 * kStScanWarps;
constexpr int kStScratch = 32;      // bytes of candidate scratch per scan thread
// one dequantization thread per 32-coordinate block of the tile's 128 rows
__host__ __device__ constexpr int st_deq_threads(int d) { return 128 * (d / 32); }
// dequantization warps, then the scan warps, then one warp that issues the MMAs and one
// that issues the copies
__host__ __device__ constexpr int st_threads(int d) { return st_deq_threads(d) + 32 * kStScanWarps + 64; }
constexpr int kStMaxK = 16;
constexpr int kStStages = 6;        // staging ring of codes and norms
constexpr int kStSampleTiles = 4;   // tiles per CTA of the sample pass
constexpr uint64_t kStWaitNs = 1000000000ull;

template <int D, int KB>
struct StCfg {
    static constexpr int NB = D / 32;
    static constexpr int KW = NB * KB;                  // code words per row
    static constexpr int CODE_BYTES = kStRows * KW * 4;
    static constexpr int NORM_BYTES = kStRows * NB * 2;
    static constexpr int STAGE = CODE_BYTES + NORM_BYTES;
    static constexpr int SLICE = 128 * 128;             // 64 fp16 columns of 128 rows, swizzled
    static constexpr int A_BYTES = kStQ * D * 2;
    static constexpr int B_BYTES = kStRows * D * 2;
    // below the pair table: A, four rows of score scales, the mbarriers
    // (bfree[2], accfull[2], accfree[2], sfull[4], full[kStStages], bfull[2],
    // empty[kStStages]), the TMEM address, the error flag and the MMA count,
    // then the low ring stages
    static constexpr int OFF_SCALE = A_BYTES;
    static constexpr int OFF_BAR = OFF_SCALE + 4 * kStRows * 4;
    static constexpr int OFF_TMEM = OFF_BAR + 8 * (12 + 2 * kStStages);
    static constexpr int OFF_ERR = OFF_TMEM + 4;
    static constexpr int OFF_ISSUED = OFF_TMEM + 8;
    static constexpr int LOW_FIXED = (OFF_TMEM + 12 + 15) / 16 * 16;
    // from the pair table up: 256 entries of 256 bytes (the table in the low
    // 128 bytes of entry e, the list of scan thread e in the high 128), the two
    // B tiles, then the high ring stages
    static constexpr int HIGH_B = 65536;
    static constexpr int HIGH_FIXED = HIGH_B + 2 * B_BYTES;
    static_assert(D == 64 || D == 128, "tensor-core search: d = 64 or 128");
    static_assert(STAGE % 16 == 0 && LOW_FIXED % 16 == 0, "16-byte copies");
};

// A load from the pair table, which no thread writes after the prologue: not
// volatile, so the compiler may batch the lookups of a row.
__device__ __forceinline__ uint32_t lds32_table(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t * p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Rotated queries as fp16 rows (the A operand of the search) and the shared
// per-query bounds reset to "none"; one CTA per query.
template <int D>
__global__ void __launch_bounds__(kThreads)
search_qrows_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ RotParams rp,
                    __half * __restrict__ qrows, uint32_t * __restrict__ bound) {
    pdl_launch_dependents();
    __shared__ float q_rot[D];
    const int q = blockIdx.x;
    rotate_queries(a, rp, 0, q, 1, q_rot);
    for (int i = threadIdx.x; i < D; i += blockDim.x) qrows[(int64_t)q * D + i] = __float2half_rn(q_rot[i]);
    if (threadIdx.x == 0) bound[q] = 0u;
}

// REP = 2: at most 64 queries, each held twice in the query operand.
// SAMPLE: keep no lists; every scan thread's list is the largest score of its
// columns of the tile (one key, then zeros), so that the k-th largest of all
// these keys is a score reached by k distinct rows.
template <int D, int KB, int REP, bool SAMPLE>
__global__ void __launch_bounds__(st_threads(D), 1)
search_tc_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CodebookParams kcb,
                 const __half * __restrict__ qrows, uint32_t * __restrict__ bound, int32_t topk,
                 int32_t n_low, int32_t tile0, int32_t tile1, int32_t lists_stride, int32_t list0,
                 uint64_t * __restrict__ cand_keys) {
    using C = StCfg<D, KB>;
    constexpr int NB = C::NB, KW = C::KW;
    constexpr int NQA = kStQ / REP;                      // queries per CTA row of the grid
    constexpr int WID = 64 / REP;                        // columns one scan thread reads per tile
    constexpr int NK = 1 << (2 * KB);
    constexpr int NT = st_threads(D), DQT = st_deq_threads(D);
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t lut_w = sbase + (uint32_t)a.mma_lut_off;
    // the pair table needs a window address with zero low 16 bits, the
    // swizzled operands 1024-byte alignment
    const bool lut_ok = (lut_w & 0xFFFFu) == 0u && (sbase & 1023u) == 0u;
    unsigned char * high = smem + a.mma_lut_off;
    const uint32_t bar = sbase + (uint32_t)C::OFF_BAR;
    const uint32_t bfree = bar, accfull = bar + 16u, accfree = bar + 32u, sfull = bar + 48u, full = bar + 80u;
    const uint32_t bfull = full + 8u * kStStages, empty = bfull + 16u;
    volatile int * s_err = reinterpret_cast<volatile int *>(smem + C::OFF_ERR);
    float * scale = reinterpret_cast<float *>(smem + C::OFF_SCALE);
    const int q0 = blockIdx.y * NQA;
    const int nq = min(NQA, a.n_q_heads - q0);
    const int64_t n_db = a.ctx;
    // this CTA's tiles: tile0 + x, tile0 + x + gridDim.x, ... below tile1
    const int n_span = tile1 - tile0;
    const int n_my = lut_ok && (int)blockIdx.x < n_span ? (n_span - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const bool deq = tid < DQT;
    const int stid = tid - DQT;                          // scan thread = TMEM lane
    const bool issuer_warp = tid >= DQT + 32 * kStScanWarps;
    constexpr int DQW = DQT / 32;

    // pair table; lists: slot i of scan thread t at byte 256 t + 128 + 8 ((i + t) % 16)
    {
        uint32_t * lw = reinterpret_cast<uint32_t *>(high);
        for (int i = tid; i < NK * 32; i += NT) {
            const int e = i >> 5, l = i & 31;
            lw[e * 64 + l] = h2_bits(kcb.centroid[e & ((1 << KB) - 1)], kcb.centroid[e >> KB]);
        }
        if (!deq && !issuer_warp) {
            uint64_t * mine = reinterpret_cast<uint64_t *>(high + 256 * stid + 128);
#pragma unroll
            for (int i = 0; i < 16; ++i) mine[i] = 0ull;
        }
    }
    // the copying thread initialises the mbarriers (it is the first to use
    // them: its copies start before the block-wide barrier below)
    const bool issuer = tid == NT - 64, copier = tid == NT - 32;
    if (copier) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bfree + 8u * i, 1);
            tc::mbar_init(accfull + 8u * i, 1);
            tc::mbar_init(accfree + 8u * i, 32 * kStScanWarps);
        }
        for (int i = 0; i < 4; ++i) tc::mbar_init(sfull + 8u * i, kStRows);
        for (int i = 0; i < kStStages; ++i) {
            tc::mbar_init(full + 8u * i, 1);
            tc::mbar_init(empty + 8u * i, DQW);
        }
        for (int i = 0; i < 2; ++i) tc::mbar_init(bfull + 8u * i, DQW);
        *s_err = 0;
        *reinterpret_cast<int *>(smem + C::OFF_ISSUED) = 0;
    }
    if (warp == 0) tc::tmem_alloc(sbase + (uint32_t)C::OFF_TMEM, 256);

    auto stage_ptr = [&](int s) -> unsigned char * {
        return s < n_low ? smem + C::LOW_FIXED + s * C::STAGE : high + C::HIGH_FIXED + (s - n_low) * C::STAGE;
    };
    // the copying thread copies this CTA's tile k (codes, then norms) into stage
    // k % kStStages with two bulk copies completing on full[stage]; the bytes
    // of a ragged last tile past the last 16-byte boundary by plain copies
    // (rows past the database keep stale values: their columns are never read)
    int copies = 0;
    auto issue = [&](int k) {
        if (k >= n_my) return;
        const int64_t r0 = ((int64_t)tile0 + blockIdx.x + (int64_t)k * gridDim.x) * kStRows;
        const int nvalid = (int)min((int64_t)kStRows, n_db - r0);
        const unsigned char * kc = reinterpret_cast<const unsigned char *>(a.k_codes) + r0 * (KW * 4);
        const unsigned char * kn = reinterpret_cast<const unsigned char *>(a.k_norms) + r0 * (NB * 2);
        unsigned char * st_p = stage_ptr(k % kStStages);
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(st_p);
        const uint32_t fb = full + 8u * (uint32_t)(k % kStStages);
        const int cb = nvalid * KW * 4, nbb = nvalid * NB * 2;
        const int cb16 = cb & ~15, nb16 = nbb & ~15;
        for (int i = cb16; i < cb; i += 4)
            *reinterpret_cast<uint32_t *>(st_p + i) = *reinterpret_cast<const uint32_t *>(kc + i);
        for (int i = nb16; i < nbb; i += 4)
            *reinterpret_cast<uint32_t *>(st_p + C::CODE_BYTES + i) = *reinterpret_cast<const uint32_t *>(kn + i);
        tc::mbar_arrive_expect_tx(fb, (uint32_t)(cb16 + nb16));
        if (cb16 > 0) tc::bulk_load(dst, kc, (uint32_t)cb16, fb);
        if (nb16 > 0) tc::bulk_load(dst + (uint32_t)C::CODE_BYTES, kn, (uint32_t)nb16, fb);
        ++copies;
    };
    if (copier)
        for (int k = 0; k < kStStages; ++k) issue(k);   // every stage starts free

    pdl_wait();                          // the query rows and the bounds
    // A: query q0 + m % NQA in row m; missing queries are zero rows
    for (int i = tid; i < kStQ * (D / 8); i += NT) {
        const int m = i / (D / 8), c = i % (D / 8);
        const int qm = m % NQA;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (qm < nq) v = *reinterpret_cast<const uint4 *>(qrows + (int64_t)(q0 + qm) * D + 8 * c);
        *reinterpret_cast<uint4 *>(smem + (c >> 3) * C::SLICE + m * 128 + 16 * ((c & 7) ^ (m & 7))) = v;
    }
    tc::fence_proxy_async();             // A, written by generic stores, is read by the MMAs
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<const uint32_t *>(smem + C::OFF_TMEM);

    if (issuer_warp) {
        // ---- copying thread: tile k + kStStages - 1 into the stage that tile
        // k - 1 released (the copy and MMA instructions hold their thread
        // about as long as the hardware takes to carry them out, so each
        // kind has a warp of its own) ----
        if (copier) {
            bool ok = true;
            for (int k = 1; k < n_my && ok; ++k) {
                ok = tc::mbar_wait(empty + 8u * (uint32_t)((k - 1) % kStStages), (uint32_t)(((k - 1) / kStStages) & 1), kStWaitNs);
                if (ok) issue(k + kStStages - 1);
            }
            if (!ok) *s_err = 1;
            // the last copy into every stage lands before the CTA ends
            for (int t = max(0, copies - kStStages); t < copies; ++t)
                tc::mbar_wait(full + 8u * (uint32_t)(t % kStStages), (uint32_t)((t / kStStages) & 1), kStWaitNs);
        }
        // ---- issuing thread: the MMAs of every tile once its B buffer is
        // written and its accumulator was read ----
        if (issuer) {
            constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(kStRows >> 3) << 17) | ((uint32_t)(kStQ >> 4) << 24);
            bool ok = true;
            int issued = 0;
            for (int k = 0; k < n_my && ok; ++k) {
                const int b = k & 1;
                ok = tc::mbar_wait(bfull + 8u * b, (uint32_t)((k >> 1) & 1), kStWaitNs) &&
                     (k < 2 || tc::mbar_wait(accfree + 8u * b, (uint32_t)(((k >> 1) & 1) ^ 1), kStWaitNs)) &&
                     *s_err == 0;
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t b0 = lut_w + (uint32_t)(C::HIGH_B + b * C::B_BYTES);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * C::SLICE + (ks & 3) * 32);
                    tc::mma_bf16(tmem + (uint32_t)(b * kStRows), tc::smem_desc_sw128(sbase + off),
                                 tc::smem_desc_sw128(b0 + off), idesc, ks > 0 ? 1u : 0u);
                }
                tc::commit(accfull + 8u * b);
                tc::commit(bfree + 8u * b);
                ++issued;
            }
            if (!ok) *s_err = 1;
            *reinterpret_cast<int *>(smem + C::OFF_ISSUED) = issued;
        }
        __syncwarp();
    } else if (deq) {
        // ---- dequantization warps: block blk of row r of the tile ----
        const int r = tid & (kStRows - 1), blk = tid >> 7;
        const uint32_t lane_off = lut_w + 4u * (uint32_t)lane;
        for (int k = 0; k < n_my; ++k) {
            const int b = k & 1;
            // tile k is in, and B[b] was read by MMA(k - 2)
            const bool go = tc::mbar_wait(full + 8u * (uint32_t)(k % kStStages), (uint32_t)((k / kStStages) & 1), kStWaitNs) &&
                            (k < 2 || tc::mbar_wait(bfree + 8u * b, (uint32_t)(((k >> 1) & 1) ^ 1), kStWaitNs)) &&
                            *s_err == 0;
            if (!__all_sync(0xffffffffu, go)) {
                *s_err = 1;
                break;
            }
            const unsigned char * cs = stage_ptr(k % kStStages);
            const unsigned char * nr = cs + C::CODE_BYTES + r * NB * 2;
            const float gb_ = __half2float(*reinterpret_cast<const __half *>(nr + 2 * blk));
            float g[NB];
            if constexpr (NB == 4) {
                const uint2 u = *reinterpret_cast<const uint2 *>(nr);
                g[0] = __half2float(__ushort_as_half((unsigned short)(u.x & 0xFFFFu)));
                g[1] = __half2float(__ushort_as_half((unsigned short)(u.x >> 16)));
                g[2] = __half2float(__ushort_as_half((unsigned short)(u.y & 0xFFFFu)));
                g[3] = __half2float(__ushort_as_half((unsigned short)(u.y >> 16)));
            } else {
                const uint32_t u = *reinterpret_cast<const uint32_t *>(nr);
                g[0] = __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu)));
                g[1] = __half2float(__ushort_as_half((unsigned short)(u >> 16)));
            }
            float smax = 0.0f;
#pragma unroll
            for (int i = 0; i < NB; ++i) smax = fmaxf(smax, g[i]);
            const float inv = smax > 0.0f ? 1.0f / smax : 0.0f;
            if (blk == 0) {
                scale[(k & 3) * kStRows + r] = smax;
                tc::mbar_arrive(sfull + 8u * (uint32_t)(k & 3));
            }
            uint32_t w[KB + 1];
            const unsigned char * cw = cs + (r * KW + blk * KB) * 4;
            if constexpr (KB == 4) {
                const uint4 u = *reinterpret_cast<const uint4 *>(cw);
                w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
            } else if constexpr (KB == 2) {
                const uint2 u = *reinterpret_cast<const uint2 *>(cw);
                w[0] = u.x; w[1] = u.y;
            } else {
#pragma unroll
                for (int i = 0; i < KB; ++i) w[i] = reinterpret_cast<const uint32_t *>(cw)[i];
            }
            w[KB] = 0u;
            unsigned char * bt = high + C::HIGH_B + b * C::B_BYTES;
            {
                constexpr int bl = 0;
                const float rt = gb_ * inv;
                const __half2 ratio = __floats2half2_rn(rt, rt);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {             // 8 coordinates = one 16-byte chunk
                    uint32_t o[4];
#pragma unroll
                    for (int p4 = 0; p4 < 4; ++p4) {
                        const int p = 4 * c4 + p4;           // coordinates 2 p, 2 p + 1 of the block
                        const int bit = 32 * KB * bl + 2 * KB * p, wi = bit >> 5, sh = bit & 31;
                        uint32_t addr;
                        if constexpr (KB == 4) {
                            // the pair's byte into byte 1 of the window address
                            addr = __byte_perm(w[wi], lane_off, 0x7604u | ((uint32_t)(sh >> 3) << 4));
                        } else {
                            const uint32_t x = sh >= 8 ? __funnelshift_r(w[wi], w[wi + 1], sh - 8)
                                                       : w[wi] << (8 - sh);
                            addr = (x & ((uint32_t)(NK - 1) << 8)) | lane_off;
                        }
                        const uint32_t pr = lds32_table(addr);
                        const __half2 hv = __hmul2(*reinterpret_cast<const __half2 *>(&pr), ratio);
                        o[p4] = *reinterpret_cast<const uint32_t *>(&hv);
                    }
                    const int c = blk * 4 + c4;              // 16-byte chunk of the row
                    *reinterpret_cast<uint4 *>(bt + (c >> 3) * C::SLICE + r * 128 + 16 * ((c & 7) ^ (r & 7))) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            tc::fence_proxy_async();
            __syncwarp();
            // this warp's rows of B[b] are written and its reads of the stage done
            if (lane == 0) {
                tc::mbar_arrive(bfull + 8u * b);
                tc::mbar_arrive(empty + 8u * (uint32_t)(k % kStStages));
            }
        }
    } else {
        // ---- scan warps: TMEM lane m, query q0 + m % NQA, columns
        // [WID sl, WID sl + WID) of every tile, sl = 2 (m / NQA) + half ----
        const int m = stid & (kStRows - 1);
        const int qm = m % NQA;
        const int sl = 2 * (m / NQA) + (stid >> 7);
        const bool scanning = qm < nq;
        uint32_t * gb = bound + q0 + (scanning ? qm : 0);
        unsigned char * lst = high + 256 * stid + 128;
        auto slot = [&](int i) -> uint64_t * { return reinterpret_cast<uint64_t *>(lst + 8 * ((i + stid) & 15)); };
        uint64_t own = 0ull;                 // the list's k-th key (0 until it holds k)
        float own_s = CUDART_NAN_F;          // its score (NaN lets every score through)
        int len = 0;                         // keys in the list
        uint32_t published = 0u;
        // kStScratch bytes of scratch after the high ring stages
        float * scratch = reinterpret_cast<float *>(high + C::HIGH_FIXED + (kStStages - n_low) * C::STAGE +
                                                    kStScratch * stid);
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        uint32_t g_ord = 0u;
        for (int k = 0; k < n_my; ++k) {
            const int b = k & 1;
            // the shared bound, every 16 tiles (all SMs read and raise the
            // same few lines of L2)
            if (!SAMPLE && scanning && (k & 15) == 0) g_ord = ld_relaxed_u32(gb);
            const bool done = tc::mbar_wait(accfull + 8u * b, (uint32_t)((k >> 1) & 1), kStWaitNs) &&
                              tc::mbar_wait(sfull + 8u * (uint32_t)(k & 3), (uint32_t)((k >> 2) & 1), kStWaitNs) &&
                              *s_err == 0;
            if (!__all_sync(0xffffffffu, done)) {
                *s_err = 1;
                break;
            }
            tc::fence_after_sync();
            const int64_t rb = ((int64_t)tile0 + blockIdx.x + (int64_t)k * gridDim.x) * kStRows + WID * sl;
            const float * sc = scale + (k & 3) * kStRows + WID * sl;
            const float thr_g = topk_score((uint64_t)g_ord << 32);
            // 32 columns at a time: scores into registers, the accumulator
            // released after the last
#pragma unroll 1
            for (int c0 = 0; c0 < WID; c0 += 32) {
                float v[32];
                tc::tmem_ld32(tl + (uint32_t)(b * kStRows + WID * sl + c0), v);
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 s4 = *reinterpret_cast<const float4 *>(sc + c0 + j);
                    v[j] *= s4.x;
                    v[j + 1] *= s4.y;
                    v[j + 2] *= s4.z;
                    v[j + 3] *= s4.w;
                }
                if (c0 + 32 >= WID) {
                    tc::fence_before_sync();
                    tc::mbar_arrive(accfree + 8u * b);
                }
                if (!scanning) continue;
                const int nv = (int)min((int64_t)32, n_db - (rb + c0));
                if constexpr (SAMPLE) {
                    float cm = -CUDART_INF_F;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nv) cm = fmaxf(cm, v[j]);
                    if (nv > 0) own = max(own, topk_key(cm, (uint32_t)(rb + c0)));
                    continue;
                }
                float thr = fmaxf(own_s, thr_g);
                // maxima of the four 8-column groups (fmaxf drops NaN
                // scores: a number as threshold means k numeric keys at or
                // above it exist, and a NaN key ranks below every number)
                float gm[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float m8 = v[8 * g];
#pragma unroll
                    for (int j = 1; j < 8; ++j) m8 = fmaxf(m8, v[8 * g + j]);
                    gm[g] = m8;
                }
                const float mx = fmaxf(fmaxf(gm[0], gm[1]), fmaxf(gm[2], gm[3]));
                if (mx < thr) continue;
                // a group that reaches the threshold: its scores through the
                // thread's scratch into one insertion loop
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    if (gm[g] < thr) continue;
                    reinterpret_cast<float4 *>(scratch)[0] = make_float4(v[8 * g], v[8 * g + 1], v[8 * g + 2], v[8 * g + 3]);
                    reinterpret_cast<float4 *>(scratch)[1] = make_float4(v[8 * g + 4], v[8 * g + 5], v[8 * g + 6], v[8 * g + 7]);
#pragma unroll 1
                    for (int j = 0; j < 8; ++j) {
                        const float sj = scratch[j];
                        if (8 * g + j >= nv || sj < thr) continue;
                        const uint64_t key = topk_key(sj, (uint32_t)(rb + c0 + 8 * g + j));
                        if (key <= own) continue;
                        // descending insertion; an unfilled list starts at its first empty slot
                        int i = min(len, topk - 1);
                        while (i > 0) {
                            const uint64_t prev = *slot(i - 1);
                            if (!(prev < key)) break;
                            *slot(i) = prev;
                            --i;
                        }
                        *slot(i) = key;
                        if (len < topk) ++len;
                        if (len == topk) {
                            own = *slot(topk - 1);
                            own_s = topk_score(own);
                            thr = fmaxf(own_s, thr_g);
                        }
                    }
                }
                const uint32_t o = (uint32_t)(own >> 32);
                if (own != 0ull && o > published) {
                    published = o;
                    atomicMax(gb, o);
                }
            }
        }
        if constexpr (SAMPLE) {
            if (scanning) *slot(0) = own;    // (the other slots stay zero)
        }
    }
    __syncthreads();
    const bool ok = *s_err == 0 && lut_ok;
    const int issued = *reinterpret_cast<const int *>(smem + C::OFF_ISSUED);
    if (!ok && tid == 0 && issued > 0) {
        // let the last MMAs finish before the columns are freed
        const int kl = issued - 1;
        tc::mbar_wait(accfull + 8u * (uint32_t)(kl & 1), (uint32_t)((kl >> 1) & 1), kStWaitNs);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
    if (!deq && !issuer_warp && stid < kStRows) {
        const int m = stid;
        const int qm = m % NQA;
        if (qm < nq) {
            // the other half's list (scan thread stid + 128, same TMEM lane)
            // merged into this one: both descending, so stop at the first key
            // that is zero or does not beat this list's k-th
            unsigned char * lst = high + 256 * stid + 128;
            const unsigned char * oth = high + 256 * (stid + kStRows) + 128;
            auto mine = [&](int i) -> uint64_t * { return reinterpret_cast<uint64_t *>(lst + 8 * ((i + stid) & 15)); };
            for (int j = 0; j < topk; ++j) {
                const uint64_t key = *reinterpret_cast<const uint64_t *>(oth + 8 * ((j + stid + kStRows) & 15));
                if (key == 0ull || key <= *mine(topk - 1)) break;
                int i = topk - 1;
                while (i > 0 && *mine(i - 1) < key) {
                    *mine(i) = *mine(i - 1);
                    --i;
                }
                *mine(i) = key;
            }
            // this lane's candidates: list list0 + REP x + m / NQA of the query,
            // cand_keys[(q * lists_stride + list) * topk + i]
            uint64_t * dst = cand_keys + ((int64_t)(q0 + qm) * lists_stride + list0 + (int64_t)blockIdx.x * REP + m / NQA) * topk;
            for (int i = 0; i < topk; ++i) dst[i] = ok ? *mine(i) : 0ull;
        }
    }
}

// The k largest of every query's candidate lists (its lists list0 ..
// list0 + n_lists - 1 of lists_stride lists of k keys, each sorted descending,
// k <= kStMaxK), one CTA per query; bound[q] is a score that k keys reach, so
// lists whose first key is below it are skipped.  The query's keys are staged
// in shared memory; warp w keeps the top 16 of the lists w, w + 8,
// ... in lanes 0-15 (descending) and merges a list only if its first key beats
// the warp's current k-th key (a bitonic merge over shuffles: the list,
// reversed, in lanes 16-31).  Warp 0 then merges the eight warps' results.
constexpr int kSelThreads = 256;

__device__ __forceinline__ uint64_t warp_merge16(uint64_t cur, const uint64_t * list, int n, int lane) {
    uint64_t x = cur;
    if (lane >= 16) x = 31 - lane < n ? list[31 - lane] : 0ull;
#pragma unroll
    for (int st = 16; st > 0; st >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, x, st);
        x = (lane & st) == 0 ? (x > y ? x : y) : (x < y ? x : y);
    }
    return x;
}

// The k-th largest of the first keys of n_lists lists of k keys at L (0 while
// fewer than k are nonzero), for the whole block: every warp sorts 32 keys at
// a time across its lanes and merges their top 16 into its own; warp 0 merges
// the warps' results.
__device__ uint64_t kth_of_heads(const uint64_t * L, int n_lists, int k, uint64_t (*res)[16]) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t cur = 0ull;
    for (int base = 32 * warp; base < n_lists; base += kSelThreads) {
        const int j = base + lane;
        uint64_t x = j < n_lists ? L[(int64_t)j * k] : 0ull;
        // bitonic sort across the lanes, descending
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
            for (int st = size >> 1; st > 0; st >>= 1) {
                const uint64_t y = __shfl_xor_sync(0xffffffffu, x, st);
                const bool desc = (lane & size) == 0, lower = (lane & st) == 0;
                x = lower == desc ? (x > y ? x : y) : (x < y ? x : y);
            }
        }
        // the top 16, reversed into lanes 16-31, merged with the warp's own
        const uint64_t rev = __shfl_sync(0xffffffffu, x, 31 - lane);
        uint64_t z = lane < 16 ? cur : rev;
#pragma unroll
        for (int st = 16; st > 0; st >>= 1) {
            const uint64_t y = __shfl_xor_sync(0xffffffffu, z, st);
            z = (lane & st) == 0 ? (z > y ? z : y) : (z < y ? z : y);
        }
        cur = z;
    }
    if (lane < 16) res[warp][lane] = cur;
    __syncthreads();
    if (warp == 0) {
        cur = lane < 16 ? res[0][lane] : 0ull;
        for (int w = 1; w < kSelThreads / 32; ++w) cur = warp_merge16(cur, res[w], 16, lane);
        const uint64_t kth = __shfl_sync(0xffffffffu, cur, k - 1);
        if (lane == 0) res[0][0] = kth;
    }
    __syncthreads();
    const uint64_t kth = res[0][0];
    __syncthreads();
    return kth;
}

__global__ void __launch_bounds__(kSelThreads)
topk_lists_kernel(const uint64_t * __restrict__ cand, int32_t list0, int32_t n_lists, int32_t lists_stride, int32_t k,
                  const uint32_t * __restrict__ bound, float * __restrict__ top_scores,
                  int32_t * __restrict__ top_rows) {
    extern __shared__ __align__(16) unsigned char sel_smem[];
    uint64_t * sk = reinterpret_cast<uint64_t *>(sel_smem);
    __shared__ uint64_t res[kSelThreads / 32][16];
    pdl_launch_dependents();             // the main pass may start its prologue
    const int q = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_keys = n_lists * k;
    const uint64_t * L = cand + ((int64_t)q * lists_stride + list0) * k;
    for (int i0 = 0; i0 < n_keys; i0 += 8 * kSelThreads) {   // eight loads in flight per thread
        uint64_t t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            t[u] = i < n_keys ? L[i] : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            if (i < n_keys) sk[i] = t[u];
        }
    }
    __syncthreads();
    // k keys of score >= bound[q] exist, and k list heads >= the k-th largest
    // head: lists whose first key is below either can be skipped
    const uint32_t b0 = bound[q];
    const uint64_t hk = kth_of_heads(sk, n_lists, k, res);
    const uint64_t thr0 = max(b0 != 0u ? ((uint64_t)b0 << 32) - 1ull : 0ull, hk != 0ull ? hk - 1ull : 0ull);
    uint64_t cur = 0ull, thr = thr0;
    for (int base = 32 * warp; base < n_lists; base += kSelThreads) {
        const int j = base + lane;
        const uint64_t top = j < n_lists ? sk[j * k] : 0ull;
        unsigned want = __ballot_sync(0xffffffffu, top > thr);
        while (want) {
            const int src = __ffs(want) - 1;
            want &= want - 1;
            if (__shfl_sync(0xffffffffu, top, src) <= thr) continue;
            cur = warp_merge16(cur, sk + (base + src) * k, k, lane);
            thr = max(thr0, __shfl_sync(0xffffffffu, cur, k - 1));
        }
    }
    if (lane < 16) res[warp][lane] = cur;
    __syncthreads();
    if (warp == 0) {
        cur = lane < 16 ? res[0][lane] : 0ull;
        for (int w = 1; w < kSelThreads / 32; ++w) cur = warp_merge16(cur, res[w], 16, lane);
        if (lane < k) {
            top_scores[(int64_t)q * k + lane] = topk_score(cur);
            top_rows[(int64_t)q * k + lane] = topk_row(cur);
        }
    }
}

// The shared bound after the sample pass: bound[q] = the ordered score of the
// k-th largest of the query's sample keys (the first key of each of its
// n_lists lists).
__global__ void __launch_bounds__(kSelThreads)
topk_bound_kernel(const uint64_t * __restrict__ cand, int32_t n_lists, int32_t lists_stride, int32_t k,
                  uint32_t * __restrict__ bound) {
    pdl_launch_dependents();             // the main pass may start its prologue
    __shared__ uint64_t res[kSelThreads / 32][16];
    const uint64_t kth = kth_of_heads(cand + (int64_t)blockIdx.x * lists_stride * k, n_lists, k, res);
    if (threadIdx.x == 0) bound[blockIdx.x] = (uint32_t)(kth >> 32);
}

// One pass of the top-k reduction: CTA (c, q) sorts chunk c (kTopkChunk keys,
// descending) of query q's input and keeps its first k.  The first pass reads
// the score matrix (row j of query q = scores[q * n_in + j]); later passes
// read the previous pass's keys.  The last pass writes scores and rows.
__global__ void __launch_bounds__(kTopkThreads)
topk_pass_kernel(const float * __restrict__ scores, const uint64_t * __restrict__ keys_in,
                 int64_t n_in, int32_t k, uint64_t * __restrict__ keys_out,
                 float * __restrict__ top_scores, int32_t * __restrict__ top_rows) {
    __shared__ uint64_t sk[kTopkChunk];
    const int64_t q = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * kTopkChunk;
    for (int i = threadIdx.x; i < kTopkChunk; i += blockDim.x) {
        const int64_t j = c0 + i;
        uint64_t key = 0ull;
        if (j < n_in)
            key = scores != nullptr ? topk_key(scores[q * n_in + j], (uint32_t)j) : keys_in[q * n_in + j];
        sk[i] = key;
    }
    __syncthreads();
    // bitonic sort, descending
    for (int size = 2; size <= kTopkChunk; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < kTopkChunk / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t x = sk[lo], y = sk[hi];
                if ((x < y) == desc) {
                    sk[lo] = y;
                    sk[hi] = x;
                }
            }
            __syncthreads();
        }
    }
    const int64_t n_chunks = gridDim.x;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        if (top_scores != nullptr) {
            top_scores[q * k + i] = topk_score(sk[i]);
            top_rows[q * k + i] = topk_row(sk[i]);
        } else {
            keys_out[(q * n_chunks + blockIdx.x) * k + i] = sk[i];
        }
    }
}

// CTAs along the database for each query group: about one CTA per SM over
// all groups, and every warp owns at least one slab.
int64_t search_ctas_x(int64_t n_db, int n_groups) {
    const int64_t slabs = (n_db + kSlab - 1) / kSlab;
    // (one CTA fits an SM: a rounded-up count would leave a second wave of a few CTAs)
    int64_t gx = device_sm_count() / n_groups;
    gx = std::min<int64_t>(gx, (slabs + kSearchWarps - 1) / kSearchWarps);
    return std::max<int64_t>(gx, 1);
}

template <int D, int KB>
int launch_search_scores_t(const AttnArgs & a, const CodebookParams & kcb, int n_groups,
                           int32_t topk, uint64_t * cand, cudaStream_t st) {
    using S = SearchCfg<D, KB>;
    int dev = 0;
    cudaGetDevice(&dev);
    int reserved = 0;
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (reserved < 0 || reserved > 65536) return (int)cudaErrorInvalidConfiguration;
    AttnArgs b = a;
    b.mma_lut_off = 65536 - reserved;
    b.mma_ring_a = std::min(kSearchWarps, b.mma_lut_off / S::RING);
    const bool fused = cand != nullptr;
    const int list_bytes = fused ? kSearchWarps * kSearchQ * 32 * 8 : 0;
    const int smem = b.mma_lut_off + kLutBytes + (kSearchWarps - b.mma_ring_a) * S::RING + list_bytes;
    const int64_t gx = search_ctas_x(a.ctx, n_groups);
    const dim3 grid((unsigned)gx, (unsigned)n_groups);
    if (fused) {
        auto k = search_scores_kernel<D, KB, true>;
        if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return e;
        k<<<grid, 32 * kSearchWarps, smem, st>>>(b, kcb, topk, cand);
    } else {
        auto k = search_scores_kernel<D, KB, false>;
        if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return e;
        k<<<grid, 32 * kSearchWarps, smem, st>>>(b, kcb, topk, nullptr);
    }
    return (int)cudaGetLastError();
}

template <int D>
int launch_search_t(const AttnArgs & a, const CodebookParams & kcb, const RotParams & rp,
                    int n_groups, int32_t topk, uint64_t * cand, cudaStream_t st) {
    search_prep_kernel<D><<<(unsigned)n_groups, kThreads, 0, st>>>(a, rp);
    if (int e = (int)cudaGetLastError()) return e;
    switch (a.k_bits) {
        case 2: return launch_search_scores_t<D, 2>(a, kcb, n_groups, topk, cand, st);
        case 3: return launch_search_scores_t<D, 3>(a, kcb, n_groups, topk, cand, st);
        case 4: return launch_search_scores_t<D, 4>(a, kcb, n_groups, topk, cand, st);
    }
    return (int)cudaErrorInvalidValue;
}

// Tensor-core search geometry: d = 64 / 128 with k <= kStMaxK; up to 64
// queries are held twice in the query operand (REP = 2).
bool search_tc_path(int32_t head_dim, int32_t k) {
    return (head_dim == 64 || head_dim == 128) && k <= kStMaxK;
}
int search_tc_rep(int32_t n_queries) { return n_queries <= kStQ / 2 ? 2 : 1; }
int search_tc_groups(int32_t n_queries) {
    const int nqa = kStQ / search_tc_rep(n_queries);
    return (n_queries + nqa - 1) / nqa;
}
// CTAs along the database per query group: about one per SM over all groups.
int64_t search_tc_ctas_x(int64_t n_db, int n_groups) {
    const int64_t tiles = (n_db + kStRows - 1) / kStRows;
    return std::max<int64_t>(1, std::min<int64_t>(device_sm_count() / n_groups, tiles));
}
// Candidate lists per query: one (REP = 1) or two (REP = 2) per CTA in each
// of the two passes (the sample pass's column maxima, the main pass's lists;
// a CTA merges the two halves of a TMEM lane into one list).
int64_t search_tc_lists(int32_t n_queries, int64_t n_db) {
    return 2 * search_tc_ctas_x(n_db, search_tc_groups(n_queries)) * search_tc_rep(n_queries);
}

template <int D, int KB>
int launch_search_tc_kb(const AttnArgs & a, const CodebookParams & kcb, int32_t topk,
                        const __half * qrows, uint32_t * bound, uint64_t * cand,
                        float * top_scores, int32_t * top_rows, cudaStream_t st) {
    using C = StCfg<D, KB>;
    int dev = 0;
    cudaGetDevice(&dev);
    int reserved = 0, optin = 0;
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (reserved < 0 || reserved > 65536 - C::LOW_FIXED) return (int)cudaErrorInvalidConfiguration;
    AttnArgs b = a;
    b.mma_lut_off = 65536 - reserved;
    const int n_low = std::min(kStStages, (b.mma_lut_off - C::LOW_FIXED) / C::STAGE);
    const int smem = b.mma_lut_off + C::HIGH_FIXED + (kStStages - n_low) * C::STAGE + kStScanThreads * kStScratch;
    if (smem > optin) return (int)cudaErrorInvalidConfiguration;
    const int rep = search_tc_rep(a.n_q_heads);
    const int n_groups = search_tc_groups(a.n_q_heads);
    const int64_t gx = search_tc_ctas_x(a.ctx, n_groups);
    const int n_tiles = (int)((a.ctx + kStRows - 1) / kStRows);
    const int split = (int)std::min<int64_t>(n_tiles, gx * kStSampleTiles);
    const int per_pass = (int)gx * rep;
    const int stride = 2 * per_pass;
    const int sel_smem = per_pass * topk * (int)sizeof(uint64_t);
    if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(topk_lists_kernel), sel_smem)) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)n_groups);
    cfg.blockDim = dim3(st_threads(D));
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto sample = rep == 2 ? search_tc_kernel<D, KB, 2, true> : search_tc_kernel<D, KB, 1, true>;
    auto kern = rep == 2 ? search_tc_kernel<D, KB, 2, false> : search_tc_kernel<D, KB, 1, false>;
    if (int r = ensure_dynamic_smem(reinterpret_cast<const void *>(sample), smem)) return r;
    if (int r = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), smem)) return r;
    // sample pass over the first kStSampleTiles tiles of every CTA: the k-th
    // largest of its column maxima is a score that k rows reach, the bound
    // the main pass starts from
    cudaError_t e = cudaLaunchKernelEx(&cfg, sample, b, kcb, qrows, bound, topk, (int32_t)n_low, (int32_t)0,
                                       (int32_t)split, (int32_t)stride, (int32_t)0, cand);
    if (e != cudaSuccess) return (int)e;
    topk_bound_kernel<<<(unsigned)a.n_q_heads, kSelThreads, 0, st>>>(cand, per_pass, stride, topk, bound);
    if (int r = (int)cudaGetLastError()) return r;
    // main pass over every tile, then the k best of its lists
    e = cudaLaunchKernelEx(&cfg, kern, b, kcb, qrows, bound, topk, (int32_t)n_low, (int32_t)0,
                           (int32_t)n_tiles, (int32_t)stride, (int32_t)per_pass, cand);
    if (e != cudaSuccess) return (int)e;
    topk_lists_kernel<<<(unsigned)a.n_q_heads, kSelThreads, sel_smem, st>>>(
        cand, per_pass, per_pass, stride, topk, bound, top_scores, top_rows);
    return (int)cudaGetLastError();
}

// Query rows, the tensor-core scores with per-thread lists, and the selection
// of every query's k best from its lists.
template <int D>
int launch_search_tc_t(const AttnArgs & a, const CodebookParams & kcb, const RotParams & rp,
                       int32_t topk, __half * qrows, uint32_t * bound, uint64_t * cand,
                       float * top_scores, int32_t * top_rows, cudaStream_t st) {
    search_qrows_kernel<D><<<(unsigned)a.n_q_heads, kThreads, 0, st>>>(a, rp, qrows, bound);
    if (int e = (int)cudaGetLastError()) return e;
    switch (a.k_bits) {
        case 2: return launch_search_tc_kb<D, 2>(a, kcb, topk, qrows, bound, cand, top_scores, top_rows, st);
        case 3: return launch_search_tc_kb<D, 3>(a, kcb, topk, qrows, bound, cand, top_scores, top_rows, st);
        case 4: return launch_search_tc_kb<D, 4>(a, kcb, topk, qrows, bound, cand, top_scores, top_rows, st);
    }
    return (int)cudaErrorInvalidValue;
}

}  // namespace

int launch_logits(const tq_rotation * rot, const CodebookParams & kcb, const AttnArgs & a,
                  void * stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RotParams rp = rot_params(rot);
    {
        // tensor-core path: d = 64/128, at most 128 QJL rows, every (batch, kv
        // head) section of codes, norms, signs and residual norms 16-byte aligned
        const int d = a.head_dim, nb = d / 32;
        const bool qjl = a.qjl_signs != nullptr;
        bool ok = (d == 64 || d == 128) && a.ctx >= 1 && (!qjl || a.qjl_m <= kLgMaxM) &&
                  a.norm_block == 32 && !a.norm_f32;
        const int64_t secs[4] = {(int64_t)nb * a.k_bits * 4, (int64_t)nb * 2,
                                 qjl ? (int64_t)a.qjl_m / 8 : 0, qjl ? 2 : 0};
        for (int i = 0; i < 4 && ok; ++i) ok = (a.ctx * secs[i]) % 16 == 0;
        const int64_t G = a.n_q_heads / a.n_kv_heads;
        const int64_t groups = (G + kQH - 1) / kQH;
        const int64_t n_bhg = (int64_t)a.batch * a.n_kv_heads * groups;
        ok = ok && (int64_t)a.batch * a.n_kv_heads * (a.ctx + kSlab) <= (int64_t)INT32_MAX &&
             n_bhg <= (int64_t)INT32_MAX;
        if (ok) {
            AttnArgs b = a;
            b.mma_groups = (int32_t)groups;
            b.mma_spb = (a.ctx + kSlab - 1) / kSlab;
            b.mma_slabs = n_bhg * b.mma_spb;
            // a CTA's range spans at most 2 spb slabs, so it meets at most 3 groups
            int64_t ctas = std::max<int64_t>(device_sm_count(), (b.mma_slabs + 2 * b.mma_spb - 1) / (2 * b.mma_spb));
            ctas = std::min<int64_t>(ctas, (b.mma_slabs + kLgWarps - 1) / kLgWarps);
            ctas = std::max<int64_t>(ctas, (b.mma_slabs + 2 * b.mma_spb - 1) / (2 * b.mma_spb));
            if (ctas <= (int64_t)INT32_MAX) {
                switch (d * 10 + a.k_bits) {
                    case 642: return launch_logits_mma_t<64, 2>(b, kcb, rp, ctas, st);
                    case 643: return launch_logits_mma_t<64, 3>(b, kcb, rp, ctas, st);
                    case 644: return launch_logits_mma_t<64, 4>(b, kcb, rp, ctas, st);
                    case 1282: return launch_logits_mma_t<128, 2>(b, kcb, rp, ctas, st);
                    case 1283: return launch_logits_mma_t<128, 3>(b, kcb, rp, ctas, st);
                    case 1284: return launch_logits_mma_t<128, 4>(b, kcb, rp, ctas, st);
                }
            }
        }
    }
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
                  const CodebookParams & vcb, const AttnArgs & a, void * stream,
                  const AppendParams * ap_in) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RotParams rp = rot_params(rot);
    AppendParams ap{};
    if (ap_in != nullptr) ap = *ap_in;
    if (ap.enabled && !a.mma_mode) return (int)cudaErrorInvalidValue;
    if (a.mma_mode) {
        int err;
        switch (a.head_dim) {
            case 64: err = launch_mma_decode<64>(a, kcb, vcb, rp, ap, st); break;
            case 128: err = launch_mma_decode<128>(a, kcb, vcb, rp, ap, st); break;
            case 256: err = launch_mma_decode<256>(a, kcb, vcb, rp, ap, st); break;
            default: return (int)cudaErrorInvalidValue;
        }
        if (err) return err;
        return launch_combine(a, rp, st, true);
    }
    if (a.qjl_signs == nullptr && a.norm_block == 32 && !a.norm_f32 && !a.v_grouped) {
        int err;
        switch (a.head_dim) {
            case 64: err = fast_kb<64>(a, kcb, vcb, rp, st); break;
            case 128: err = fast_kb<128>(a, kcb, vcb, rp, st); break;
            case 256: err = fast_kb<256>(a, kcb, vcb, rp, st); break;
            default: return (int)cudaErrorInvalidValue;
        }
        if (err) return err;
        return launch_combine(a, rp, st, false);
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
    return launch_combine(a, rp, st, false);
}

size_t decode_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t n_splits,
                              int32_t head_dim) {
    const size_t parts = (size_t)batch * n_q_heads * n_splits;
    return parts * ((size_t)head_dim + 2) * sizeof(float);
}

size_t qrot_workspace_bytes(int32_t, int32_t, int32_t, int32_t) { return 0; }

MmaDecodePlan plan_mma_decode(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int64_t ctx,
                              int32_t head_dim, int32_t k_bits, int32_t v_bits, int32_t qjl_m,
                              bool paged) {
    MmaDecodePlan p{};
    p.ok = false;
    if (batch < 1 || n_kv_heads < 1 || ctx < 1) return p;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return p;
    if (k_bits < 2 || k_bits > 4 || v_bits < 2 || v_bits > 4) return p;
    // QJL keys: d = 64 / 128 and at most kMmaMaxM projection rows
    if (qjl_m != 0 && (head_dim > 128 || qjl_m < 16 || qjl_m > kMmaMaxM || qjl_m % 32 != 0)) return p;
    const int nb = head_dim / 32;
    // every (batch, kv head) section of codes, norms, sign words and residual
    // norms must start on a 16-byte boundary for the 16-byte copies
    const int64_t rows_bytes[5] = {(int64_t)nb * k_bits * 4, (int64_t)nb * 2, (int64_t)nb * v_bits * 4,
                                   (int64_t)qjl_m / 8, qjl_m ? 2 : 0};
    // (a paged cache's slabs start on 16-row boundaries of their page)
    for (int i = 0; i < 5 && !paged; ++i)
        if ((ctx * rows_bytes[i]) % 16 != 0) return p;
    const int64_t G = n_q_heads / n_kv_heads;
    p.groups = (int32_t)((G + kQH - 1) / kQH);
    // the kernel's cursors hold rows, tokens and groups in 32 bits
    if ((int64_t)batch * n_kv_heads * (ctx + kSlab) > (int64_t)INT32_MAX ||
        (int64_t)batch * n_kv_heads * p.groups > (int64_t)INT32_MAX)
        return p;
    p.spb = (ctx + kSlab - 1) / kSlab;
    const int64_t n_bhg = (int64_t)batch * n_kv_heads * p.groups;
    p.slabs = n_bhg * p.spb;
    p.warps_per_cta = qjl_m ? MmaCfg<128, true>::WPC
                            : (head_dim <= 128 ? MmaCfg<128, false>::WPC : MmaCfg<256, false>::WPC);
    const int64_t want = (p.slabs + p.warps_per_cta - 1) / p.warps_per_cta;
    p.ctas = (int32_t)std::min<int64_t>(device_sm_count(), want);
    // no more warps than slabs, so every warp owns at least one slab and the
    // slots of a group are exactly the warps from its first to its last
    const int64_t W = std::min<int64_t>((int64_t)p.ctas * p.warps_per_cta, p.slabs);
    p.warps = (int32_t)W;
    int64_t slots = 1;
    for (int64_t bhg = 0; bhg < n_bhg; ++bhg) {
        const int64_t n = warp_of_slab((bhg + 1) * p.spb - 1, p.slabs, W) -
                          warp_of_slab(bhg * p.spb, p.slabs, W) + 1;
        slots = std::max(slots, n);
    }
    p.slots = (int32_t)slots;
    const bool q = qjl_m != 0;
    p.smem_bytes = head_dim == 64    ? mma_smem_bytes<64>(k_bits, v_bits, q)
                   : head_dim == 128 ? mma_smem_bytes<128>(k_bits, v_bits, q)
                                     : mma_smem_bytes<256>(k_bits, v_bits, q);
    p.partial_bytes = decode_workspace_bytes(batch, n_q_heads, p.slots, head_dim);
    p.partial_bytes = (p.partial_bytes + 255) / 256 * 256;
    // per lane: NB * 4 query words (+ the QJL fragment words); a multiple of 4
    // so that the lane's words load as 16-byte vectors
    p.qfrag_words = nb * 4 + (q ? (kMmaMaxM / 16) * 2 : 0);
    p.qfrag_bytes = (size_t)n_bhg * 32 * p.qfrag_words * sizeof(uint32_t);
    p.ok = true;
    return p;
}

int search_groups(int32_t n_queries) { return (n_queries + kSearchQ - 1) / kSearchQ; }

// Workspace: [scores (k > kSearchHeapK) or the candidate keys][query
// fragments, or the fp16 query rows of the tensor-core search][the shared
// per-query bounds of the tensor-core search][two key buffers of the top-k
// passes].
struct SearchLayout {
    size_t first, qfrag, bound, keys;
};
SearchLayout search_layout(int32_t n_queries, int64_t n_db, int32_t head_dim, int32_t k) {
    SearchLayout l{};
    const int n_groups = search_groups(n_queries);
    l.qfrag = ((size_t)n_groups * 32 * (head_dim / 32) * 4 * sizeof(uint32_t) + 255) / 256 * 256;
    if (search_tc_path(head_dim, k)) {
        const int64_t n_in = search_tc_lists(n_queries, n_db) * k;
        l.first = ((size_t)n_queries * (size_t)n_in * sizeof(uint64_t) + 255) / 256 * 256;
        l.bound = ((size_t)n_queries * sizeof(uint32_t) + 255) / 256 * 256;
        return l;
    }
    int64_t n_in = n_db;
    if (k <= kSearchHeapK) {
        const int64_t w = search_ctas_x(n_db, n_groups) * kSearchWarps;
        n_in = w * k;
        l.first = ((size_t)n_queries * (size_t)n_in * sizeof(uint64_t) + 255) / 256 * 256;
    } else {
        l.first = ((size_t)n_queries * (size_t)n_db * sizeof(float) + 255) / 256 * 256;
    }
    const size_t chunks = (size_t)((n_in + kTopkChunk - 1) / kTopkChunk);
    l.keys = ((size_t)n_queries * chunks * (size_t)k * sizeof(uint64_t) + 255) / 256 * 256;
    return l;
}

size_t search_workspace_bytes(int32_t n_queries, int64_t n_db, int32_t head_dim, int32_t k) {
    const SearchLayout l = search_layout(n_queries, n_db, head_dim, k);
    return l.first + l.qfrag + l.bound + 2 * l.keys;
}

int launch_search(const tq_rotation * rot, const CodebookParams & kcb, const AttnArgs & a_in,
                  int32_t k, float * top_scores, int32_t * top_rows, void * stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RotParams rp = rot_params(rot);
    const int32_t nq = a_in.n_q_heads;
    const int64_t n_db = a_in.ctx;
    const int d = a_in.head_dim;
    const int n_groups = search_groups(nq);
    unsigned char * ws = static_cast<unsigned char *>(a_in.workspace);
    const SearchLayout l = search_layout(nq, n_db, d, k);
    if (search_tc_path(d, k)) {
        uint64_t * cand = reinterpret_cast<uint64_t *>(ws);
        __half * qrows = reinterpret_cast<__half *>(ws + l.first);
        uint32_t * bound = reinterpret_cast<uint32_t *>(ws + l.first + l.qfrag);
        if (d == 64) return launch_search_tc_t<64>(a_in, kcb, rp, k, qrows, bound, cand, top_scores, top_rows, st);
        return launch_search_tc_t<128>(a_in, kcb, rp, k, qrows, bound, cand, top_scores, top_rows, st);
    }
    const bool fused = k <= kSearchHeapK;
    AttnArgs a = a_in;
    a.logits = reinterpret_cast<float *>(ws);
    a.mma_qfrag = reinterpret_cast<uint32_t *>(ws + l.first);
    uint64_t * cand = fused ? reinterpret_cast<uint64_t *>(ws) : nullptr;
    uint64_t * keys[2] = {reinterpret_cast<uint64_t *>(ws + l.first + l.qfrag),
                          reinterpret_cast<uint64_t *>(ws + l.first + l.qfrag + l.keys)};
    int err;
    switch (d) {
        case 64: err = launch_search_t<64>(a, kcb, rp, n_groups, k, cand, st); break;
        case 128: err = launch_search_t<128>(a, kcb, rp, n_groups, k, cand, st); break;
        case 256: err = launch_search_t<256>(a, kcb, rp, n_groups, k, cand, st); break;
        default: return (int)cudaErrorInvalidValue;
    }
    if (err) return err;
    // top-k passes: chunks of kTopkChunk keys -> k keys each, until one chunk
    int64_t n_in = fused ? search_ctas_x(n_db, n_groups) * kSearchWarps * k : n_db;
    const uint64_t * kin = fused ? cand : nullptr;
    int which = 0;
    for (;;) {
        const int64_t n_chunks = (n_in + kTopkChunk - 1) / kTopkChunk;
        const bool last = n_chunks == 1;
        topk_pass_kernel<<<dim3((unsigned)n_chunks, (unsigned)nq), kTopkThreads, 0, st>>>(
            kin == nullptr ? a.logits : nullptr, kin, n_in, k, last ? nullptr : keys[which],
            last ? top_scores : nullptr, last ? top_rows : nullptr);
        if (int e = (int)cudaGetLastError()) return e;
        if (last) break;
        kin = keys[which];
        which ^= 1;
        n_in = n_chunks * k;
    }
    return 0;
}

}  // namespace tq
