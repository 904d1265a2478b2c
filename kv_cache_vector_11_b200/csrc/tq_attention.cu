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
