// KV-cache quantization kernels (sm_100a).
//
// "TurboQuant+ upstream guide", sec. 5.1 / 5.2: rotate each row, take the
// norm of every 32-value block, quantize each normalised coordinate against
// the Lloyd-Max centroid table and pack the indices; sec. 4: the rotation is
// either the structured D1 @ H @ D2 Walsh-Hadamard form or a dense Haar QR
// matrix.
//
// Work decomposition of the Walsh-Hadamard kernel: every lane owns 64
// consecutive rotated coordinates (two norm blocks) of one row, so a row of
// d = 64 / 128 / 256 coordinates is handled by 1 / 2 / 4 lanes with no data
// exchange between them.  The top log2(d / 64) butterfly stages act across
// the 64-wide slices; a lane evaluates them while loading (it reads the whole
// row, which the other lanes of the row read too -- the duplicate reads are
// served by L1), then runs the remaining six stages in registers.  D2 is
// applied as a sign-bit XOR on the loaded words; D1 and the 1/sqrt(d) factor
// never touch the data: codes depend only on the direction of a block (D1
// becomes a mirror of the code, idx -> 2^b - 1 - idx, applied to whole packed
// words) and the stored norm takes the 1/sqrt(d) factor.

#include <cuda_runtime.h>

#include "tq_device.cuh"

namespace tq {

namespace {

struct WhtKernelSigns {
    // bf16 input: word p holds the sign masks of elements 2p (bit 15) and
    // 2p+1 (bit 31); fp32 input: word i holds element i's mask in bit 31.
    uint32_t d2_mask[256];
    uint32_t d1_bits[8];
};

__device__ __forceinline__ void wht64(float * z) {
#pragma unroll
    for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if ((i & h) == 0) {
                const float a = z[i], b = z[i + h];
                z[i] = a + b;
                z[i + h] = a - b;
            }
        }
    }
}

template <int BITS>
__device__ __forceinline__ void place_field(uint32_t * words, int j, uint32_t v) {
    const int p = j * BITS;
    const int wi = p >> 5, sh = p & 31;
    words[wi] |= v << sh;
    if (sh + BITS > 32) words[wi + 1] |= v >> (32 - sh);
}

// Encode one 32-coordinate block y (unnormalised rotated values) into BITS
// packed words.  `mirror` holds, per code field, 2^(b-1) XOR (D1 = -1 ? all
// ones : 0); `g` is the block norm of y.
template <int BITS>
__device__ __forceinline__ void encode_block(const float * y, float g, const CodebookParams & cb,
                                             const uint32_t * mirror, uint32_t * out) {
    constexpr uint32_t FIELD = (1u << BITS) - 1u;
    constexpr int NT = (1 << (BITS - 1)) - 1;
    float T[NT > 0 ? NT : 1];
#pragma unroll
    for (int k = 0; k < NT; ++k) T[k] = g * cb.pos_boundary[k];
    uint32_t acc[BITS], neg[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) { acc[k] = 0u; neg[k] = 0u; }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float v = y[j];
        const uint32_t m = magnitude_rank<BITS>(fabsf(v), T);
        const uint32_t s = (uint32_t)(__float_as_int(v) >> 31) & FIELD;
        place_field<BITS>(acc, j, m);
        place_field<BITS>(neg, j, s);
    }
    if (g > 0.0f) {
#pragma unroll
        for (int k = 0; k < BITS; ++k) out[k] = acc[k] ^ neg[k] ^ mirror[k];
    } else {
        // a zero block stores the middle code 2^(b-1) everywhere
        uint32_t half[BITS];
#pragma unroll
        for (int k = 0; k < BITS; ++k) half[k] = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) place_field<BITS>(half, j, 1u << (BITS - 1));
#pragma unroll
        for (int k = 0; k < BITS; ++k) out[k] = half[k];
    }
}

template <int WORDS>
__device__ __forceinline__ void store_words(uint32_t * dst, const uint32_t * w) {
    if constexpr (WORDS % 4 == 0) {
#pragma unroll
        for (int k = 0; k < WORDS; k += 4)
            *reinterpret_cast<uint4 *>(dst + k) = make_uint4(w[k], w[k + 1], w[k + 2], w[k + 3]);
    } else {
#pragma unroll
        for (int k = 0; k < WORDS; k += 2)
            *reinterpret_cast<uint2 *>(dst + k) = make_uint2(w[k], w[k + 1]);
    }
}

// Norms, codes and stores for the lane's 64 rotated coordinates z of `row`.
template <int D, int BITS>
__device__ __forceinline__ void finish_row(const float * z, int64_t row, int q,
                                           const CodebookParams & cb, const uint32_t * mirror,
                                           float norm_scale, const QuantizeArgs & a,
                                           uint32_t & status) {
    constexpr int NB = D / 32;
    uint32_t words[2 * BITS];
    uint16_t nh[2];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) ss = fmaf(z[32 * bb + j], z[32 * bb + j], ss);
        const float g = sqrtf(ss);
        if (!isfinite(ss)) status |= TQ_STATUS_NONFINITE;
        bool sat;
        nh[bb] = norm_to_half_bits(g * norm_scale, &sat);
        if (sat) status |= TQ_STATUS_NORM_SATURATED;
        encode_block<BITS>(z + 32 * bb, g, cb, mirror + bb * BITS, words + bb * BITS);
    }
    store_words<2 * BITS>(a.codes + row * (NB * BITS) + q * 2 * BITS, words);
    *reinterpret_cast<uint32_t *>(a.norms + row * NB + 2 * q) =
        (uint32_t)nh[0] | ((uint32_t)nh[1] << 16);
}

template <int D, int BITS, bool BF16>
__global__ void __launch_bounds__(256)
quantize_wht_kernel(const QuantizeArgs a, const CodebookParams cb,
                    const __grid_constant__ WhtKernelSigns sg) {
    constexpr int LPR = D / 64;   // lanes per row
    constexpr int RPW = 32 / LPR; // rows per warp step
    constexpr uint32_t FIELD = (1u << BITS) - 1u;
    const int lane = threadIdx.x & 31;
    const int q = lane % LPR;
    const int rsub = lane / LPR;

    // Per-field XOR constant for the lane's two blocks (2q, 2q+1):
    // 2^(b-1) for the sign-magnitude to index step, and all ones where D1 = -1.
    uint32_t mirror[2 * BITS];
#pragma unroll
    for (int k = 0; k < 2 * BITS; ++k) mirror[k] = 0u;
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        const uint32_t d1 = sg.d1_bits[2 * q + bb];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const uint32_t f = (1u << (BITS - 1)) ^ (((d1 >> j) & 1u) ? FIELD : 0u);
            place_field<BITS>(mirror + bb * BITS, j, f);
        }
    }
    // Signs of the slice-level butterflies for this lane: (-1)^popcount(q & a).
    const float s1 = (q & 1) ? -1.0f : 1.0f;
    const float s2 = (q & 2) ? -1.0f : 1.0f;
    const float norm_scale = rsqrtf((float)D);

    uint32_t status = 0u;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r0 = gwarp * RPW; r0 < a.n_rows; r0 += nwarps * RPW) {
        const int64_t row = r0 + rsub;
        if (row >= a.n_rows) continue;
        float z[64];
        if constexpr (BF16) {
            const uint16_t * xr = static_cast<const uint16_t *>(a.x) + row * D;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float v[LPR][8];
#pragma unroll
                for (int s = 0; s < LPR; ++s) {
                    const uint4 u = ldg_nc_v4(xr + s * 64 + c * 8);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t w = w4[k] ^ sg.d2_mask[(s * 64 + c * 8) / 2 + k];
                        v[s][2 * k] = bf16_lo(w);
                        v[s][2 * k + 1] = bf16_hi(w);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if constexpr (LPR == 1) z[c * 8 + e] = v[0][e];
                    else if constexpr (LPR == 2) z[c * 8 + e] = fmaf(s1, v[1][e], v[0][e]);
                    else z[c * 8 + e] = fmaf(s2, fmaf(s1, v[3][e], v[2][e]), fmaf(s1, v[1][e], v[0][e]));
                }
            }
        } else {
            const float * xr = static_cast<const float *>(a.x) + row * D;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                float v[LPR][4];
#pragma unroll
                for (int s = 0; s < LPR; ++s) {
                    const uint4 u = ldg_nc_v4(xr + s * 64 + c * 4);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        v[s][k] = __uint_as_float(w4[k] ^ sg.d2_mask[s * 64 + c * 4 + k]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (LPR == 1) z[c * 4 + e] = v[0][e];
                    else if constexpr (LPR == 2) z[c * 4 + e] = fmaf(s1, v[1][e], v[0][e]);
                    else z[c * 4 + e] = fmaf(s2, fmaf(s1, v[3][e], v[2][e]), fmaf(s1, v[1][e], v[0][e]));
                }
            }
        }
        wht64(z);
        finish_row<D, BITS>(z, row, q, cb, mirror, norm_scale, a, status);
    }
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

// Dense rotation y = P x computed on the CUDA cores from the fp32 matrix in
// global memory (L1/L2 resident); same lane decomposition and epilogue as the
// Walsh-Hadamard kernel.  This is the straightforward form of the dense path.
template <int D, int BITS, bool BF16>
__global__ void __launch_bounds__(256)
quantize_dense_simple_kernel(const QuantizeArgs a, const CodebookParams cb) {
    constexpr int LPR = D / 64;
    constexpr int RPW = 32 / LPR;
    const int lane = threadIdx.x & 31;
    const int q = lane % LPR;
    const int rsub = lane / LPR;
    uint32_t mirror[2 * BITS];
#pragma unroll
    for (int k = 0; k < 2 * BITS; ++k) mirror[k] = 0u;
#pragma unroll
    for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int j = 0; j < 32; ++j) place_field<BITS>(mirror + bb * BITS, j, 1u << (BITS - 1));

    uint32_t status = 0u;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r0 = gwarp * RPW; r0 < a.n_rows; r0 += nwarps * RPW) {
        const int64_t row = r0 + rsub;
        if (row >= a.n_rows) continue;
        float z[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) z[e] = 0.0f;
        for (int i0 = 0; i0 < D; i0 += 8) {
            float xv[8];
            if constexpr (BF16) {
                const uint4 u = ldg_nc_v4(static_cast<const uint16_t *>(a.x) + row * D + i0);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) { xv[2 * k] = bf16_lo(w4[k]); xv[2 * k + 1] = bf16_hi(w4[k]); }
            } else {
                const float * xr = static_cast<const float *>(a.x) + row * D + i0;
                const uint4 u0 = ldg_nc_v4(xr), u1 = ldg_nc_v4(xr + 4);
                xv[0] = __uint_as_float(u0.x); xv[1] = __uint_as_float(u0.y);
                xv[2] = __uint_as_float(u0.z); xv[3] = __uint_as_float(u0.w);
                xv[4] = __uint_as_float(u1.x); xv[5] = __uint_as_float(u1.y);
                xv[6] = __uint_as_float(u1.z); xv[7] = __uint_as_float(u1.w);
            }
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const float * pr = a.rot_f32 + (int64_t)(64 * q + e) * D + i0;
                const uint4 p0 = ldg_nc_v4(pr), p1 = ldg_nc_v4(pr + 4);
                float acc = z[e];
                acc = fmaf(__uint_as_float(p0.x), xv[0], acc);
                acc = fmaf(__uint_as_float(p0.y), xv[1], acc);
                acc = fmaf(__uint_as_float(p0.z), xv[2], acc);
                acc = fmaf(__uint_as_float(p0.w), xv[3], acc);
                acc = fmaf(__uint_as_float(p1.x), xv[4], acc);
                acc = fmaf(__uint_as_float(p1.y), xv[5], acc);
                acc = fmaf(__uint_as_float(p1.z), xv[6], acc);
                acc = fmaf(__uint_as_float(p1.w), xv[7], acc);
                z[e] = acc;
            }
        }
        finish_row<D, BITS>(z, row, q, cb, mirror, 1.0f, a, status);
    }
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

template <typename K>
int grid_for(K kernel, int threads) {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
    if (per_sm < 1) per_sm = 1;
    return per_sm * device_sm_count();
}

template <int D, int BITS, bool BF16>
int launch_wht_t(const tq_rotation * rot, const CodebookParams & cb, const QuantizeArgs & a,
                 cudaStream_t st) {
    WhtKernelSigns sg{};
    const double * r = rot->host.data();
    (void)r;
    for (int i = 0; i < 8; ++i) sg.d1_bits[i] = rot->d1_bits[i];
    for (int i = 0; i < D; ++i) {
        const uint32_t neg = (rot->d2_bits[i >> 5] >> (i & 31)) & 1u;
        if (BF16) sg.d2_mask[i >> 1] |= neg << ((i & 1) ? 31 : 15);
        else sg.d2_mask[i] = neg << 31;
    }
    auto k = quantize_wht_kernel<D, BITS, BF16>;
    const int threads = 256;
    const int64_t rows_per_cta = (int64_t)(threads / 32) * (32 / (D / 64));
    int64_t grid = grid_for(k, threads);
    const int64_t need = (a.n_rows + rows_per_cta - 1) / rows_per_cta;
    if (grid > need) grid = need;
    k<<<(unsigned)grid, threads, 0, st>>>(a, cb, sg);
    return (int)cudaGetLastError();
}

template <int D, int BITS, bool BF16>
int launch_dense_t(const CodebookParams & cb, const QuantizeArgs & a, cudaStream_t st) {
    auto k = quantize_dense_simple_kernel<D, BITS, BF16>;
    const int threads = 256;
    const int64_t rows_per_cta = (int64_t)(threads / 32) * (32 / (D / 64));
    int64_t grid = grid_for(k, threads);
    const int64_t need = (a.n_rows + rows_per_cta - 1) / rows_per_cta;
    if (grid > need) grid = need;
    k<<<(unsigned)grid, threads, 0, st>>>(a, cb);
    return (int)cudaGetLastError();
}

template <int D, int BITS>
int dispatch_dtype(const tq_rotation * rot, bool bf16, const CodebookParams & cb,
                   const QuantizeArgs & a, cudaStream_t st) {
    if (rot->kind == TQ_ROT_WHT)
        return bf16 ? launch_wht_t<D, BITS, true>(rot, cb, a, st)
                    : launch_wht_t<D, BITS, false>(rot, cb, a, st);
    return bf16 ? launch_dense_t<D, BITS, true>(cb, a, st) : launch_dense_t<D, BITS, false>(cb, a, st);
}

template <int D>
int dispatch_bits(const tq_rotation * rot, int bits, bool bf16, const CodebookParams & cb,
                  const QuantizeArgs & a, cudaStream_t st) {
    switch (bits) {
        case 2: return dispatch_dtype<D, 2>(rot, bf16, cb, a, st);
        case 3: return dispatch_dtype<D, 3>(rot, bf16, cb, a, st);
        case 4: return dispatch_dtype<D, 4>(rot, bf16, cb, a, st);
    }
    return (int)cudaErrorInvalidValue;
}

}  // namespace

int launch_quantize(const tq_rotation * rot, const tq_rotation * qjl, int bits, bool bf16,
                    int head_dim, const CodebookParams & cb, const QuantizeArgs & a,
                    void * stream) {
    (void)qjl;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (head_dim) {
        case 64: return dispatch_bits<64>(rot, bits, bf16, cb, a, st);
        case 128: return dispatch_bits<128>(rot, bits, bf16, cb, a, st);
        case 256: return dispatch_bits<256>(rot, bits, bf16, cb, a, st);
    }
    return (int)cudaErrorInvalidValue;
}

}  // namespace tq
