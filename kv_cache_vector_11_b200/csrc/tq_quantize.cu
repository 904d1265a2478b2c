// KV-cache quantization kernels (sm_100a).
//
// "TurboQuant+ upstream guide", sec. 5.1 / 5.2: rotate each row, take the
// norm of every 32-value block, quantize each normalised coordinate against
// the Lloyd-Max centroid table and pack the indices; sec. 4: the rotation is
// either the structured D1 @ H @ D2 Walsh-Hadamard form or a dense Haar QR
// matrix.
//
// Which kernel runs: bf16 rows take quantize_rot_tc_kernel (the rotation as
// one tcgen05 GEMM per 128-row tile, Walsh-Hadamard or Haar; at d = 256 two
// CTAs share a tile, one per half of the output) or, with QJL signs at d = 64 /
// 128, quantize_qjl_tc_kernel; the register kernels below serve fp32 input,
// the block-64/128 and fp32-norm formats and the other QJL shapes.
//
// Work decomposition of the register Walsh-Hadamard kernels: every lane owns 64
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

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>

#include "tq_device.cuh"
#include "tq_tc.cuh"

namespace tq {

namespace {

struct WhtKernelSigns {
    // bf16 input: word p holds the sign masks of elements 2p (bit 15) and
    // 2p+1 (bit 31); fp32 input: word i holds element i's mask in bit 31.
    uint32_t d2_mask[256];
    uint32_t d1_bits[8];
};

// 64-point unnormalised Walsh-Hadamard transform in registers.  Element
// 2i + s lives in z[i].x (s = 0) or z[i].y (s = 1): stage 1 acts inside the
// pairs, the five wider stages act on whole pairs with f32x2 adds.
__device__ __forceinline__ void wht64x2(float2 * z) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float a = z[i].x, b = z[i].y;
        z[i] = make_float2(a + b, a - b);
    }
    const float2 neg1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int hp = 1; hp < 32; hp <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((i & hp) == 0) {
                const float2 p = z[i], q = z[i + hp];
                z[i] = __fadd2_rn(p, q);
                z[i + hp] = __ffma2_rn(q, neg1, p);
            }
        }
    }
}

template <int BITS>
__device__ __forceinline__ void place_field(uint32_t * words, int j, uint32_t v) {
    const int p = j * BITS;
    const int wi = p >> 5, sh = p & 31;
    words[wi] += v << sh;
    if (sh + BITS > 32) words[wi + 1] += v >> (32 - sh);
}

// Quantizer constants shared by every row of a launch.
struct SearchParams {
    float scale, offset;
    uint32_t mask;        // (table size - 1) << 7: selects 128 * cell from the bits
};

// sqrt(x) with the hardware approximation (relative error ~2^-23; the
// stored norm is this rounded to fp16)
__device__ __forceinline__ float sqrt_approx(float x) {
    float y;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rsqrt_approx(float x) {
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Table row of value u (already divided by its block norm): the byte offset
// of the cell's 128-byte row, OR-ed with this lane's slot in the row.
__device__ __forceinline__ uint32_t cell_offset(float u, const SearchParams & sp, uint32_t slot) {
    return (__float_as_uint(fmaf(u, sp.scale, sp.offset)) & sp.mask) | slot;
}

// Code of coordinate j (value u, search key x = fmaf(u, scale, offset)) added
// into the packed words: acc += (base + [u >= t]) << (j * BITS), written as a
// multiply-add of base and a predicated add of the step, so the comparison
// never becomes a 0/1 value.  Fields that straddle two words take the plain
// route.
template <int BITS>
__device__ __forceinline__ void encode_one_at(uint32_t * acc, int p, float u, float x,
                                              const unsigned char * tab, uint32_t slot,
                                              uint32_t mask) {
    const float2 e = *reinterpret_cast<const float2 *>(tab + ((__float_as_uint(x) & mask) | slot));
    const int wi = p >> 5, sh = p & 31;
    if (sh + BITS <= 32) {
        asm("{\n\t.reg .pred q;\n\t"
            "setp.ge.f32 q, %2, %3;\n\t"
            "mad.lo.u32 %0, %1, %4, %0;\n\t"
            "@q add.u32 %0, %0, %4;\n\t}"
            : "+r"(acc[wi])
            : "r"(__float_as_uint(e.y)), "f"(u), "f"(e.x), "r"(1u << sh));
    } else {
        const uint32_t code = __float_as_uint(e.y) + (u >= e.x ? 1u : 0u);
        acc[wi] += code << sh;
        acc[wi + 1] += code >> (32 - sh);
    }
}

template <int BITS>
__device__ __forceinline__ void encode_one(uint32_t * acc, int j, float u, float x,
                                           const unsigned char * tab, uint32_t slot,
                                           uint32_t mask) {
    encode_one_at<BITS>(acc, j * BITS, u, x, tab, slot, mask);
}

// f(integral_constant<int, 0>) ... f(integral_constant<int, N - 1>)
template <typename F, int... I>
__device__ __forceinline__ void static_for_q_seq(F & f, std::integer_sequence<int, I...>) {
    (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for_q(F && f) {
    static_for_q_seq(f, std::make_integer_sequence<int, N>{});
}

// Lane-grouped row order (rows of NB 32-value blocks): code (block b,
// coordinate 4 g + e) at bit BITS * (4 (NB g + b) + e) of the row's stream, so
// that the decode lane that owns coordinates 4 g .. 4 g + 3 of every block
// finds all of them together.
template <int BITS, int NB>
__host__ __device__ constexpr int grouped_pos(int b, int j) {
    return BITS * (4 * (NB * (j >> 2) + b) + (j & 3));
}
// Bits of word w that block b's codes occupy (mask) and the pattern of its
// zero-block codes 2^(BITS-1) there (half).
template <int BITS, int NB>
__host__ __device__ constexpr uint32_t grouped_word_bits(int b, int w, bool half) {
    uint32_t m = 0u;
    for (int j = 0; j < 32; ++j)
        for (int t = 0; t < BITS; ++t) {
            const int bit = grouped_pos<BITS, NB>(b, j) + t;
            if ((bit >> 5) == w && (!half || t == BITS - 1)) m |= 1u << (bit & 31);
        }
    return m;
}

// Encode one 32-coordinate block (16 pairs z of unnormalised rotated values;
// `inv` = 1 / block norm, `nonzero` = block norm > 0) into BITS packed words.
// `tab` is the search table (entry e of slot s at byte e * 128 + 8 s, as
// {t, base}); `slot` = 8 * (this lane's slot); `mirror` has all-ones code
// fields where D1 = -1 (code -> 2^b - 1 - code).
template <int BITS>
__device__ __forceinline__ void encode_block(const float2 * z, float inv, bool nonzero,
                                             const unsigned char * tab, uint32_t slot,
                                             const SearchParams & sp, const uint32_t * mirror,
                                             uint32_t * out) {
    uint32_t acc[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) acc[k] = 0u;
    const float2 inv2 = make_float2(inv, inv);
    const float2 sc2 = make_float2(sp.scale, sp.scale);
    const float2 of2 = make_float2(sp.offset, sp.offset);
#pragma unroll
    for (int jp = 0; jp < 16; ++jp) {
        const float2 u = __fmul2_rn(z[jp], inv2);
        const float2 x = __ffma2_rn(u, sc2, of2);
        encode_one<BITS>(acc, 2 * jp, u.x, x.x, tab, slot, sp.mask);
        encode_one<BITS>(acc, 2 * jp + 1, u.y, x.y, tab, slot, sp.mask);
    }
    if (nonzero) {
#pragma unroll
        for (int k = 0; k < BITS; ++k) out[k] = acc[k] ^ mirror[k];
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

// The same encode, adding block b's codes into the words of a whole row in
// the lane-grouped order; a zero block gets the middle code 2^(BITS-1).
template <int BITS, int NB, int B>
__device__ __forceinline__ void encode_block_grouped(const float2 * z, float inv, bool nonzero,
                                                     const unsigned char * tab, uint32_t slot,
                                                     const SearchParams & sp, uint32_t * row) {
    const float2 inv2 = make_float2(inv, inv);
    const float2 sc2 = make_float2(sp.scale, sp.scale);
    const float2 of2 = make_float2(sp.offset, sp.offset);
#pragma unroll
    for (int jp = 0; jp < 16; ++jp) {
        const float2 u = __fmul2_rn(z[jp], inv2);
        const float2 x = __ffma2_rn(u, sc2, of2);
        encode_one_at<BITS>(row, grouped_pos<BITS, NB>(B, 2 * jp), u.x, x.x, tab, slot, sp.mask);
        encode_one_at<BITS>(row, grouped_pos<BITS, NB>(B, 2 * jp + 1), u.y, x.y, tab, slot, sp.mask);
    }
    if (!nonzero) {
#pragma unroll
        for (int w = 0; w < NB * BITS; ++w)
            row[w] = (row[w] & ~grouped_word_bits<BITS, NB>(B, w, false)) |
                     grouped_word_bits<BITS, NB>(B, w, true);
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
__device__ __forceinline__ void finish_row(const float2 * z, int64_t row, int q,
                                           const unsigned char * tab, uint32_t slot,
                                           const SearchParams & sp, const uint32_t * mirror,
                                           float norm_scale, const QuantizeArgs & a,
                                           uint32_t & status, bool valid = true) {
    constexpr int NB = D / 32;
    uint32_t words[2 * BITS];
    uint16_t nh[2];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int jp = 0; jp < 16; ++jp) ss2 = __ffma2_rn(z[16 * bb + jp], z[16 * bb + jp], ss2);
        const float ss = ss2.x + ss2.y;
        const float g = sqrt_approx(ss);
        if (valid && !isfinite(ss)) status |= TQ_STATUS_NONFINITE;
        bool sat;
        nh[bb] = norm_to_half_bits(g * norm_scale, &sat);
        if (valid && sat) status |= TQ_STATUS_NORM_SATURATED;
        encode_block<BITS>(z + 16 * bb, rsqrt_approx(ss), ss > 0.0f, tab, slot, sp,
                           mirror + bb * BITS, words + bb * BITS);
    }
    if (!valid) return;
    store_words<2 * BITS>(a.codes + row * (NB * BITS) + q * 2 * BITS, words);
    *reinterpret_cast<uint32_t *>(a.norms + row * NB + 2 * q) =
        (uint32_t)nh[0] | ((uint32_t)nh[1] << 16);
}

// Codes of one 32-coordinate piece by binary search over the ascending
// decision boundaries t (shared memory): code = #{i : u >= t_i}, u = z * inv.
// Used by the format variants, whose codebooks (up to block 128) can have
// boundaries closer than the uniform-grid table resolves.
template <int BITS>
__device__ __forceinline__ void encode_block_bs(const float2 * z, float inv, bool nonzero,
                                                const float * t, const uint32_t * mirror,
                                                uint32_t * out) {
    constexpr int L = (1 << BITS) - 1;
    uint32_t acc[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) acc[k] = 0u;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float u = (j & 1 ? z[j >> 1].y : z[j >> 1].x) * inv;
        uint32_t c = 0u;
#pragma unroll
        for (int step = 1 << (BITS - 1); step > 0; step >>= 1) {
            const uint32_t p = c + (uint32_t)step - 1u;
            if (p < (uint32_t)L && u >= t[p]) c += (uint32_t)step;
        }
        place_field<BITS>(acc, j, nonzero ? c : (1u << (BITS - 1)));
    }
#pragma unroll
    for (int k = 0; k < BITS; ++k) out[k] = nonzero ? (acc[k] ^ mirror[k]) : acc[k];
}

// Epilogue of the format variants: norm blocks of BLOCK = 32 / 64 / 128
// coordinates (the codebook of that block size is in the search table), norms
// stored as fp16 or fp32, optionally divided by ||c[idx_blk]|| (norm
// correction: the dequantized block then has the block's own norm).  The
// lane holds the 64 coordinates of slice q of the row, i.e. two 32-sub-blocks
// whose codes have the same layout at every block size; a 128-block spans the
// slices of lanes q and q ^ 1, which are adjacent lanes of the warp.
template <int D, int BITS, int BLOCK>
__device__ __forceinline__ void finish_row_var(const float2 * z, int64_t row, int q,
                                               const unsigned char * tab, uint32_t slot,
                                               const SearchParams & sp, const uint32_t * mirror,
                                               float norm_scale, const QuantizeArgs & a,
                                               const float * c2, const float * tb,
                                               uint32_t & status) {
    constexpr int NB = D / 32;
    constexpr int NBK = D / BLOCK;
    static_assert(BLOCK == 32 || BLOCK == 64 || (BLOCK == 128 && D >= 128), "block");
    const int lane = threadIdx.x & 31;
    const unsigned pair_mask = 3u << (lane & ~1);   // the two lanes of a 128-block
    float ss[2];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int jp = 0; jp < 16; ++jp) s2 = __ffma2_rn(z[16 * bb + jp], z[16 * bb + jp], s2);
        ss[bb] = s2.x + s2.y;
    }
    float sblk[2];
    if constexpr (BLOCK == 32) {
        sblk[0] = ss[0];
        sblk[1] = ss[1];
    } else {
        float t = ss[0] + ss[1];
        if constexpr (BLOCK == 128) t += __shfl_xor_sync(pair_mask, t, 1);
        sblk[0] = sblk[1] = t;
    }
    uint32_t words[2 * BITS];
    float csq[2] = {0.0f, 0.0f};
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        (void)tab; (void)slot; (void)sp;
        encode_block_bs<BITS>(z + 16 * bb, rsqrt_approx(sblk[bb]), sblk[bb] > 0.0f, tb,
                              mirror + bb * BITS, words + bb * BITS);
        if (a.norm_corr) {
            // squared centroids are symmetric, so the mirrored codes serve
#pragma unroll
            for (int j = 0; j < 32; ++j) csq[bb] += c2[extract_code<BITS>(words + bb * BITS, j)];
        }
    }
    float cblk[2] = {csq[0], csq[1]};
    if constexpr (BLOCK != 32) {
        float t = csq[0] + csq[1];
        if constexpr (BLOCK == 128) t += __shfl_xor_sync(pair_mask, t, 1);
        cblk[0] = cblk[1] = t;
    }
    float g[2];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        if (!isfinite(sblk[bb])) status |= TQ_STATUS_NONFINITE;
        g[bb] = sqrt_approx(sblk[bb]) * norm_scale;
        if (a.norm_corr) g[bb] = cblk[bb] > 0.0f ? g[bb] / sqrtf(cblk[bb]) : 0.0f;
    }
    store_words<2 * BITS>(a.codes + row * (NB * BITS) + q * 2 * BITS, words);
    // the lane's norms: blocks 2q, 2q+1 (BLOCK 32), q (64) or q/2 (128, even q)
    constexpr int PER = BLOCK == 32 ? 2 : 1;
    const int first = BLOCK == 32 ? 2 * q : BLOCK == 64 ? q : q >> 1;
    const bool writer = BLOCK != 128 || (q & 1) == 0;
    if (!writer) return;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int64_t idx = row * NBK + first + i;
        if (a.norm_f32) {
            reinterpret_cast<float *>(a.norms)[idx] = g[i];
        } else {
            bool sat;
            a.norms[idx] = norm_to_half_bits(g[i], &sat);
            if (sat) status |= TQ_STATUS_NORM_SATURATED;
        }
    }
}

// Copy the search table into shared memory, one copy per lane of a half
// warp (entry e, copy c at float2 index e * 16 + c: byte e * 128 + 8 c), so
// that table reads never conflict; returns the table's base.
__device__ __forceinline__ const unsigned char * load_search_table(float2 * stab,
                                                                 const SearchTable & st) {
    for (uint32_t i = threadIdx.x; i < st.size * 16; i += blockDim.x) {
        const uint32_t e = i >> 4;
        stab[i] = make_float2(st.t[e], __int_as_float(st.base[e]));
    }
    __syncthreads();
    return reinterpret_cast<const unsigned char *>(stab);
}

// VAR: the format variants' epilogue (finish_row_var) for norm blocks of
// BLOCK coordinates; the default instance keeps the 32-block fp16 epilogue.
template <int D, int BITS, bool BF16, bool VAR = false, int BLOCK = 32>
__global__ void __launch_bounds__(256)
quantize_wht_kernel(const __grid_constant__ QuantizeArgs a, const __grid_constant__ SearchTable st,
                    const __grid_constant__ WhtKernelSigns sg) {
    constexpr int LPR = D / 64;   // lanes per row
    constexpr int RPW = 32 / LPR; // rows per warp step
    constexpr uint32_t FIELD = (1u << BITS) - 1u;
    extern __shared__ float2 stab[];
    float * c2 = reinterpret_cast<float *>(stab + st.size * 16);
    float * tb = c2 + 16;
    if (VAR && threadIdx.x < 16) {
        c2[threadIdx.x] = a.centroid_sq[threadIdx.x];
        tb[threadIdx.x] = a.boundary[threadIdx.x];
    }
    const unsigned char * tab = load_search_table(stab, st);
    const uint32_t slot = 8u * (threadIdx.x & 15u);
    const SearchParams sp{st.scale, st.offset, st.mask};
    const int lane = threadIdx.x & 31;
    const int q = lane % LPR;
    const int rsub = lane / LPR;

    // All-ones code fields where D1 = -1, for the lane's two blocks (2q, 2q+1).
    uint32_t mirror[2 * BITS];
#pragma unroll
    for (int k = 0; k < 2 * BITS; ++k) mirror[k] = 0u;
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        const uint32_t d1 = sg.d1_bits[2 * q + bb];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            place_field<BITS>(mirror + bb * BITS, j, ((d1 >> j) & 1u) ? FIELD : 0u);
    }
    // Signs of the slice-level butterflies for this lane: (-1)^popcount(q & a).
    const float s1 = (q & 1) ? -1.0f : 1.0f;
    const float s2 = (q & 2) ? -1.0f : 1.0f;
    const float2 s1v = make_float2(s1, s1), s2v = make_float2(s2, s2);
    const float norm_scale = rsqrtf((float)D);

    uint32_t status = 0u;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r0 = gwarp * RPW; r0 < a.n_rows; r0 += nwarps * RPW) {
        const int64_t row = r0 + rsub;
        if (row >= a.n_rows) continue;
        float2 z[32];
        if constexpr (BF16) {
            const uint16_t * xr = static_cast<const uint16_t *>(a.x) + row * D;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float2 v[LPR][4];
#pragma unroll
                for (int s = 0; s < LPR; ++s) {
                    const uint4 u = ldg_nc_v4(xr + s * 64 + c * 8);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t w = w4[k] ^ sg.d2_mask[(s * 64 + c * 8) / 2 + k];
                        v[s][k] = make_float2(bf16_lo(w), bf16_hi(w));
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if constexpr (LPR == 1) z[c * 4 + k] = v[0][k];
                    else if constexpr (LPR == 2) z[c * 4 + k] = __ffma2_rn(s1v, v[1][k], v[0][k]);
                    else z[c * 4 + k] = __ffma2_rn(s2v, __ffma2_rn(s1v, v[3][k], v[2][k]),
                                                   __ffma2_rn(s1v, v[1][k], v[0][k]));
                }
            }
        } else {
            const float * xr = static_cast<const float *>(a.x) + row * D;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                float2 v[LPR][2];
#pragma unroll
                for (int s = 0; s < LPR; ++s) {
                    const uint4 u = ldg_nc_v4(xr + s * 64 + c * 4);
                    const int e = s * 64 + c * 4;
                    v[s][0] = make_float2(__uint_as_float(u.x ^ sg.d2_mask[e]),
                                          __uint_as_float(u.y ^ sg.d2_mask[e + 1]));
                    v[s][1] = make_float2(__uint_as_float(u.z ^ sg.d2_mask[e + 2]),
                                          __uint_as_float(u.w ^ sg.d2_mask[e + 3]));
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    if constexpr (LPR == 1) z[c * 2 + k] = v[0][k];
                    else if constexpr (LPR == 2) z[c * 2 + k] = __ffma2_rn(s1v, v[1][k], v[0][k]);
                    else z[c * 2 + k] = __ffma2_rn(s2v, __ffma2_rn(s1v, v[3][k], v[2][k]),
                                                   __ffma2_rn(s1v, v[1][k], v[0][k]));
                }
            }
        }
        wht64x2(z);
        if constexpr (VAR)
            finish_row_var<D, BITS, BLOCK>(z, row, q, tab, slot, sp, mirror, norm_scale, a, c2, tb,
                                           status);
        else
            finish_row<D, BITS>(z, row, q, tab, slot, sp, mirror, norm_scale, a, status);
    }
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

constexpr uint64_t kQWaitNs = 1000000000ull;      // 1 s bound on one wait of the tensor-core kernels

// ---------------------------------------------------------------------------
// Rotation of bf16 rows on the tensor cores, y = R x for a tile of 128 rows as
// a tcgen05 GEMM with fp32 accumulation: A = the x tile exactly as its TMA
// boxes land (64-column slices, 128-byte swizzle), B = R, built once per CTA in
// the same layout.  Walsh-Hadamard: D1 H D2 has entries +-1 (the 1/sqrt(d)
// factor only scales the stored norm), exact in bf16: one MMA per K step.
// Dense (Haar) R: B = R_hi + R_lo, two bf16 matrices, two MMAs per K step
// (products carry ~17 bits).  At d = 256, R (128 or 256 KB) does not fit next
// to the tiles, so two CTAs share each tile: CTA 2 p + h computes output
// columns 128 h .. 128 h + 127 (blocks 4 h .. 4 h + 3) of pair p's tiles, with
// its half of R resident; the pair reads every tile at about the same time,
// so the second read comes from L2.  Warp roles:
//  * warps 0 .. 4 G - 1 (epilogue, G = output columns / 32 per CTA), in G
//    groups of four: group g encodes the tiles k = g, g + G, ..., so G tiles
//    are in flight, each in its own TMEM accumulator; warp 4 g + q reads TMEM
//    lanes 32 q .. + 31, one row per thread, and the thread runs the norm and
//    table search of every block of its row (its CTA's half at d = 256) and
//    stores those code words in 16-byte stores (8-byte ones where a row of
//    3-bit codes at d = 64 is only 8-byte aligned) and the norms in one store.
//    Consecutive threads hold consecutive rows, so a warp's stores cover one
//    contiguous stretch of the output;
//  * warp 4 G, one thread: TMA copies into a ring of tile stages (4 at d <= 128;
//    at d = 256, 2 for Walsh-Hadamard, 1 for Haar) and the MMAs into the G
//    accumulators.
// Every wait is bounded.
// ---------------------------------------------------------------------------
constexpr int kWtStages = 4;
constexpr int kWtRows = 128;

template <int D, int BITS, bool DENSE>
struct WtCfg {
    // CTAs per tile, each with its half of the output columns at d = 256 (64 KB
    // of B for Walsh-Hadamard, 128 KB of hi + lo for Haar)
    static constexpr int NH = D <= 128 ? 1 : 2;
    static constexpr int NOUT = D / NH;                    // output columns per CTA
    static constexpr int NB = D / 32;                      // blocks of a row
    static constexpr int NBO = NOUT / 32;                  // blocks per CTA
    static constexpr int GROUPS = NBO;                     // tiles in flight
    static constexpr int EPI_WARPS = 4 * GROUPS;
    static constexpr int EPI_THREADS = 32 * EPI_WARPS;
    static constexpr int THREADS = EPI_THREADS + 32;       // + MMA warp
    static constexpr int SLICE = kWtRows * 128;            // one 64-column slice of a tile
    static constexpr int SPT = D / 64;                     // slices per tile
    static constexpr int B_SLICE = NOUT * 128;             // 64 K-columns of B
    static constexpr int B_BYTES = NOUT * D * 2;           // one bf16 matrix (DENSE: hi, then lo)
    // slices in the ring: 4 tile stages at d <= 128; at d = 256 two next to
    // the Walsh-Hadamard half of B, one next to the Haar half (quarters with
    // two stages measured slower: half the epilogue warps per SM)
    static constexpr int RING = D <= 128 ? kWtStages * SPT : (DENSE ? 1 : 2) * SPT;
    static constexpr int OFF_B = RING * SLICE;
    static constexpr int SMEM = 1024 + OFF_B + (DENSE ? 2 : 1) * B_BYTES;   // + slack to align to 1024
    static constexpr int ROW_WORDS = NB * BITS;            // code words of a row
    static constexpr int CTA_WORDS = NBO * BITS;           // code words this CTA writes per row
    static constexpr uint32_t TCOLS = GROUPS * NOUT;       // one accumulator per group
    static_assert(D == 64 || D == 128 || D == 256, "tensor-core rotation path: d = 64, 128 or 256");
    static_assert(TCOLS <= 512 && (TCOLS & (TCOLS - 1)) == 0, "TMEM allocation: power of 2, <= 512");
    static_assert(RING % SPT == 0 && RING <= 8, "whole tiles in the ring, at most 8 slots");
};

template <int D, int BITS, bool DENSE, bool GROUPED = false>
__global__ void __launch_bounds__(WtCfg<D, BITS, DENSE>::THREADS, 1)
quantize_rot_tc_kernel(const __grid_constant__ QuantizeArgs a,
                       const __grid_constant__ SearchTable st,
                       const __grid_constant__ WhtKernelSigns sg,
                       const __grid_constant__ CUtensorMap tmap) {
    using C = WtCfg<D, BITS, DENSE>;
    constexpr int NB = C::NB, NBO = C::NBO, G = C::GROUPS, RW = C::ROW_WORDS, SPT = C::SPT;
    constexpr int ST = C::RING / SPT, NOUT = C::NOUT;      // tile stages
    extern __shared__ unsigned char wsm_raw[];
    __shared__ __align__(128) float2 s_qtab[kSearchMax * 16];
    // full[ST], empty[ST], accumulator full[G] / empty[G]
    __shared__ __align__(8) uint64_t s_bar[2 * ST + 2 * G];
    __shared__ uint32_t s_tmem;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = (int)(blockIdx.x % C::NH);            // output half of this CTA
    const int64_t pair = blockIdx.x / C::NH, n_pairs = gridDim.x / C::NH;
    const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(wsm_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;   // swizzle atoms need 1024-byte alignment
    unsigned char * wsm = wsm_raw + (base_s - raw_s);
    const uint32_t bar_s = (uint32_t)__cvta_generic_to_shared(s_bar);
    const uint32_t full_b = bar_s, empty_b = bar_s + 8u * ST;
    const uint32_t accf_b = bar_s + 16u * ST, acce_b = accf_b + 8u * G;

    // B[n][k] = d1_n' (-1)^popc(n' & k) d2_k as bf16 +-1 (or R[n'][k] as hi and
    // lo parts), n' = NOUT * half + n the output column; element (n, k) in
    // slice k / 64, row n, 16-byte chunk ((k % 64) / 8) ^ (n % 8)
    for (int i = tid; i < NOUT * (D / 8); i += C::THREADS) {
        const int n = i / (D / 8), kc = i % (D / 8);
        const int ng = NOUT * half + n;
        const int boff = C::OFF_B + (kc >> 3) * C::B_SLICE + n * 128 + 16 * ((kc & 7) ^ (n & 7));
        if constexpr (DENSE) {
            *reinterpret_cast<uint4 *>(wsm + boff) = ldg_nc_v4(a.rot_hi + (int64_t)ng * D + 8 * kc);
            *reinterpret_cast<uint4 *>(wsm + boff + C::B_BYTES) = ldg_nc_v4(a.rot_lo + (int64_t)ng * D + 8 * kc);
            continue;
        }
        const uint32_t sn = (sg.d1_bits[ng >> 5] >> (ng & 31)) & 1u;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t pr = 0u;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int k = 8 * kc + 2 * e + h;
                const uint32_t sk = (sg.d2_mask[k >> 1] >> ((k & 1) ? 31 : 15)) & 1u;
                const uint32_t neg = (sn ^ sk ^ (uint32_t)__popc(ng & k)) & 1u;
                pr |= (neg ? 0xBF80u : 0x3F80u) << (16 * h);
            }
            w[e] = pr;
        }
        *reinterpret_cast<uint4 *>(wsm + boff) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (tid == 0) {
        for (int i = 0; i < ST; ++i) {
            tc::mbar_init(full_b + 8u * i, 1);
            tc::mbar_init(empty_b + 8u * i, 1);
        }
        for (int b = 0; b < G; ++b) {
            tc::mbar_init(accf_b + 8u * b, 1);
            tc::mbar_init(acce_b + 8u * b, 4);       // the four warps of group b
        }
    }
    if (warp == C::EPI_WARPS) tc::tmem_alloc((uint32_t)__cvta_generic_to_shared(&s_tmem), C::TCOLS);
    tc::fence_proxy_async();            // B, written by generic stores, is read by the MMAs
    tc::fence_before_sync();
    const unsigned char * tab = load_search_table(s_qtab, st);   // ends with __syncthreads
    tc::fence_after_sync();
    const uint32_t tmem = s_tmem;

    const int64_t n_tiles = (a.n_rows + kWtRows - 1) / kWtRows;
    const int64_t n_my = pair < n_tiles ? (n_tiles - 1 - pair) / n_pairs + 1 : 0;
    auto tile_of = [&](int64_t k) { return pair + k * n_pairs; };
    uint32_t status = 0u;

    if (warp == C::EPI_WARPS) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kWtRows, NOUT);
            // tile t -> stage t % ST (its SPT slices in consecutive slots)
            auto issue = [&](int64_t t) {
                const int s = (int)(t % ST);
                tc::mbar_arrive_expect_tx(full_b + 8u * s, (uint32_t)(SPT * C::SLICE));
#pragma unroll
                for (int sp = 0; sp < SPT; ++sp)
                    tc::tma_load_2d(base_s + (uint32_t)((s * SPT + sp) * C::SLICE), &tmap, 64 * sp,
                                    (int32_t)(tile_of(t) * kWtRows), full_b + 8u * s);
            };
            int64_t issued = 0;
            for (; issued < n_my && issued < ST; ++issued) issue(issued);
            int64_t k = 0;
            bool ok = true;
            for (; k < n_my; ++k) {
                const int s = (int)(k % ST), b = (int)(k % G);
                const uint32_t ph = (uint32_t)((k / ST) & 1);
                // tile k has landed; accumulator b was read back (tile k - G)
                ok = tc::mbar_wait(full_b + 8u * s, ph, kQWaitNs) &&
                     tc::mbar_wait(acce_b + 8u * b, (uint32_t)(((k / G) & 1) ^ 1), kQWaitNs);
                if (!ok) break;
                tc::fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int sp = ks >> 2;
                    const uint64_t ad = tc::smem_desc_sw128(base_s + (uint32_t)((s * SPT + sp) * C::SLICE + (ks & 3) * 32));
                    const uint32_t bo = base_s + (uint32_t)(C::OFF_B + sp * C::B_SLICE + (ks & 3) * 32);
                    tc::mma_bf16(tmem + (uint32_t)(b * NOUT), ad, tc::smem_desc_sw128(bo), idesc, ks > 0 ? 1u : 0u);
                    if constexpr (DENSE)
                        tc::mma_bf16(tmem + (uint32_t)(b * NOUT), ad,
                                     tc::smem_desc_sw128(bo + (uint32_t)C::B_BYTES), idesc, 1u);
                }
                tc::commit(empty_b + 8u * s);
                tc::commit(accf_b + 8u * b);
                if (issued < n_my) {
                    // refill the stage once this tile's MMAs have read it
                    if (!tc::mbar_wait(empty_b + 8u * s, ph, kQWaitNs)) {
                        ok = false;
                        ++k;                  // tile k was consumed
                        break;
                    }
                    issue(issued++);
                }
            }
            if (!ok) {
                status |= TQ_STATUS_TIMEOUT;
                // let the copies still in flight land before the CTA exits
                for (int64_t t = k; t < issued; ++t)
                    tc::mbar_wait(full_b + 8u * (uint32_t)(t % ST), (uint32_t)((t / ST) & 1), kQWaitNs);
            }
        }
    } else {
        const int grp = warp >> 2, quad = warp & 3;
        const int r = 32 * quad + lane;                      // row within the tile
        const uint32_t slot = 8u * (uint32_t)(lane & 15);
        const SearchParams sp{st.scale, st.offset, st.mask};
        const float norm_scale = DENSE ? 1.0f : rsqrtf((float)D);
        const uint32_t no_mirror[BITS] = {};
        constexpr int CW = C::CTA_WORDS;
        // 16-byte stores need 16-byte aligned outputs (and a multiple of 16
        // bytes per row and CTA)
        constexpr bool kRow16 = (CW % 4) == 0;
        const bool vec_ok = ((reinterpret_cast<uintptr_t>(a.codes) | reinterpret_cast<uintptr_t>(a.norms)) & 15u) == 0;
        const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(grp * NOUT);
        for (int64_t k = grp; k < n_my; k += G) {
            const bool ok = tc::mbar_wait(accf_b + 8u * grp, (uint32_t)((k / G) & 1), kQWaitNs);
            if (!__all_sync(0xffffffffu, ok)) {      // warp-uniform exit
                status |= TQ_STATUS_TIMEOUT;
                break;
            }
            tc::fence_after_sync();
            const int64_t row = tile_of(k) * kWtRows + r;
            const bool valid = row < a.n_rows;       // rows past the end arrive as zeros
            uint32_t * dst = a.codes + row * RW + half * CW;
            uint32_t words[CW];
            uint16_t nh[NBO];
            if constexpr (GROUPED) {
                static_assert(C::NH == 1 && RW % 4 == 0, "lane-grouped rows: one CTA per tile, whole 16-byte chunks");
                // every block adds its codes at their lane-grouped places in
                // the row's words; the row leaves after its last block
#pragma unroll
                for (int i = 0; i < RW; ++i) words[i] = 0u;
                static_for_q<NBO>([&](auto BLK) {
                    constexpr int blk = decltype(BLK)::value;
                    float v[32];
                    tc::tmem_ld32(tl + (uint32_t)(32 * blk), v);
                    if (blk == NBO - 1) {
                        tc::fence_before_sync();
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(acce_b + 8u * grp);
                    }
                    float2 z[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) z[i] = make_float2(v[2 * i], v[2 * i + 1]);
                    float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int i = 0; i < 16; ++i) ss2 = __ffma2_rn(z[i], z[i], ss2);
                    const float ss = ss2.x + ss2.y;
                    if (valid && !isfinite(ss)) status |= TQ_STATUS_NONFINITE;
                    bool sat;
                    nh[blk] = norm_to_half_bits(sqrt_approx(ss) * norm_scale, &sat);
                    if (valid && sat) status |= TQ_STATUS_NORM_SATURATED;
                    encode_block_grouped<BITS, NB, blk>(z, rsqrt_approx(ss), ss > 0.0f, tab, slot, sp, words);
                });
                if (!valid) continue;
                if (vec_ok) {
#pragma unroll
                    for (int i = 0; i < RW; i += 4)
                        *reinterpret_cast<uint4 *>(dst + i) = make_uint4(words[i], words[i + 1], words[i + 2], words[i + 3]);
                    *reinterpret_cast<uint2 *>(a.norms + row * NB) =
                        make_uint2(nh[0] | ((uint32_t)nh[1] << 16), nh[2] | ((uint32_t)nh[3] << 16));
                } else {
#pragma unroll
                    for (int i = 0; i < RW; ++i) dst[i] = words[i];
#pragma unroll
                    for (int i = 0; i < NB; ++i) a.norms[row * NB + i] = nh[i];
                }
                continue;
            }
#pragma unroll
            for (int blk = 0; blk < NBO; ++blk) {
                float v[32];
                tc::tmem_ld32(tl + (uint32_t)(32 * blk), v);
                if (blk == NBO - 1) {
                    // the accumulator is free for tile k + G
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(acce_b + 8u * grp);
                }
                float2 z[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) z[i] = make_float2(v[2 * i], v[2 * i + 1]);
                float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int i = 0; i < 16; ++i) ss2 = __ffma2_rn(z[i], z[i], ss2);
                const float ss = ss2.x + ss2.y;
                if (valid && !isfinite(ss)) status |= TQ_STATUS_NONFINITE;
                bool sat;
                nh[blk] = norm_to_half_bits(sqrt_approx(ss) * norm_scale, &sat);
                if (valid && sat) status |= TQ_STATUS_NORM_SATURATED;
                encode_block<BITS>(z, rsqrt_approx(ss), ss > 0.0f, tab, slot, sp, no_mirror,
                                   words + blk * BITS);
                // store every vector chunk of the row that is complete now, so
                // that few code words stay live across blocks
                if (valid && vec_ok) {
                    constexpr int VW = kRow16 ? 4 : 2;
#pragma unroll
                    for (int c = 0; c < CW / VW; ++c) {
                        if (VW * c + VW > blk * BITS && VW * c + VW <= (blk + 1) * BITS) {
                            if constexpr (VW == 4)
                                *reinterpret_cast<uint4 *>(dst + 4 * c) =
                                    make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
                            else
                                *reinterpret_cast<uint2 *>(dst + 2 * c) = make_uint2(words[2 * c], words[2 * c + 1]);
                        }
                    }
                } else if (valid) {
#pragma unroll
                    for (int i = 0; i < BITS; ++i) dst[blk * BITS + i] = words[blk * BITS + i];
                }
            }
            if (!valid) continue;
            uint16_t * ndst = a.norms + row * NB + half * NBO;
            if (vec_ok) {
                if constexpr (NBO == 4)
                    *reinterpret_cast<uint2 *>(ndst) = make_uint2(nh[0] | ((uint32_t)nh[1] << 16), nh[2] | ((uint32_t)nh[3] << 16));
                else
                    *reinterpret_cast<uint32_t *>(ndst) = nh[0] | ((uint32_t)nh[1] << 16);
            } else {
#pragma unroll
                for (int i = 0; i < NBO; ++i) ndst[i] = nh[i];
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == C::EPI_WARPS) tc::tmem_dealloc(tmem, C::TCOLS);
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

// Dense rotation y = P x computed on the CUDA cores from the fp32 matrix in
// global memory (L1/L2 resident); same lane decomposition and epilogue as the
// Walsh-Hadamard kernel.  This is the straightforward form of the dense path.
template <int D, int BITS, bool BF16, bool VAR = false, int BLOCK = 32>
__global__ void __launch_bounds__(256)
quantize_dense_simple_kernel(const __grid_constant__ QuantizeArgs a,
                             const __grid_constant__ SearchTable st) {
    constexpr int LPR = D / 64;
    constexpr int RPW = 32 / LPR;
    extern __shared__ float2 stab[];
    float * c2 = reinterpret_cast<float *>(stab + st.size * 16);
    float * tb = c2 + 16;
    if (VAR && threadIdx.x < 16) {
        c2[threadIdx.x] = a.centroid_sq[threadIdx.x];
        tb[threadIdx.x] = a.boundary[threadIdx.x];
    }
    const unsigned char * tab = load_search_table(stab, st);
    const uint32_t slot = 8u * (threadIdx.x & 15u);
    const SearchParams sp{st.scale, st.offset, st.mask};
    const int lane = threadIdx.x & 31;
    const int q = lane % LPR;
    const int rsub = lane / LPR;
    uint32_t mirror[2 * BITS];
#pragma unroll
    for (int k = 0; k < 2 * BITS; ++k) mirror[k] = 0u;

    uint32_t status = 0u;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r0 = gwarp * RPW; r0 < a.n_rows; r0 += nwarps * RPW) {
        const int64_t row = r0 + rsub;
        if (row >= a.n_rows) continue;
        float zf[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) zf[e] = 0.0f;
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
                float acc = zf[e];
                acc = fmaf(__uint_as_float(p0.x), xv[0], acc);
                acc = fmaf(__uint_as_float(p0.y), xv[1], acc);
                acc = fmaf(__uint_as_float(p0.z), xv[2], acc);
                acc = fmaf(__uint_as_float(p0.w), xv[3], acc);
                acc = fmaf(__uint_as_float(p1.x), xv[4], acc);
                acc = fmaf(__uint_as_float(p1.y), xv[5], acc);
                acc = fmaf(__uint_as_float(p1.z), xv[6], acc);
                acc = fmaf(__uint_as_float(p1.w), xv[7], acc);
                zf[e] = acc;
            }
        }
        float2 z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = make_float2(zf[2 * i], zf[2 * i + 1]);
        if constexpr (VAR)
            finish_row_var<D, BITS, BLOCK>(z, row, q, tab, slot, sp, mirror, 1.0f, a, c2, tb, status);
        else
            finish_row<D, BITS>(z, row, q, tab, slot, sp, mirror, 1.0f, a, status);
    }
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

// ---------------------------------------------------------------------------
// Quantize with the QJL residual stage ("Google TurboQuant deep dive",
// sec. 2.2: the residual of the first stage goes through a Gaussian
// projection and only the signs are kept).
//
// A CTA of 128 * (d / 64) threads handles tiles of 128 rows.  Lanes rotate,
// take norms and encode exactly as above; the table entry of each coordinate
// also carries the two centroids of its cell, so the residual
// r' = y / sqrt(d) - fp16(norm) c[code] (for the Walsh-Hadamard rotation,
// before D1; D1 is folded into the projection as S diag(D1)) is formed in
// registers.  The projection z = S' r' of the whole tile is one GEMM on the
// tensor cores: r' and S' are split into bf16 high and low parts (written in
// the canonical K-major layout), three tcgen05.mma per 16-wide K step
// (hi*hi + hi*lo + lo*hi, ~17-bit products) accumulate the 128 x m fp32
// result in TMEM, one thread issues them and commits to an mbarrier (bounded
// wait), and each row's m signs are read back from its TMEM lane.
// ---------------------------------------------------------------------------
constexpr uint64_t kQjlWaitNs = 1000000000ull;   // 1 s bound on one tile's MMAs

template <int D>
struct QjlCfg {
    static constexpr int LPR = D / 64;
    static constexpr int THREADS = 128 * LPR;
    static constexpr int TILE = 128;                     // rows per tile (MMA M)
    static constexpr int OFF_TAB = 0;                    // float4 entries, 8 copies
    static constexpr int OFF_AHI = kSearchMax * 8 * 16;  // residual tile, bf16 high part
    static constexpr int OFF_ALO = OFF_AHI + TILE * D * 2;
    static constexpr int OFF_B = OFF_ALO + TILE * D * 2; // S' high part, then low part (m x d)
    // bf16 rows of d <= 128 arrive by TMA into two 1 KiB-aligned stages after
    // the barrier words (2-D boxes of 64 columns x 128 rows, 128-byte swizzle)
    static constexpr bool STAGED_D = D <= 128;
    static constexpr int X_STAGE = TILE * D * 2;
    __host__ __device__ static int off_x(int m) { return (OFF_B + 2 * m * D * 2 + 64 + 1023) / 1024 * 1024; }
    static int smem_bytes(int m, bool staged) {
        return staged ? off_x(m) + 2 * X_STAGE : OFF_B + 2 * m * D * 2 + 64;
    }
};

// Byte offset of element (r, k) of a K-major bf16 matrix with K = `kdim` in
// the canonical no-swizzle layout (8-row x 16-byte core matrices).
__device__ __forceinline__ uint32_t canon_elem(int r, int k, int kdim) {
    return (uint32_t)((((r >> 3) * (kdim >> 3) + (k >> 3)) << 7) + ((r & 7) << 4) + ((k & 7) << 1));
}

__device__ __forceinline__ uint32_t bf16x2_hi_lo(float a, float b, uint32_t * lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - __low2float(h), b - __high2float(h));
    *lo = *reinterpret_cast<const uint32_t *>(&l);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D, int BITS, bool BF16, bool DENSE>
__global__ void __launch_bounds__(QjlCfg<D>::THREADS, 1)
quantize_qjl_kernel(const __grid_constant__ QuantizeArgs a, const __grid_constant__ SearchTable st,
                    const __grid_constant__ WhtKernelSigns sg, const __grid_constant__ CodebookParams cb,
                    const __grid_constant__ CUtensorMap xmap) {
    using C = QjlCfg<D>;
    constexpr bool STAGED = BF16 && C::STAGED_D;
    constexpr int LPR = C::LPR;
    constexpr int TILE = C::TILE;
    constexpr int THREADS = C::THREADS;
    constexpr uint32_t FIELD = (1u << BITS) - 1u;
    extern __shared__ __align__(128) unsigned char qs[];
    float4 * tab4 = reinterpret_cast<float4 *>(qs + C::OFF_TAB);
    const int m = a.qjl_m;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int q = lane % LPR;
    const int trow = warp * (32 / LPR) + lane / LPR;     // row within the tile
    const int ncode = 1 << BITS;
    const uint32_t qs_s = (uint32_t)__cvta_generic_to_shared(qs);
    const uint32_t s_ahi = qs_s + C::OFF_AHI, s_alo = qs_s + C::OFF_ALO;
    const uint32_t s_bhi = qs_s + C::OFF_B, s_blo = s_bhi + (uint32_t)(m * D * 2);
    const int off_misc = C::OFF_B + 2 * m * D * 2;
    const uint32_t s_mbar = qs_s + off_misc;
    uint32_t * tmem_holder = reinterpret_cast<uint32_t *>(qs + off_misc + 8);
    volatile int * abort_flag = reinterpret_cast<volatile int *>(qs + off_misc + 12);
    const uint32_t s_full = qs_s + off_misc + 16;        // two stage barriers (STAGED)
    const int off_x = C::off_x(m);
    uint32_t tcols = 32;
    while ((int)tcols < m) tcols <<= 1;

    // table: {t, base, c[base], c[base + 1]}, entry e copy c at e * 8 + c
    for (uint32_t i = tid; i < st.size * 8; i += THREADS) {
        const uint32_t e = i >> 3;
        const int b = st.base[e];
        tab4[i] = make_float4(st.t[e], __int_as_float(b), cb.centroid[b < ncode ? b : ncode - 1],
                              cb.centroid[b + 1 < ncode ? b + 1 : ncode - 1]);
    }
    // S' = S diag(D1) as bf16 high / low parts, canonical K-major (row i, k)
    for (int idx = tid; idx < m * (D / 2); idx += THREADS) {
        const int i = idx / (D / 2), k = 2 * (idx % (D / 2));
        float v0 = a.qjl_f32[(int64_t)i * D + k], v1 = a.qjl_f32[(int64_t)i * D + k + 1];
        if (!DENSE) {
            if ((sg.d1_bits[k >> 5] >> (k & 31)) & 1u) v0 = -v0;
            if ((sg.d1_bits[(k + 1) >> 5] >> ((k + 1) & 31)) & 1u) v1 = -v1;
        }
        uint32_t lo;
        const uint32_t hi = bf16x2_hi_lo(v0, v1, &lo);
        const uint32_t off = canon_elem(i, k, D);
        *reinterpret_cast<uint32_t *>(qs + C::OFF_B + off) = hi;
        *reinterpret_cast<uint32_t *>(qs + C::OFF_B + m * D * 2 + off) = lo;
    }
    if (tid == 0) {
        tc::mbar_init(s_mbar, 1);
        if (STAGED) {
            tc::mbar_init(s_full, 1);
            tc::mbar_init(s_full + 8, 1);
        }
        *abort_flag = 0;
    }
    if (warp == 0) tc::tmem_alloc((uint32_t)__cvta_generic_to_shared(tmem_holder), tcols);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const uint32_t idesc = tc::idesc_bf16_f32(TILE, m);
    // TMA copy of tile `t` into stage `stg` (STAGED only; one thread)
    auto issue_x = [&](int64_t t, int stg) {
        if (!STAGED || tid != 0 || t >= (a.n_rows + TILE - 1) / TILE) return;
        const uint32_t bar = s_full + 8u * stg;
        tc::mbar_arrive_expect_tx(bar, (uint32_t)C::X_STAGE);
#pragma unroll
        for (int h = 0; h < LPR; ++h)
            tc::tma_load_2d(qs_s + off_x + stg * C::X_STAGE + h * TILE * 128, &xmap, 64 * h,
                            (int32_t)(t * TILE), bar);
    };
    issue_x(blockIdx.x, 0);
    const unsigned char * tabb = reinterpret_cast<const unsigned char *>(tab4);
    const uint32_t slot = 16u * (uint32_t)(lane & 7);      // entry e, copy c at byte e * 128 + 16 c
    const SearchParams sp{st.scale, st.offset, st.mask};

    uint32_t mirror[2 * BITS];
#pragma unroll
    for (int k = 0; k < 2 * BITS; ++k) mirror[k] = 0u;
    if constexpr (!DENSE) {
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
            const uint32_t d1 = sg.d1_bits[2 * q + bb];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                place_field<BITS>(mirror + bb * BITS, j, ((d1 >> j) & 1u) ? FIELD : 0u);
        }
    }
    const float s1 = (q & 1) ? -1.0f : 1.0f;
    const float s2 = (q & 2) ? -1.0f : 1.0f;
    const float2 s1v = make_float2(s1, s1), s2v = make_float2(s2, s2);
    const float norm_scale = DENSE ? 1.0f : rsqrtf((float)D);
    constexpr int NB = D / 32;
    uint32_t status = 0u;

    const int64_t n_tiles = (a.n_rows + TILE - 1) / TILE;
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        const int64_t row = tile * TILE + trow;
        const bool valid = row < a.n_rows;
        // staged rows: this tile's copy has landed; the next tile's copy goes
        // into the other stage (its previous tile was finished at the last barrier)
        const unsigned char * xs = qs + off_x + (it & 1) * C::X_STAGE + trow * 128;
        if (STAGED) {
            if (!tc::mbar_wait(s_full + 8u * (it & 1), (it >> 1) & 1u, kQjlWaitNs)) {
                status |= TQ_STATUS_TIMEOUT;
                *abort_flag = 1;
            }
            issue_x(tile + gridDim.x, (int)((it + 1) & 1));
        }
        const int xkey = trow & 7;
        float2 z[32];
        if (valid) {
            if constexpr (DENSE) {
                float zf[64];
#pragma unroll
                for (int e = 0; e < 64; ++e) zf[e] = 0.0f;
                for (int i0 = 0; i0 < D; i0 += 8) {
                    float xv[8];
                    if constexpr (BF16) {
                        const uint4 u = STAGED
                            ? *reinterpret_cast<const uint4 *>(xs + (i0 >> 6) * (TILE * 128) + 16 * (((i0 & 63) >> 3) ^ xkey))
                            : ldg_nc_v4(static_cast<const uint16_t *>(a.x) + row * D + i0);
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
                        float acc = zf[e];
                        acc = fmaf(__uint_as_float(p0.x), xv[0], acc);
                        acc = fmaf(__uint_as_float(p0.y), xv[1], acc);
                        acc = fmaf(__uint_as_float(p0.z), xv[2], acc);
                        acc = fmaf(__uint_as_float(p0.w), xv[3], acc);
                        acc = fmaf(__uint_as_float(p1.x), xv[4], acc);
                        acc = fmaf(__uint_as_float(p1.y), xv[5], acc);
                        acc = fmaf(__uint_as_float(p1.z), xv[6], acc);
                        acc = fmaf(__uint_as_float(p1.w), xv[7], acc);
                        zf[e] = acc;
                    }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = make_float2(zf[2 * i], zf[2 * i + 1]);
            } else {
                if constexpr (BF16) {
                    const uint16_t * xr = static_cast<const uint16_t *>(a.x) + row * D;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float2 v[LPR][4];
#pragma unroll
                        for (int s = 0; s < LPR; ++s) {
                            const uint4 u = STAGED
                                ? *reinterpret_cast<const uint4 *>(xs + s * (TILE * 128) + 16 * (c ^ xkey))
                                : ldg_nc_v4(xr + s * 64 + c * 8);
                            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint32_t w = w4[k] ^ sg.d2_mask[(s * 64 + c * 8) / 2 + k];
                                v[s][k] = make_float2(bf16_lo(w), bf16_hi(w));
                            }
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if constexpr (LPR == 1) z[c * 4 + k] = v[0][k];
                            else if constexpr (LPR == 2) z[c * 4 + k] = __ffma2_rn(s1v, v[1][k], v[0][k]);
                            else z[c * 4 + k] = __ffma2_rn(s2v, __ffma2_rn(s1v, v[3][k], v[2][k]),
                                                           __ffma2_rn(s1v, v[1][k], v[0][k]));
                        }
                    }
                } else {
                    const float * xr = static_cast<const float *>(a.x) + row * D;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        float2 v[LPR][2];
#pragma unroll
                        for (int s = 0; s < LPR; ++s) {
                            const uint4 u = ldg_nc_v4(xr + s * 64 + c * 4);
                            const int e = s * 64 + c * 4;
                            v[s][0] = make_float2(__uint_as_float(u.x ^ sg.d2_mask[e]),
                                                  __uint_as_float(u.y ^ sg.d2_mask[e + 1]));
                            v[s][1] = make_float2(__uint_as_float(u.z ^ sg.d2_mask[e + 2]),
                                                  __uint_as_float(u.w ^ sg.d2_mask[e + 3]));
                        }
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            if constexpr (LPR == 1) z[c * 2 + k] = v[0][k];
                            else if constexpr (LPR == 2) z[c * 2 + k] = __ffma2_rn(s1v, v[1][k], v[0][k]);
                            else z[c * 2 + k] = __ffma2_rn(s2v, __ffma2_rn(s1v, v[3][k], v[2][k]),
                                                           __ffma2_rn(s1v, v[1][k], v[0][k]));
                        }
                    }
                }
                wht64x2(z);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = make_float2(0.0f, 0.0f);
        }

        // norms, codes, residual (in place of z), residual norm
        uint32_t words[2 * BITS];
        uint16_t nh[2];
        float rss = 0.0f;
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
            float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int jp = 0; jp < 16; ++jp) ss2 = __ffma2_rn(z[16 * bb + jp], z[16 * bb + jp], ss2);
            const float ss = ss2.x + ss2.y;
            const float g = sqrtf(ss);
            if (valid && !isfinite(ss)) status |= TQ_STATUS_NONFINITE;
            bool sat;
            nh[bb] = norm_to_half_bits(g * norm_scale, &sat);
            if (valid && sat) status |= TQ_STATUS_NORM_SATURATED;
            const float g16 = __half2float(__ushort_as_half(nh[bb]));
            uint32_t acc[BITS];
#pragma unroll
            for (int k = 0; k < BITS; ++k) acc[k] = 0u;
            const float inv = rsqrt_approx(ss);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float2 & zz = z[16 * bb + (j >> 1)];
                const float yv = (j & 1) ? zz.y : zz.x;
                const float u = yv * inv;
                const float4 e = *reinterpret_cast<const float4 *>(tabb + cell_offset(u, sp, slot));
                const bool up = u >= e.x;
                place_field<BITS>(acc, j, __float_as_uint(e.y) + (up ? 1u : 0u));
                // zero blocks store the middle code and a zero norm: residual = y = 0
                const float r = (g > 0.0f) ? fmaf(-g16, up ? e.w : e.z, yv * norm_scale) : 0.0f;
                rss = fmaf(r, r, rss);
                if (j & 1) zz.y = r; else zz.x = r;
            }
            if (g > 0.0f) {
#pragma unroll
                for (int k = 0; k < BITS; ++k) words[bb * BITS + k] = acc[k] ^ mirror[bb * BITS + k];
            } else {
#pragma unroll
                for (int k = 0; k < BITS; ++k) words[bb * BITS + k] = 0u;
#pragma unroll
                for (int j = 0; j < 32; ++j) place_field<BITS>(words + bb * BITS, j, 1u << (BITS - 1));
            }
        }
        if (valid) {
            store_words<2 * BITS>(a.codes + row * (NB * BITS) + q * 2 * BITS, words);
            *reinterpret_cast<uint32_t *>(a.norms + row * NB + 2 * q) =
                (uint32_t)nh[0] | ((uint32_t)nh[1] << 16);
        }
        // residual norm over the LPR lanes of the row
#pragma unroll
        for (int o = 1; o < LPR; o <<= 1) rss += __shfl_xor_sync(0xffffffffu, rss, o);
        if (valid && q == 0) {
            bool sat;
            a.qjl_rnorm[row] = norm_to_half_bits(sqrtf(rss), &sat);
            if (sat) status |= TQ_STATUS_NORM_SATURATED;
        }
        // residual tile: bf16 high / low parts, canonical K-major (row, k)
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) hi[t] = bf16x2_hi_lo(z[4 * kc + t].x, z[4 * kc + t].y, &lo[t]);
            const uint32_t off = canon_elem(trow, 64 * q + 8 * kc, D);
            *reinterpret_cast<uint4 *>(qs + C::OFF_AHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(qs + C::OFF_ALO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        tc::fence_proxy_async();
        __syncthreads();
        // z = S' r' for the 128 rows: hi*hi + hi*lo + lo*hi per 16-wide K step
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t SBO = (uint32_t)(D / 8) * 128u;
#pragma unroll 1
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t ko = (uint32_t)(256 * ks);
                const uint64_t ah = tc::smem_desc(s_ahi + ko, 128, SBO), al = tc::smem_desc(s_alo + ko, 128, SBO);
                const uint64_t bh = tc::smem_desc(s_bhi + ko, 128, SBO), bl = tc::smem_desc(s_blo + ko, 128, SBO);
                tc::mma_bf16(tmem, ah, bh, idesc, ks > 0 ? 1u : 0u);
                tc::mma_bf16(tmem, ah, bl, idesc, 1u);
                tc::mma_bf16(tmem, al, bh, idesc, 1u);
            }
            tc::commit(s_mbar);
        }
        if (!tc::mbar_wait(s_mbar, it & 1u, kQjlWaitNs)) {
            status |= TQ_STATUS_TIMEOUT;
            *abort_flag = 1;
        }
        tc::fence_after_sync();
        // signs: warp w reads TMEM lanes 32 (w % 4) .. + 31 (its tile rows) and
        // column group w / 4 of the m outputs, 32 columns per load
        {
            // column group w / 4 takes whole 32-column sign words
            const int quad = warp & 3, cgrp = warp >> 2;
            const int cw = 32 * ((m / 32 + LPR - 1) / LPR);
            const int64_t srow = tile * TILE + 32 * quad + lane;
            for (int c0 = cgrp * cw; c0 < (cgrp + 1) * cw && c0 < m; c0 += 32) {
                float v[32];
                tc::tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)c0, v);
                uint32_t bits = 0u;
#pragma unroll
                for (int j = 0; j < 32; ++j) bits |= (v[j] >= 0.0f ? 1u : 0u) << j;
                if (srow < a.n_rows && !*abort_flag) a.qjl_signs[srow * (m / 32) + c0 / 32] = bits;
            }
        }
        tc::fence_before_sync();
        __syncthreads();   // TMEM and the residual tile are rewritten next
        if (*abort_flag) break;
    }
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, tcols);
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

// ---------------------------------------------------------------------------
// Walsh-Hadamard quantize + QJL signs of bf16 rows with both products on the
// tensor cores (d = 64 or 128, m <= 128).  Per 128-row tile:
//  1. y = (D1 H D2) x: one tcgen05 GEMM, A = the x tile as its TMA boxes land,
//     into one of two TMEM accumulators;
//  2. epilogue 1 (warp w < 4 NB: TMEM lanes 32 (w % 4) .., block w / 4): norm,
//     codes, residual r = y / sqrt(d) - fp16(norm) c[code] in the rotated
//     frame, written as bf16 high / low parts straight into the 128-byte
//     swizzled K-major layout -- the high part over the x tile's own stage,
//     which the first GEMM has finished reading -- and the block's share of
//     |r|^2; the four warps of a row group add their shares through shared
//     memory (an mbarrier per row group, no CTA-wide barrier);
//  3. z = S r: hi*hi + hi*lo + lo*hi per 16-wide K step into a third
//     accumulator (products carry ~17 bits);
//  4. epilogue 2: each thread turns 32 columns of z into one word of signs.
// One thread of the last warp issues the copies and both GEMMs; the x tile of
// k + 2 is loaded once the second GEMM of tile k has read its stage.  Every
// wait is bounded.
// ---------------------------------------------------------------------------
template <int D>
struct QtCfg {
    static constexpr int NB = D / 32;
    static constexpr int EPI_WARPS = 4 * NB;
    static constexpr int THREADS = 32 * (EPI_WARPS + 1);
    static constexpr int ROWS = 128;
    static constexpr int SLICE = ROWS * 128;               // 64 K-columns of a 128-row tile
    static constexpr int X_STAGE = ROWS * D * 2;           // also the residual's high part
    static constexpr int MMAX = 128;                       // largest m
    static constexpr int OFF_RLO = 2 * X_STAGE;            // residual low part
    static constexpr int OFF_B = OFF_RLO + X_STAGE;        // D1 H D2 (bf16 +-1)
    static constexpr int OFF_S = OFF_B + D * D * 2;        // S high part, then low part (m x d)
    static constexpr int SMEM = 1024 + OFF_S + 2 * MMAX * D * 2;
    static constexpr uint32_t TCOLS = 512;                 // 2 D (y) + m (z) <= 384
    static_assert(D == 64 || D == 128, "tensor-core QJL path: d = 64 or 128");
};

template <int D, int BITS>
__global__ void __launch_bounds__(QtCfg<D>::THREADS, 1)
quantize_qjl_tc_kernel(const __grid_constant__ QuantizeArgs a, const __grid_constant__ SearchTable st,
                       const __grid_constant__ WhtKernelSigns sg, const __grid_constant__ CodebookParams cb,
                       const __grid_constant__ CUtensorMap xmap) {
    using C = QtCfg<D>;
    constexpr int NB = C::NB;
    extern __shared__ unsigned char qsm_raw[];
    // search table {t, base}: entry e, copy c at float2 e * 16 + c; centroid
    // of code k for lane l at k * 32 + l (both read without bank conflicts)
    __shared__ __align__(128) float2 s_qtab[kSearchMax * 16];
    __shared__ float s_cent[16 * 32];
    __shared__ float s_rss[2][C::ROWS][NB];                   // per-block shares of |r|^2
    // xfull[2], acc1 full[2] / empty[2], rfull, rfree, acc2 full / empty, row groups[4]
    __shared__ __align__(8) uint64_t s_bar[16];
    __shared__ uint32_t s_tmem;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m = a.qjl_m;
    const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(qsm_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    unsigned char * sm = qsm_raw + (base_s - raw_s);
    const uint32_t bar = (uint32_t)__cvta_generic_to_shared(s_bar);
    const uint32_t xfull_b = bar, a1f_b = bar + 16, a1e_b = bar + 32, rfull_b = bar + 48,
                   rfree_b = bar + 56, a2f_b = bar + 64, a2e_b = bar + 72, grp_b = bar + 80;

    for (uint32_t i = tid; i < st.size * 16; i += C::THREADS) {
        const uint32_t e = i >> 4;
        s_qtab[i] = make_float2(st.t[e], __int_as_float(st.base[e]));
    }
    for (int i = tid; i < 16 * 32; i += C::THREADS) s_cent[i] = cb.centroid[(i >> 5) < (1 << BITS) ? (i >> 5) : 0];
    // B[n][k] = d1_n (-1)^popc(n & k) d2_k; S[i][k] high / low parts; both
    // K-major, 64-column slices, 16-byte chunk ((k % 64) / 8) ^ (row % 8)
    for (int i = tid; i < D * (D / 8); i += C::THREADS) {
        const int n = i / (D / 8), kc = i % (D / 8);
        const uint32_t sn = (sg.d1_bits[n >> 5] >> (n & 31)) & 1u;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t pair = 0u;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int k = 8 * kc + 2 * e + h;
                const uint32_t sk = (sg.d2_mask[k >> 1] >> ((k & 1) ? 31 : 15)) & 1u;
                pair |= (((sn ^ sk ^ (uint32_t)__popc(n & k)) & 1u) ? 0xBF80u : 0x3F80u) << (16 * h);
            }
            w[e] = pair;
        }
        *reinterpret_cast<uint4 *>(sm + C::OFF_B + (kc >> 3) * (D * 128) + n * 128 + 16 * ((kc & 7) ^ (n & 7))) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int i = tid; i < m * (D / 8); i += C::THREADS) {
        const int n = i / (D / 8), kc = i % (D / 8);
        const int off = C::OFF_S + (kc >> 3) * (m * 128) + n * 128 + 16 * ((kc & 7) ^ (n & 7));
        *reinterpret_cast<uint4 *>(sm + off) = ldg_nc_v4(a.qjl_hi + (int64_t)n * D + 8 * kc);
        *reinterpret_cast<uint4 *>(sm + off + m * D * 2) = ldg_nc_v4(a.qjl_lo + (int64_t)n * D + 8 * kc);
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(xfull_b + 8u * i, 1);
            tc::mbar_init(a1f_b + 8u * i, 1);
            tc::mbar_init(a1e_b + 8u * i, C::EPI_WARPS);
        }
        tc::mbar_init(rfull_b, C::EPI_WARPS);
        tc::mbar_init(rfree_b, 1);
        tc::mbar_init(a2f_b, 1);
        tc::mbar_init(a2e_b, C::EPI_WARPS);
        for (int q = 0; q < 4; ++q) tc::mbar_init(grp_b + 8u * q, NB);
    }
    if (warp == C::EPI_WARPS) tc::tmem_alloc((uint32_t)__cvta_generic_to_shared(&s_tmem), C::TCOLS);
    tc::fence_proxy_async();             // B and S, written by generic stores, feed the MMAs
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s_tmem;
    const uint32_t z_col = 2 * D;        // z accumulator after the two y accumulators

    const int64_t n_tiles = (a.n_rows + C::ROWS - 1) / C::ROWS;
    const int64_t n_my = (int64_t)blockIdx.x < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    auto tile_of = [&](int64_t k) { return (int64_t)blockIdx.x + k * gridDim.x; };
    uint32_t status = 0u;

    if (warp == C::EPI_WARPS) {
        if (lane == 0) {
            const uint32_t id1 = tc::idesc_bf16_f32(C::ROWS, D), id2 = tc::idesc_bf16_f32(C::ROWS, m);
            auto issue = [&](int64_t j) {
                const uint32_t s = (uint32_t)(j & 1);
                tc::mbar_arrive_expect_tx(xfull_b + 8u * s, (uint32_t)C::X_STAGE);
#pragma unroll
                for (int h = 0; h < D / 64; ++h)
                    tc::tma_load_2d(base_s + s * C::X_STAGE + h * C::SLICE, &xmap, 64 * h,
                                    (int32_t)(tile_of(j) * C::ROWS), xfull_b + 8u * s);
            };
            int64_t issued = 0;
            for (; issued < n_my && issued < 2; ++issued) issue(issued);
            bool ok = true;
            // second GEMM of tile j (its residual is in place), then the next copy into its stage
            auto gemm2 = [&](int64_t j) {
                const uint32_t s = (uint32_t)(j & 1), ph = (uint32_t)(j & 1);
                if (!(tc::mbar_wait(rfull_b, ph, kQjlWaitNs) && tc::mbar_wait(a2e_b, ph ^ 1u, kQjlWaitNs)))
                    return false;
                tc::fence_after_sync();
                const uint32_t rh = base_s + s * C::X_STAGE, rl = base_s + C::OFF_RLO;
                const uint32_t sh = base_s + C::OFF_S, sl = sh + (uint32_t)(m * D * 2);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t ao = (uint32_t)((ks >> 2) * C::SLICE + (ks & 3) * 32);
                    const uint32_t bo = (uint32_t)((ks >> 2) * (m * 128) + (ks & 3) * 32);
                    const uint64_t ah = tc::smem_desc_sw128(rh + ao), al = tc::smem_desc_sw128(rl + ao);
                    const uint64_t bh = tc::smem_desc_sw128(sh + bo), bl = tc::smem_desc_sw128(sl + bo);
                    tc::mma_bf16(tmem + z_col, ah, bh, id2, ks > 0 ? 1u : 0u);
                    tc::mma_bf16(tmem + z_col, ah, bl, id2, 1u);
                    tc::mma_bf16(tmem + z_col, al, bh, id2, 1u);
                }
                tc::commit(a2f_b);
                tc::commit(rfree_b);
                if (issued < n_my) {
                    if (!tc::mbar_wait(rfree_b, ph, kQjlWaitNs)) return false;
                    issue(issued++);
                }
                return true;
            };
            int64_t k = 0;
            for (; k < n_my && ok; ++k) {
                const uint32_t s = (uint32_t)(k & 1), ph = (uint32_t)((k >> 1) & 1);
                ok = tc::mbar_wait(xfull_b + 8u * s, ph, kQjlWaitNs) &&
                     tc::mbar_wait(a1e_b + 8u * s, ph ^ 1u, kQjlWaitNs);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t x0 = base_s + s * C::X_STAGE, b0 = base_s + C::OFF_B;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc_sw128(x0 + (uint32_t)((ks >> 2) * C::SLICE + (ks & 3) * 32));
                    const uint64_t bd = tc::smem_desc_sw128(b0 + (uint32_t)((ks >> 2) * (D * 128) + (ks & 3) * 32));
                    tc::mma_bf16(tmem + s * D, ad, bd, id1, ks > 0 ? 1u : 0u);
                }
                tc::commit(a1f_b + 8u * s);
                if (k >= 1) ok = gemm2(k - 1);
            }
            if (ok && n_my > 0) ok = gemm2(n_my - 1);
            if (!ok) {
                status |= TQ_STATUS_TIMEOUT;
                // let copies still in flight land before the CTA exits
                for (int64_t j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j)
                    tc::mbar_wait(xfull_b + 8u * (uint32_t)(j & 1), (uint32_t)((j >> 1) & 1), kQjlWaitNs);
            }
        }
    } else {
        const int quad = warp & 3, blk = warp >> 2;
        const int r = 32 * quad + lane;                  // row within the tile
        const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
        const uint32_t slot = 8u * (uint32_t)(lane & 15);
        const unsigned char * tabb = reinterpret_cast<const unsigned char *>(s_qtab);
        const float * cent = s_cent + lane;
        const SearchParams sp{st.scale, st.offset, st.mask};
        const float norm_scale = rsqrtf((float)D);
        const float sqrt_d = sqrtf((float)D);
        bool ok = true;
        for (int64_t j = 0; j <= n_my && ok; ++j) {
            if (j < n_my) {
                // ---- epilogue 1: tile j ----
                const uint32_t s = (uint32_t)(j & 1);
                ok = __all_sync(0xffffffffu, tc::mbar_wait(a1f_b + 8u * s, (uint32_t)((j >> 1) & 1), kQjlWaitNs));
                if (!ok) break;
                tc::fence_after_sync();
                float y[32];
                tc::tmem_ld32(tmem + lane_addr + s * D + 32 * blk, y);
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(a1e_b + 8u * s);

                const int64_t row = tile_of(j) * C::ROWS + r;
                const bool valid = row < a.n_rows;
                float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 v = make_float2(y[2 * i], y[2 * i + 1]);
                    ss2 = __ffma2_rn(v, v, ss2);
                }
                const float ss = ss2.x + ss2.y;
                const float g = sqrt_approx(ss);
                if (valid && !isfinite(ss)) status |= TQ_STATUS_NONFINITE;
                bool sat;
                const uint16_t nh = norm_to_half_bits(g * norm_scale, &sat);
                if (valid && sat) status |= TQ_STATUS_NORM_SATURATED;
                // the residual is kept in units of 1/sqrt(d): r' = y - (fp16 norm
                // sqrt(d)) c = sqrt(d) r, whose projections have the signs of
                // those of r; |r| = |r'| / sqrt(d) (a zero block has y = 0 and a
                // zero norm, so r' = 0)
                const float gs = __half2float(__ushort_as_half(nh)) * sqrt_d;
                const float inv = rsqrt_approx(ss);
                uint32_t acc[BITS];
#pragma unroll
                for (int i = 0; i < BITS; ++i) acc[i] = 0u;
                float rss = 0.0f;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float u = y[e] * inv;
                    const float2 t = *reinterpret_cast<const float2 *>(tabb + cell_offset(u, sp, slot));
                    const uint32_t code = __float_as_uint(t.y) + (u >= t.x ? 1u : 0u);
                    place_field<BITS>(acc, e, code);
                    const float rv = fmaf(-gs, cent[32 * code], y[e]);
                    rss = fmaf(rv, rv, rss);
                    y[e] = rv;
                }
                if (!(g > 0.0f)) {
#pragma unroll
                    for (int i = 0; i < BITS; ++i) acc[i] = 0u;
#pragma unroll
                    for (int e = 0; e < 32; ++e) place_field<BITS>(acc, e, 1u << (BITS - 1));
                }
                if (valid) {
                    uint32_t * dst = a.codes + row * (NB * BITS) + blk * BITS;
                    if constexpr (BITS == 4) *reinterpret_cast<uint4 *>(dst) = make_uint4(acc[0], acc[1], acc[2], acc[3]);
                    else if constexpr (BITS == 2) *reinterpret_cast<uint2 *>(dst) = make_uint2(acc[0], acc[1]);
                    else {
#pragma unroll
                        for (int i = 0; i < BITS; ++i) dst[i] = acc[i];
                    }
                    a.norms[row * NB + blk] = nh;
                }
                s_rss[s][r][blk] = rss;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(grp_b + 8u * quad);
                // the residual's low part reuses one buffer: the previous tile's
                // second GEMM must have read it
                if (j >= 1) {
                    ok = __all_sync(0xffffffffu, tc::mbar_wait(rfree_b, (uint32_t)((j - 1) & 1), kQjlWaitNs));
                    if (!ok) break;
                }
                unsigned char * rh = sm + s * C::X_STAGE;
                unsigned char * rl = sm + C::OFF_RLO;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) hi[t] = bf16x2_hi_lo(y[8 * c + 2 * t], y[8 * c + 2 * t + 1], &lo[t]);
                    const int kc = 4 * blk + c;
                    const int off = (kc >> 3) * C::SLICE + r * 128 + 16 * ((kc & 7) ^ (r & 7));
                    *reinterpret_cast<uint4 *>(rh + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(rl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
                tc::fence_proxy_async();          // the second GEMM reads through the async proxy
                if (blk == 0) {
                    // residual norm of the row: the four blocks' shares
                    ok = __all_sync(0xffffffffu, tc::mbar_wait(grp_b + 8u * quad, (uint32_t)(j & 1), kQjlWaitNs));
                    if (ok && valid) {
                        float t2 = 0.0f;
#pragma unroll
                        for (int b2 = 0; b2 < NB; ++b2) t2 += s_rss[s][r][b2];
                        bool sat2;
                        a.qjl_rnorm[row] = norm_to_half_bits(sqrtf(t2) * norm_scale, &sat2);
                        if (sat2) status |= TQ_STATUS_NORM_SATURATED;
                    }
                    if (!ok) break;
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(rfull_b);
            }
            if (j >= 1) {
                // ---- epilogue 2: signs of tile j - 1 ----
                const int64_t jj = j - 1;
                ok = __all_sync(0xffffffffu, tc::mbar_wait(a2f_b, (uint32_t)(jj & 1), kQjlWaitNs));
                if (!ok) break;
                tc::fence_after_sync();
                const int64_t row = tile_of(jj) * C::ROWS + r;
                for (int grp = blk; grp < m / 32; grp += NB) {
                    float z[32];
                    tc::tmem_ld32(tmem + lane_addr + z_col + 32 * grp, z);
                    // bit e = [z_e >= 0]: the sign bits of z_e + 0 (which turns -0
                    // into +0) shifted in by funnel shifts, in four independent
                    // chains of eight, then inverted
                    uint32_t part[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int i = 7; i >= 0; --i)
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            part[c] = __funnelshift_l(__float_as_uint(z[8 * c + i] + 0.0f), part[c], 1);
                    const uint32_t neg = __byte_perm(__byte_perm(part[0], part[1], 0x0040u),
                                                     __byte_perm(part[2], part[3], 0x0040u), 0x5410u);
                    if (row < a.n_rows) a.qjl_signs[row * (m / 32) + grp] = ~neg;
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(a2e_b);
            }
        }
        if (!ok) status |= TQ_STATUS_TIMEOUT;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == C::EPI_WARPS) tc::tmem_dealloc(tmem, C::TCOLS);
    if (status != 0u && a.status != nullptr) atomicOr(a.status, status);
}

template <int D, int BITS>
int launch_qjl_tc_t(const tq_rotation * rot, const SearchTable & tabp, const CodebookParams & cb,
                    const QuantizeArgs & a, cudaStream_t st) {
    using C = QtCfg<D>;
    WhtKernelSigns sg{};
    for (int i = 0; i < 8; ++i) sg.d1_bits[i] = rot->d1_bits[i];
    for (int i = 0; i < D; ++i) {
        const uint32_t neg = (rot->d2_bits[i >> 5] >> (i & 31)) & 1u;
        sg.d2_mask[i >> 1] |= neg << ((i & 1) ? 31 : 15);
    }
    const int64_t n_tiles = (a.n_rows + C::ROWS - 1) / C::ROWS;
    if (n_tiles == 0) return 0;
    CUtensorMap xmap;
    if (!encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)D, (uint64_t)a.n_rows,
                              (uint64_t)D * 2, 64u, (uint32_t)C::ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return (int)cudaErrorInvalidValue;
    auto k = quantize_qjl_tc_kernel<D, BITS>;
    // one CTA per SM (each holds all 512 TMEM columns): ask for enough shared
    // memory that a second one never fits
    const int smem = C::SMEM > 120 * 1024 ? C::SMEM : 120 * 1024;
    if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return e;
    int64_t grid = device_sm_count();
    if (grid > n_tiles) grid = n_tiles;
    k<<<(unsigned)grid, C::THREADS, smem, st>>>(a, tabp, sg, cb, xmap);
    return (int)cudaGetLastError();
}

template <int D, int BITS, bool BF16, bool DENSE>
int launch_qjl_t(const tq_rotation * rot, const SearchTable & tabp, const CodebookParams & cb,
                 const QuantizeArgs & a, cudaStream_t st) {
    using C = QjlCfg<D>;
    WhtKernelSigns sg{};
    for (int i = 0; i < 8; ++i) sg.d1_bits[i] = rot->d1_bits[i];
    for (int i = 0; i < D; ++i) {
        const uint32_t neg = (rot->d2_bits[i >> 5] >> (i & 31)) & 1u;
        if (BF16) sg.d2_mask[i >> 1] |= neg << ((i & 1) ? 31 : 15);
        else sg.d2_mask[i] = neg << 31;
    }
    auto k = quantize_qjl_kernel<D, BITS, BF16, DENSE>;
    constexpr bool staged = BF16 && C::STAGED_D;
    const size_t smem = (size_t)C::smem_bytes(a.qjl_m, staged);
    CUtensorMap xmap;
    memset(&xmap, 0, sizeof(xmap));
    if (staged && !encode_tensor_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)D,
                                        (uint64_t)a.n_rows, (uint64_t)D * 2, 64u, (uint32_t)C::TILE,
                                        CU_TENSOR_MAP_SWIZZLE_128B))
        return (int)cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, C::THREADS, smem);
    if (per_sm < 1) per_sm = 1;
    // each resident CTA holds a TMEM allocation of up to 256 columns
    if (per_sm > 2) per_sm = 2;
    int64_t grid = (int64_t)per_sm * device_sm_count();
    const int64_t need = (a.n_rows + C::TILE - 1) / C::TILE;
    if (grid > need) grid = need;
    k<<<(unsigned)grid, C::THREADS, smem, st>>>(a, tabp, sg, cb, xmap);
    return (int)cudaGetLastError();
}

template <int D, int BITS>
int qjl_dtype(const tq_rotation * rot, bool bf16, const SearchTable & tabp,
              const CodebookParams & cb, const QuantizeArgs & a, cudaStream_t st) {
    const bool dense = rot->kind != TQ_ROT_WHT;
    if constexpr (D <= 128) {
        if (bf16 && !dense && a.qjl_m % 32 == 0 && a.qjl_m <= QtCfg<D>::MMAX && a.qjl_hi != nullptr &&
            a.qjl_lo != nullptr)
            return launch_qjl_tc_t<D, BITS>(rot, tabp, cb, a, st);
    }
    if (bf16) return dense ? launch_qjl_t<D, BITS, true, true>(rot, tabp, cb, a, st)
                           : launch_qjl_t<D, BITS, true, false>(rot, tabp, cb, a, st);
    return dense ? launch_qjl_t<D, BITS, false, true>(rot, tabp, cb, a, st)
                 : launch_qjl_t<D, BITS, false, false>(rot, tabp, cb, a, st);
}

template <int D>
int qjl_bits(const tq_rotation * rot, int bits, bool bf16, const SearchTable & tabp,
             const CodebookParams & cb, const QuantizeArgs & a, cudaStream_t st) {
    switch (bits) {
        case 2: return qjl_dtype<D, 2>(rot, bf16, tabp, cb, a, st);
        case 3: return qjl_dtype<D, 3>(rot, bf16, tabp, cb, a, st);
        case 4: return qjl_dtype<D, 4>(rot, bf16, tabp, cb, a, st);
    }
    return (int)cudaErrorInvalidValue;
}

template <typename K>
int grid_for(K kernel, int threads, size_t smem) {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (per_sm < 1) per_sm = 1;
    return per_sm * device_sm_count();
}





// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void * p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cudaGetLastError();
    });
    return fn;
}


template <int D, int BITS, bool DENSE, bool GROUPED = false>
int launch_rot_tc_t(const WhtKernelSigns & sg, const SearchTable & tabp, const QuantizeArgs & a,
                    cudaStream_t st) {
    if constexpr (!GROUPED) {
        // lane-grouped rows: d = 128 only (the caller checks)
        if (a.grouped) {
            if constexpr (D == 128) return launch_rot_tc_t<D, BITS, DENSE, true>(sg, tabp, a, st);
            return (int)cudaErrorInvalidValue;
        }
    }
    using C = WtCfg<D, BITS, DENSE>;
    auto k = quantize_rot_tc_kernel<D, BITS, DENSE, GROUPED>;
    const int64_t n_tiles = (a.n_rows + kWtRows - 1) / kWtRows;
    if (n_tiles == 0) return 0;
    // [n_rows][D] bf16, boxes of 64 columns x 128 rows, 128-byte swizzle
    CUtensorMap tmap;
    if (!encode_tensor_map_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)D,
                              (uint64_t)a.n_rows, (uint64_t)D * 2, 64u, (uint32_t)kWtRows,
                              CU_TENSOR_MAP_SWIZZLE_128B))
        return (int)cudaErrorInvalidValue;
    if (int e = ensure_dynamic_smem(reinterpret_cast<const void *>(k), C::SMEM)) return e;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, C::THREADS, (size_t)C::SMEM);
    if (per_sm < 1) per_sm = 1;
    if (per_sm * C::TCOLS > 512u) per_sm = (int)(512u / C::TCOLS);   // TMEM columns per SM
    // CTA pairs at d = 256 (one per output half of the same tiles)
    int64_t pairs = (int64_t)per_sm * device_sm_count() / C::NH;
    if (pairs > n_tiles) pairs = n_tiles;
    if (pairs < 1) pairs = 1;
    k<<<(unsigned)(pairs * C::NH), C::THREADS, C::SMEM, st>>>(a, tabp, sg, tmap);
    return (int)cudaGetLastError();
}

template <int D, int BITS, bool BF16>
int launch_wht_t(const tq_rotation * rot, const SearchTable & tabp, const QuantizeArgs & a,
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
    if constexpr (BF16) {
        return launch_rot_tc_t<D, BITS, false>(sg, tabp, a, st);
    }
    auto k = quantize_wht_kernel<D, BITS, BF16>;
    const int threads = 256;
    const size_t smem = (size_t)tabp.size * 16 * sizeof(float2);
    const int64_t rows_per_cta = (int64_t)(threads / 32) * (32 / (D / 64));
    int64_t grid = grid_for(k, threads, smem);
    const int64_t need = (a.n_rows + rows_per_cta - 1) / rows_per_cta;
    if (grid > need) grid = need;
    k<<<(unsigned)grid, threads, smem, st>>>(a, tabp, sg);
    return (int)cudaGetLastError();
}

template <int D, int BITS, bool BF16>
int launch_dense_t(const SearchTable & tabp, const QuantizeArgs & a, cudaStream_t st) {
    auto k = quantize_dense_simple_kernel<D, BITS, BF16>;
    const int threads = 256;
    const size_t smem = (size_t)tabp.size * 16 * sizeof(float2);
    const int64_t rows_per_cta = (int64_t)(threads / 32) * (32 / (D / 64));
    int64_t grid = grid_for(k, threads, smem);
    const int64_t need = (a.n_rows + rows_per_cta - 1) / rows_per_cta;
    if (grid > need) grid = need;
    k<<<(unsigned)grid, threads, smem, st>>>(a, tabp);
    return (int)cudaGetLastError();
}

// Format variants (norm block 32 / 64 / 128, fp32 norms, norm correction):
// the register kernels with the variant epilogue, for either rotation.
template <int D, int BITS, bool BF16, int BLOCK>
int launch_var_t(const tq_rotation * rot, const SearchTable & tabp, const QuantizeArgs & a,
                 cudaStream_t st) {
    const int threads = 256;
    const size_t smem = (size_t)tabp.size * 16 * sizeof(float2) + 32 * sizeof(float);
    const int64_t rows_per_cta = (int64_t)(threads / 32) * (32 / (D / 64));
    const int64_t need = (a.n_rows + rows_per_cta - 1) / rows_per_cta;
    if (rot->kind == TQ_ROT_WHT) {
        WhtKernelSigns sg{};
        for (int i = 0; i < 8; ++i) sg.d1_bits[i] = rot->d1_bits[i];
        for (int i = 0; i < D; ++i) {
            const uint32_t neg = (rot->d2_bits[i >> 5] >> (i & 31)) & 1u;
            if (BF16) sg.d2_mask[i >> 1] |= neg << ((i & 1) ? 31 : 15);
            else sg.d2_mask[i] = neg << 31;
        }
        auto k = quantize_wht_kernel<D, BITS, BF16, true, BLOCK>;
        int64_t grid = grid_for(k, threads, smem);
        if (grid > need) grid = need;
        k<<<(unsigned)grid, threads, smem, st>>>(a, tabp, sg);
    } else {
        auto k = quantize_dense_simple_kernel<D, BITS, BF16, true, BLOCK>;
        int64_t grid = grid_for(k, threads, smem);
        if (grid > need) grid = need;
        k<<<(unsigned)grid, threads, smem, st>>>(a, tabp);
    }
    return (int)cudaGetLastError();
}

template <int D, int BITS>
int var_block(const tq_rotation * rot, bool bf16, const SearchTable & tabp, const QuantizeArgs & a,
              cudaStream_t st) {
    switch (a.norm_block) {
        case 32: return bf16 ? launch_var_t<D, BITS, true, 32>(rot, tabp, a, st)
                             : launch_var_t<D, BITS, false, 32>(rot, tabp, a, st);
        case 64: return bf16 ? launch_var_t<D, BITS, true, 64>(rot, tabp, a, st)
                             : launch_var_t<D, BITS, false, 64>(rot, tabp, a, st);
        case 128:
            if constexpr (D >= 128)
                return bf16 ? launch_var_t<D, BITS, true, 128>(rot, tabp, a, st)
                            : launch_var_t<D, BITS, false, 128>(rot, tabp, a, st);
            return (int)cudaErrorInvalidValue;
    }
    return (int)cudaErrorInvalidValue;
}

template <int D>
int var_bits(const tq_rotation * rot, int bits, bool bf16, const SearchTable & tabp,
             const QuantizeArgs & a, cudaStream_t st) {
    switch (bits) {
        case 2: return var_block<D, 2>(rot, bf16, tabp, a, st);
        case 3: return var_block<D, 3>(rot, bf16, tabp, a, st);
        case 4: return var_block<D, 4>(rot, bf16, tabp, a, st);
    }
    return (int)cudaErrorInvalidValue;
}

template <int D, int BITS>
int dispatch_dtype(const tq_rotation * rot, bool bf16, const SearchTable & tabp,
                   const QuantizeArgs & a, cudaStream_t st) {
    if (rot->kind == TQ_ROT_WHT)
        return bf16 ? launch_wht_t<D, BITS, true>(rot, tabp, a, st)
                    : launch_wht_t<D, BITS, false>(rot, tabp, a, st);
    if (bf16) return launch_rot_tc_t<D, BITS, true>(WhtKernelSigns{}, tabp, a, st);
    return bf16 ? launch_dense_t<D, BITS, true>(tabp, a, st)
                : launch_dense_t<D, BITS, false>(tabp, a, st);
}

template <int D>
int dispatch_bits(const tq_rotation * rot, int bits, bool bf16, const SearchTable & tabp,
                  const QuantizeArgs & a, cudaStream_t st) {
    switch (bits) {
        case 2: return dispatch_dtype<D, 2>(rot, bf16, tabp, a, st);
        case 3: return dispatch_dtype<D, 3>(rot, bf16, tabp, a, st);
        case 4: return dispatch_dtype<D, 4>(rot, bf16, tabp, a, st);
    }
    return (int)cudaErrorInvalidValue;
}

}  // namespace

bool encode_tensor_map_2d(CUtensorMap * map, CUtensorMapDataType dtype, const void * base,
                          uint64_t inner, uint64_t outer, uint64_t stride, uint32_t box_inner,
                          uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    const cuuint64_t gstride[1] = {(cuuint64_t)stride};
    const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
    const cuuint32_t estride[2] = {1u, 1u};
    return enc(map, dtype, 2, const_cast<void *>(base), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_quantize(const tq_rotation * rot, const tq_rotation * qjl, int bits, bool bf16,
                    int head_dim, const CodebookParams & cb, const SearchTable & tabp,
                    const QuantizeArgs & a, void * stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (qjl != nullptr) {
        switch (head_dim) {
            case 64: return qjl_bits<64>(rot, bits, bf16, tabp, cb, a, st);
            case 128: return qjl_bits<128>(rot, bits, bf16, tabp, cb, a, st);
            case 256: return qjl_bits<256>(rot, bits, bf16, tabp, cb, a, st);
        }
        return (int)cudaErrorInvalidValue;
    }
    if (a.norm_block != 32 || a.norm_f32 || a.norm_corr) {
        switch (head_dim) {
            case 64: return var_bits<64>(rot, bits, bf16, tabp, a, st);
            case 128: return var_bits<128>(rot, bits, bf16, tabp, a, st);
            case 256: return var_bits<256>(rot, bits, bf16, tabp, a, st);
        }
        return (int)cudaErrorInvalidValue;
    }
    switch (head_dim) {
        case 64: return dispatch_bits<64>(rot, bits, bf16, tabp, a, st);
        case 128: return dispatch_bits<128>(rot, bits, bf16, tabp, a, st);
        case 256: return dispatch_bits<256>(rot, bits, bf16, tabp, a, st);
    }
    return (int)cudaErrorInvalidValue;
}

}  // namespace tq
