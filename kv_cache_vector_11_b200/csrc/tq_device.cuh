// Device helpers shared by the TurboQuant kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "tq_internal.h"

namespace tq {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

// fp16 bits of a non-negative norm, round to nearest even, saturating at 65504.
__device__ __forceinline__ uint16_t norm_to_half_bits(float v, bool * saturated) {
    *saturated = v > 65504.0f;
    float c = fminf(v, 65504.0f);
    return __half_as_ushort(__float2half_rn(c));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void * p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Number of positive boundaries at or below a = |y| (the magnitude rank),
// by branch-free binary search over thresholds T[k] = gamma * t_pos[k].
template <int BITS>
__device__ __forceinline__ uint32_t magnitude_rank(float a, const float * T) {
    if constexpr (BITS == 1) {
        return 0u;
    } else if constexpr (BITS == 2) {
        return a >= T[0] ? 1u : 0u;
    } else if constexpr (BITS == 3) {
        const bool p1 = a >= T[1];
        const float t0 = p1 ? T[2] : T[0];
        const bool p0 = a >= t0;
        return (p1 ? 2u : 0u) + (p0 ? 1u : 0u);
    } else {
        const bool p2 = a >= T[3];
        const float t1 = p2 ? T[5] : T[1];
        const bool p1 = a >= t1;
        const float ta = p1 ? T[2] : T[0];
        const float tb = p1 ? T[6] : T[4];
        const bool p0 = a >= (p2 ? tb : ta);
        return (p2 ? 4u : 0u) + (p1 ? 2u : 0u) + (p0 ? 1u : 0u);
    }
}

// Code j of a block: bit position j*BITS of the block's little-endian stream.
template <int BITS>
__device__ __forceinline__ uint32_t extract_code(const uint32_t * words, int j) {
    const int p = j * BITS;
    const int wi = p >> 5, sh = p & 31;
    uint32_t v = words[wi] >> sh;
    if (sh + BITS > 32) v |= words[wi + 1] << (32 - sh);
    return v & ((1u << BITS) - 1u);
}

}  // namespace tq
