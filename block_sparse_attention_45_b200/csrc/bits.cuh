// bits.cuh -- small fp32 helpers shared by the exact top-p selections (the
// per-row cut of mask.cu and the pooled cut of eg.cu): both bin scores >= 0 by
// their fp32 bit patterns and keep exact integer sums of the significands.
#pragma once

#include <stdint.h>

namespace bsa {

// The 24-bit significand of a non-negative fp32 pattern (the implicit leading
// bit included for normal numbers).
__device__ __forceinline__ uint32_t significand(uint32_t u) {
    return (u & 0x7FFFFFu) | ((u >> 23) ? 0x800000u : 0u);
}

// 2^(max(e, 1) - 150): the weight of one significand unit in binade e.
__device__ __forceinline__ double unit_of_binade(uint32_t e) {
    const int k = static_cast<int>(e > 1u ? e : 1u) - 150;
    return __longlong_as_double(static_cast<long long>(k + 1023) << 52);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// log2 on the special-function unit (approximate; the entropies only).
__device__ __forceinline__ float lg2_approx(float y) {
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

}  // namespace bsa
