// w4_half.cuh -- 16-bit float helpers shared by the elementwise kernels:
// exact widening of eight fp16/bf16 values held in one 16-byte word, and
// round-to-nearest-even narrowing of fp32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "w4a16.h"

namespace w4 {

// Eight 16-bit floats of one 16-byte word, widened exactly to fp32.
template <int XT>
__device__ __forceinline__ void widen8(const uint4 v, float f[8]) {
    const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (XT == W4_F16) {
            const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&r[i]));
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        } else {
            f[2 * i] = __uint_as_float(r[i] << 16);
            f[2 * i + 1] = __uint_as_float(r[i] & 0xFFFF0000u);
        }
    }
}

template <int XT>
__device__ __forceinline__ float widen1(uint16_t h) {
    if (XT == W4_F16) return __half2float(__ushort_as_half(h));
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// fp32 -> 16-bit, round to nearest even.
template <int XT>
__device__ __forceinline__ uint16_t narrow1(float x) {
    if (XT == W4_F16) return __half_as_ushort(__float2half_rn(x));
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

}  // namespace w4
