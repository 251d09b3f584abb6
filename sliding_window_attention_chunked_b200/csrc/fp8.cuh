// fp8.cuh -- OCP E4M3 codes for the FP8 window cache (SALA blog §4.3: the KV cache stored in
// FP8). One fp32 scale per cache: a stored code is the nearest E4M3 value to x / scale (the
// quotient in fp32, ties to even, magnitudes past 448 saturated), and reads multiply the code's
// value by the scale. The conversions are the hardware's (cvt with .satfinite / to f16).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "common.cuh"

namespace rod {

// two E4M3 codes (low byte first) -> an f16 pair (exact)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}
// 16 bf16 values (two uint4, in order) as 16 E4M3 codes of x / scale (the quotient in fp32, the
// nearest code, ties to even, saturated), the first value in the lowest byte
__device__ __forceinline__ uint4 quantize16(uint4 a, uint4 b, float scale) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 p0 = make_float2(__fdiv_rn(bf16lo(w[2 * i]), scale), __fdiv_rn(bf16hi(w[2 * i]), scale));
        const float2 p1 = make_float2(__fdiv_rn(bf16lo(w[2 * i + 1]), scale), __fdiv_rn(bf16hi(w[2 * i + 1]), scale));
        const uint32_t c0 = __nv_cvt_float2_to_fp8x2(p0, __NV_SATFINITE, __NV_E4M3);
        const uint32_t c1 = __nv_cvt_float2_to_fp8x2(p1, __NV_SATFINITE, __NV_E4M3);
        out[i] = (c0 & 0xffffu) | (c1 << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace rod
