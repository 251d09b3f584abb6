// exp2x2.cuh -- two-wide fp32 arithmetic and 2^x for pairs of values, on the SFU or on the FMA
// pipe. The attention kernels' softmax needs one exponential per score; the SFU retires 16 per
// clock per SM, which for head dim 128 is as much time as the tensor core spends on the tile, so
// part of the exponentials go to the FMA pipe instead.
#pragma once

#include <stdint.h>

#include "tc.cuh"

namespace rod {
namespace fx {

// two-wide fp32 fma / add / sub / mul (one instruction for both lanes of the pair)
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 f2add(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 f2sub(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 2^x for both lanes on the SFU
__device__ __forceinline__ float2 ex2x2_sfu(float2 x) { return make_float2(tc::ex2(x.x), tc::ex2(x.y)); }

// 2^x for both lanes on the FMA pipe, for x <= 0. Range reduction: adding 1.5 * 2^23 rounds x
// to the nearest integer n (held in the low mantissa bits of the sum), and f = x - n lies in
// [-1/2, 1/2]. 2^f is the minimax cubic for relative error on that interval (Lawson's algorithm,
// fit_exp2_cubic.py beside this file prints these constants): at most 7.5e-5 relative, below the
// bf16 rounding the probabilities get. 2^n is added into the exponent field. Inputs are clamped
// at -125 so the exponent stays normal: masked (-inf) scores give 2^-125.
constexpr float kExpC0 = 0.9999280571937561f;
constexpr float kExpC1 = 0.6932609677314758f;
constexpr float kExpC2 = 0.24261116981506348f;
constexpr float kExpC3 = 0.0551716648042202f;
__device__ __forceinline__ float2 ex2x2_fma(float2 x) {
    x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
    const float2 shifter = make_float2(12582912.f, 12582912.f);
    const float2 j = f2add(x, shifter);
    const float2 fr = f2sub(x, f2sub(j, shifter));
    float2 q = f2fma(make_float2(kExpC3, kExpC3), fr, make_float2(kExpC2, kExpC2));
    q = f2fma(q, fr, make_float2(kExpC1, kExpC1));
    q = f2fma(q, fr, make_float2(kExpC0, kExpC0));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(j.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(j.y) << 23)));
}

}  // namespace fx
}  // namespace rod
