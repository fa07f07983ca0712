// Scale arithmetic of the INT8 quantiser shared by the K/V append and the weight quantiser
// (fluxbbs.com "单卡 4090 怎么做到的", first technique: INT8 storage with float scale factors; the
// formula is this library's reading, stated in nomas.h): s = RN(absmax / 127), codes rint(x / s).
#pragma once

#include "common.cuh"

namespace nomas {

// s = RN(a / 127) for a = absmax of bf16 values, without the division routine: q0 = RN(a c) with
// c = RN(1/127), the remainder a - 127 q0 is exact by FMA, and s = RN(q0 + (a - 127 q0) c) is
// Markstein's correction step ("Computation of elementary functions on the IBM RISC System/6000
// processor", 1990).  Checked by exact rational arithmetic against RN(a / 127) for every bf16 a in
// [2^-110, max finite], where q0 and s are normals and the remainder (a subnormal at the low end) is
// exact; zero gives zero, and subnormal or non-finite a take the IEEE division.
__device__ __forceinline__ float div127(float a) {
    constexpr float c = 0x1.020408p-7f;                   // RN(1/127)
    const float q0 = __fmul_rn(a, c);
    const float s = __fmaf_rn(__fmaf_rn(-q0, 127.0f, a), c, q0);
    if (!(a >= 0x1p-110f && a <= 0x1.fffffep127f) && a != 0.0f) return __fdiv_rn(a, 127.0f);
    return s;
}

// 1/s for normal s: the hardware approximation (PTX rcp.approx.f32, relative error about 2^-23)
// refined by one Newton-Raphson step r = r0 + r0 (1 - s r0), both by FMA, leaves a relative error
// below 2^-24 + 2^-40.
__device__ __forceinline__ float recip_nr(float s) {
    float r0;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r0) : "f"(s));
    return __fmaf_rn(r0, __fmaf_rn(-s, r0, 1.0f), r0);
}

// Code rint(RN(x / s)) (half-even) of one value, given s > 0 and r = recip_nr(s) (a NaN for s below
// 2^-125).  t = RN(x r + 1.5 * 2^23) holds the integer q nearest x r; when d = RN(x r - q) is farther
// than 2^-15 from a half, rint(RN(x / s)) = q (the argument is stated with the append kernel's quant16);
// otherwise the exact quotient decides.
__device__ __forceinline__ int code_of(float x, float s, float r) {
    constexpr float kMagic = 12582912.0f;                 // 1.5 * 2^23
    constexpr float kFar = 0.5f - 0x1p-15f;
    const float t = __fmaf_rn(x, r, kMagic);
    const float q = __fsub_rn(t, kMagic);
    const float d = __fmaf_rn(x, r, -q);
    if (fabsf(d) < kFar) return (int)q;
    return (int)rintf(__fdiv_rn(x, s));
}

}  // namespace nomas
