// sscan_complex_math.cuh -- device helpers of the complex-A scan: cosine and sine
// of an angle of any size on the MUFU pipe (sin.approx / cos.approx after
// reduction to [-pi, pi] with a two-part 2 pi).
#pragma once

namespace sscan {
namespace cplx {

constexpr float kTwoPiHi = 6.28318548202514648f;   // fp32 nearest to 2 pi
constexpr float kTwoPiLo = -1.7484556e-7f;         // 2 pi - kTwoPiHi
constexpr float kInvTwoPi = 0.159154943091895336f;

__device__ __forceinline__ float sin_approx(float x) {
    float y;
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float cos_approx(float x) {
    float y;
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Nearest integer to p on the FMA pipe (rintf is a conversion, which runs on the
// MUFU/XU pipe the exponentials, sines and cosines already keep busy): adding 1.5 * 2^23
// leaves no fraction bits for |p| < 2^22, so the sum is rounded to an integer (ties to
// even, as rintf) and subtracting the constant again is exact.  __fadd_rn keeps the
// compiler from contracting the additions into an fma with the product that forms p.
// Beyond |p| = 2^22 the sum keeps no fraction bit and the turn count is not the nearest
// integer (for -2^23 < p <= -2^22 it may be off by half a turn); such an angle exceeds
// 2.6e7 rad, where the fp32 angle itself carries an error of a radian or more, so no
// reduction could give its sine.  (A clamp of p to 2^22 cost 5% of the complex forward.)
__device__ __forceinline__ float round_fma(float p) {
    constexpr float kShift = 12582912.f;  // 1.5 * 2^23
    return __fadd_rn(__fadd_rn(p, kShift), -kShift);
}

// round_fma for two values with packed adds.
__device__ __forceinline__ float2 round2_fma(float2 p) {
    constexpr float kShift = 12582912.f;
    return __fadd2_rn(__fadd2_rn(p, make_float2(kShift, kShift)), make_float2(-kShift, -kShift));
}

// cos and sin of an angle of any size: reduce by a multiple of 2 pi first.
__device__ __forceinline__ float2 cis(float th) {
    const float k = round_fma(th * kInvTwoPi);
    float r = fmaf(-k, kTwoPiHi, th);
    r = fmaf(-k, kTwoPiLo, r);
    return make_float2(cos_approx(r), sin_approx(r));
}

}  // namespace cplx
}  // namespace sscan
