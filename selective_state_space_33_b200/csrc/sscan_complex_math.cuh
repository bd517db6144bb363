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

// cos and sin of an angle of any size: reduce by a multiple of 2 pi first.
__device__ __forceinline__ float2 cis(float th) {
    const float k = rintf(th * kInvTwoPi);
    float r = fmaf(-k, kTwoPiHi, th);
    r = fmaf(-k, kTwoPiLo, r);
    return make_float2(cos_approx(r), sin_approx(r));
}

}  // namespace cplx
}  // namespace sscan
