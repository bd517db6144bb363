// sscan_act.cuh -- the activations of the scan's input stage for two values at
// once (sec. 3.2: delta passes through softplus; Fig. 3: SiLU on the gate branch and,
// optionally, on the input branch): exponentials, logarithm and reciprocal on the MUFU
// pipe, the surrounding arithmetic packed f32x2.
#pragma once

#include "sscan_math.cuh"
#include "sscan_tma.cuh"

namespace sscan {

// softplus and SiLU of two values at once: the exponentials, logarithm and
// reciprocal stay on the MUFU pipe, the surrounding arithmetic is packed f32x2.
// softplus(r) = log(1 + e^r) in the same three regions as sscan::softplus
// (r > 20: r; e^r < 2^-5: the log1p series; else ln2 * log2(1 + e^r)).
__device__ __forceinline__ float2 softplus_x2(float2 r) {
    const float2 q = __fmul2_rn(r, f2(kLog2e, kLog2e));
    const float2 u = f2(ex2(q.x), ex2(q.y));
    float2 ser = __ffma2_rn(u, f2(0.2f, 0.2f), f2(-0.25f, -0.25f));
    ser = __ffma2_rn(ser, u, f2(1.f / 3.f, 1.f / 3.f));
    ser = __ffma2_rn(ser, u, f2(-0.5f, -0.5f));
    ser = __ffma2_rn(ser, u, f2(1.f, 1.f));
    ser = __fmul2_rn(ser, u);
    const float2 w = __fadd2_rn(u, f2(1.f, 1.f));
    const float2 lg = __fmul2_rn(f2(lg2(w.x), lg2(w.y)), f2(kLn2, kLn2));
    const float vx = u.x < 0.03125f ? ser.x : lg.x, vy = u.y < 0.03125f ? ser.y : lg.y;
    return f2(r.x > 20.f ? r.x : vx, r.y > 20.f ? r.y : vy);
}

__device__ __forceinline__ float2 silu_x2(float2 z) {
    const float2 q = __fmul2_rn(z, f2(-kLog2e, -kLog2e));
    const float2 d = __fadd2_rn(f2(ex2(q.x), ex2(q.y)), f2(1.f, 1.f));
    return __fmul2_rn(z, f2(rcp(d.x), rcp(d.y)));
}

}  // namespace sscan
