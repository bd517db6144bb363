// sscan_math.cuh -- fp32 device arithmetic of the selective scan.
//
// Everything here is written from the mathematics; the only hardware primitives
// are the sm_100a MUFU instructions ex2.approx / lg2.approx / rcp.approx, reached
// through inline PTX.  Accuracy targets: a relative error of a few 1e-6 in delta,
// Abar and Bbar, well inside the 1e-4 (fp32 I/O) output tolerance.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace sscan {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(r) = log(1 + e^r)  (sec. 3.2: delta passes through softplus).
//   r > 20          : r (the neglected log1p(e^-r) is below 2.1e-9 absolute)
//   e^r < 2^-5      : log1p(u) by its alternating Taylor series u - u^2/2 + ... + u^5/5;
//                     the dropped tail is below u^6/6, i.e. < 5e-9 relative
//   otherwise       : ln2 * log2(1 + u); 1 + u >= 1.03 so the rounding of the sum
//                     costs at most ~2e-6 relative
__device__ __forceinline__ float softplus(float r) {
    if (r > 20.f) return r;
    const float u = ex2(r * kLog2e);
    if (u < 0.03125f) {
        return u * fmaf(u, fmaf(u, fmaf(u, fmaf(u, 0.2f, -0.25f), 1.f / 3.f), -0.5f), 1.f);
    }
    return kLn2 * lg2(1.f + u);
}

// d softplus / dr = sigmoid(r) = 1 / (1 + e^-r).
__device__ __forceinline__ float sigmoid(float r) { return rcp(1.f + ex2(-r * kLog2e)); }

// SiLU(v) = v * sigmoid(v)  (Fig. 3: the block's gate activation).
__device__ __forceinline__ float silu(float v) { return v * sigmoid(v); }

// d SiLU / dv = s (1 + v (1 - s)), s = sigmoid(v).
__device__ __forceinline__ float dsilu(float v) {
    const float s = sigmoid(v);
    return s * fmaf(v, 1.f - s, 1.f);
}

// phi1(q) = expm1(q) / q for |q| < 1/16, by the Taylor series 1 + q/2 + q^2/6 + q^3/24
// + q^4/120 (the dropped q^5/720 term is < 1.3e-9 relative).
__device__ __forceinline__ float phi1_series(float q) {
    return fmaf(q, fmaf(q, fmaf(q, fmaf(q, 1.f / 120.f, 1.f / 24.f), 1.f / 6.f), 0.5f), 1.f);
}

// Bbar / B for one state (eq. (2) with diagonal A): expm1(delta A) / A.
//   |q| = |delta A| < 1/16 : delta * phi1(q)  (also the A = 0 limit, delta)
//   otherwise              : (abar - 1) / A, with abar = exp(q) already computed; the
//                            subtraction loses at most ~2e-6 relative at |q| = 1/16
__device__ __forceinline__ float bbar_coef(float delta, float q, float abar, float invA) {
    return fabsf(q) < 0.0625f ? delta * phi1_series(q) : (abar - 1.f) * invA;
}

// I/O element access (fp32 or bf16 storage, fp32 arithmetic).
template <typename T> struct IO;
template <> struct IO<float> {
    static __device__ __forceinline__ float load(const float* p, int64_t i) { return __ldg(p + i); }
    static __device__ __forceinline__ void store(float* p, int64_t i, float v) { p[i] = v; }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p, int64_t i) {
        return __bfloat162float(__ldg(p + i));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, int64_t i, float v) {
        p[i] = __float2bfloat16_rn(v);
    }
};

}  // namespace sscan
