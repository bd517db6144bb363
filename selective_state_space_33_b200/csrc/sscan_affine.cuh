// sscan_affine.cuh -- the warp-shuffle scan of affine pairs that carries state
// across sequence chunks (forward chunks, ranks' stretches, backward segments).
//
// A stretch of the recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t (Mamba technical
// summary page, sec. 2.1, eq. (3a)) is affine in its initial state: h -> a h + b with
// a the product of the stretch's Abar and b its end state from zero.  Consecutive
// stretches compose as (a', b') after (a, b) = (a' a, a' b + b'), an associative
// operation, so the states entering K stretches are an exclusive scan of their
// pairs.
#pragma once

#include <cstdint>

namespace sscan {

// Inclusive scan of affine maps h -> a h + b over the 32 lanes of a warp, in lane
// order: lane i ends with the composition of the maps of lanes 0..i (lane 0's map
// applied first).  Composition: (a', b') after (a, b) is (a' a, a' b + b').
// Hillis-Steele over 5 shuffle rounds.
__device__ __forceinline__ void affine_scan_warp(float& a, float& b) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float ap = __shfl_up_sync(0xffffffffu, a, off);
        const float bp = __shfl_up_sync(0xffffffffu, b, off);
        if (lane >= off) {
            b = fmaf(a, bp, b);
            a *= ap;
        }
    }
}

// Carry through K consecutive affine maps for one (batch, channel, state): the warp
// takes the maps 32 at a time (map k from get(k) = (a_k, b_k)), scans them with
// shuffles, hands every map the state entering it through put(k, h) and returns the
// state after the last.  Lanes past K hold the identity map.
template <typename Get, typename Put>
__device__ __forceinline__ float affine_carry_warp(int64_t K, float h, Get get, Put put) {
    const int lane = threadIdx.x & 31;
    for (int64_t k0 = 0; k0 < K; k0 += 32) {
        const int64_t k = k0 + lane;
        float a = 1.f, b = 0.f;
        if (k < K) get(k, a, b);
        affine_scan_warp(a, b);
        // the state entering map k: the inclusive result of lane - 1 applied to h
        float ae = __shfl_up_sync(0xffffffffu, a, 1), be = __shfl_up_sync(0xffffffffu, b, 1);
        if (lane == 0) {
            ae = 1.f;
            be = 0.f;
        }
        if (k < K) put(k, fmaf(ae, h, be));
        h = fmaf(__shfl_sync(0xffffffffu, a, 31), h, __shfl_sync(0xffffffffu, b, 31));
    }
    return h;
}

}  // namespace sscan
