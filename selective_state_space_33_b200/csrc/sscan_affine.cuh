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

// Inclusive scan of affine maps h -> a h + b over segments of W lanes of a warp (W a
// power of two, 1 .. 32), in lane order: sub-lane i ends with the composition of
// the maps of sub-lanes 0..i (sub-lane 0's map applied first).  Composition:
// (a', b') after (a, b) is (a' a, a' b + b').  Hillis-Steele, log2(W) shuffle rounds.
__device__ __forceinline__ void affine_scan_warp(float& a, float& b, int W) {
    const int sub = (int)(threadIdx.x & 31) & (W - 1);
    for (int off = 1; off < W; off <<= 1) {
        const float ap = __shfl_up_sync(0xffffffffu, a, off, W);
        const float bp = __shfl_up_sync(0xffffffffu, b, off, W);
        if (sub >= off) {
            b = fmaf(a, bp, b);
            a *= ap;
        }
    }
}

// Lanes per row for carrying through K maps: the smallest power of two >= K, at
// most 32 (a warp then serves 32 / W rows).
inline int affine_lanes(int64_t K) {
    int W = 1;
    while (W < 32 && W < K) W <<= 1;
    return W;
}

// Carry through K consecutive affine maps for one row (a (batch, channel, state)):
// the row's W lanes take the maps W at a time (map k from get(k, a, b)), scan them
// with shuffles, hand every map the state entering it through put(k, h) and return
// the state after the last.  Lanes past K hold the identity map; a row past the end
// of the problem (valid == false) takes part in the shuffles with identities only.
// Every lane of the warp must call this (the shuffles use the full mask).
template <typename Get, typename Put>
__device__ __forceinline__ float affine_carry_warp(int64_t K, float h, int W, bool valid, Get get, Put put) {
    const int sub = (int)(threadIdx.x & 31) & (W - 1);
    for (int64_t k0 = 0; k0 < K; k0 += W) {
        const int64_t k = k0 + sub;
        float a = 1.f, b = 0.f;
        if (valid && k < K) get(k, a, b);
        affine_scan_warp(a, b, W);
        // the state entering map k: the inclusive result of sub-lane - 1 applied to h
        float ae = __shfl_up_sync(0xffffffffu, a, 1, W), be = __shfl_up_sync(0xffffffffu, b, 1, W);
        if (sub == 0) {
            ae = 1.f;
            be = 0.f;
        }
        if (valid && k < K) put(k, fmaf(ae, h, be));
        h = fmaf(__shfl_sync(0xffffffffu, a, W - 1, W), h, __shfl_sync(0xffffffffu, b, W - 1, W));
    }
    return h;
}

}  // namespace sscan
