// sscan_generic.cuh -- the general-purpose kernels of the selective scan: one
// thread per (batch, channel) row, all N states in registers, any layout
// alignment, any D, N <= 16.  They carry every size the fast path does not
// take, and the long-sequence split (chunk aggregates + carry) is built on them.
//
// Formulas: eqs. (2), (3a), (3b) of sec. 2.1, softplus of sec. 3.2, SiLU gate of
// Fig. 3 (Mamba technical summary page, kb.agiseed.tech).
#pragma once

#include "sscan_affine.cuh"
#include "sscan_check.cuh"
#include "sscan_math.cuh"

namespace sscan {

struct ScanArgs {
    int64_t batch, L, D, N;
    const void* u;
    const void* delta_raw;
    const float* bias;   // (D) or null
    const float* A;      // (D, N)
    const void* B;       // (batch, L, N)
    const void* C;       // (batch, L, N) or null when no output is written
    const float* Dskip;  // (D) or null
    const void* z;       // (batch, L, D) or null
    const float* h0;     // (batch, D, N) or null
    void* out;           // (batch, L, D) or null
    float* h_last;       // (batch, D, N) or null
    int softplus;
    int input_silu;      // the scan's input is SiLU(u)
    // sequence split: chunk c covers steps [c*chunk_len, min(L, (c+1)*chunk_len))
    int64_t chunk_len;
    int64_t nchunks;
    float* ws_state;  // [batch][nchunks][D][N]: chunk end states from zero, then carry-ins
    float* ws_dsum;   // [batch][nchunks][D]: sum of delta over each chunk
};

enum { kModeOutput = 0, kModeAggregate = 1 };

// One thread per (row, chunk); consecutive threads take consecutive channels of
// the same chunk, so the (batch, L, D) loads coalesce across the warp and the
// (batch, L, N) loads of B and C are warp-wide broadcasts.
//   kModeOutput   : starts from h0 (one chunk) or the chunk's carry-in, writes out
//                   for its steps; the last chunk writes h_last.
//   kModeAggregate: starts from zero, writes the chunk's end state and sum of delta.
template <typename T, int NMAX, int MODE>
__global__ void __launch_bounds__(128) fwd_rows_kernel(ScanArgs a) {
    const int64_t rows = a.batch * a.D;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows * a.nchunks) return;
    const int64_t c = gid / rows, row = gid - c * rows;
    const int64_t b = row / a.D, d = row - b * a.D;
    const int N = (int)a.N;
    const int64_t t0 = c * a.chunk_len;
    const int64_t t1 = min(a.L, t0 + a.chunk_len);
    const T* u = static_cast<const T*>(a.u);
    const T* dr = static_cast<const T*>(a.delta_raw);
    const T* Bm = static_cast<const T*>(a.B);
    const T* Cm = static_cast<const T*>(a.C);
    const T* z = static_cast<const T*>(a.z);
    T* out = static_cast<T*>(a.out);

    float h[NMAX], Al[NMAX], A2[NMAX], invA[NMAX];
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        const float An = n < N && in_range(d * N + n, a.D * N) ? __ldg(a.A + d * N + n) : 0.f;
        Al[n] = An;
        A2[n] = An * kLog2e;
        invA[n] = An != 0.f ? 1.f / An : 0.f;
        float h_init = 0.f;
        if (MODE == kModeOutput && n < N) {
            if (a.nchunks > 1)
                h_init = in_range(((b * a.nchunks + c) * a.D + d) * N + n, a.batch * a.nchunks * a.D * N)
                             ? a.ws_state[((b * a.nchunks + c) * a.D + d) * N + n]
                             : 0.f;
            else if (a.h0)
                h_init = in_range(row * N + n, a.batch * a.D * N) ? __ldg(a.h0 + row * N + n) : 0.f;
        }
        h[n] = h_init;
    }
    const float bias = a.bias ? __ldg(a.bias + d) : 0.f;
    const float dsk = a.Dskip ? __ldg(a.Dskip + d) : 0.f;
    float dsum = 0.f;

    for (int64_t t = t0; t < t1; ++t) {
        const int64_t e = (b * a.L + t) * a.D + d;
        const int64_t s = (b * a.L + t) * N;
        const float uv = IO<T>::load(u, e);
        const float x = a.input_silu ? silu(uv) : uv;
        const float r = IO<T>::load(dr, e) + bias;
        const float delta = a.softplus ? softplus(r) : r;
        if (MODE == kModeAggregate) dsum += delta;
        float y = 0.f;
#pragma unroll
        for (int n = 0; n < NMAX; ++n) {
            if (n < N) {
                const float abar = ex2(delta * A2[n]);
                const float beta = bbar_coef(delta, delta * Al[n], abar, invA[n]);
                h[n] = fmaf(abar, h[n], beta * IO<T>::load(Bm, s + n) * x);
                if (MODE == kModeOutput && out) y = fmaf(IO<T>::load(Cm, s + n), h[n], y);
            }
        }
        if (MODE == kModeOutput && out) {
            y = fmaf(dsk, x, y);
            if (z) y *= silu(IO<T>::load(z, e));
            IO<T>::store(out, e, y);
        }
    }
    if (MODE == kModeAggregate) {
#pragma unroll
        for (int n = 0; n < NMAX; ++n)
            if (n < N && in_range(((b * a.nchunks + c) * a.D + d) * N + n, a.batch * a.nchunks * a.D * N))
                a.ws_state[((b * a.nchunks + c) * a.D + d) * N + n] = h[n];
        if (in_range((b * a.nchunks + c) * a.D + d, a.batch * a.nchunks * a.D))
            a.ws_dsum[(b * a.nchunks + c) * a.D + d] = dsum;
    } else if (a.h_last && c == a.nchunks - 1) {
#pragma unroll
        for (int n = 0; n < NMAX; ++n)
            if (n < N && in_range(row * N + n, a.batch * a.D * N)) a.h_last[row * N + n] = h[n];
    }
}

// Cross-chunk carry.  Each chunk is the affine map h -> P_c h + H_c with
// P_c = exp(A_n * sum of delta over the chunk) (the product of its Abar) and H_c the
// chunk's end state from zero.  Composing the maps in order gives every chunk's
// carry-in; the composition of all of them applied to h0 is h_last.
// W lanes (affine_lanes(nchunks)) per (batch, channel, state); the carry-ins
// overwrite H in place.
__global__ void __launch_bounds__(128) carry_kernel(ScanArgs a, int W) {
    const int64_t total = a.batch * a.D * a.N;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / W;
    const bool valid = r < total;
    const int64_t w = valid ? r : total - 1;
    const int64_t n = w % a.N, bd = w / a.N;
    const int64_t d = bd % a.D, b = bd / a.D;
    const float A2 = __ldg(a.A + d * a.N + n) * kLog2e;
    const float h0 = a.h0 ? __ldg(a.h0 + w) : 0.f;
    const float h = affine_carry_warp(
        a.nchunks, h0, W, valid,
        [&](int64_t c, float& p, float& q) {
            const int64_t id = (b * a.nchunks + c) * a.D + d;
            p = in_range(id, a.batch * a.nchunks * a.D) ? ex2(A2 * a.ws_dsum[id]) : 0.f;
            q = in_range(id * a.N + n, a.batch * a.nchunks * a.D * a.N) ? a.ws_state[id * a.N + n] : 0.f;
        },
        [&](int64_t c, float v) {
            const int64_t is = ((b * a.nchunks + c) * a.D + d) * a.N + n;
            if (in_range(is, a.batch * a.nchunks * a.D * a.N)) a.ws_state[is] = v;
        });
    if (valid && a.h_last && (threadIdx.x & (W - 1)) == 0) a.h_last[w] = h;
}

// P = exp(A_n * sum of delta): the decay of a chunk summary, from the per-row sums
// that the aggregate pass leaves in dsum (batch, D).  One thread per (b, d, n).
__global__ void __launch_bounds__(128) decay_kernel(const float* dsum, const float* A, float* P, int64_t batch,
                                                    int64_t D, int64_t N) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= batch * D * N) return;
    const int64_t n = gid % N, bd = gid / N, d = bd % D;
    P[gid] = ex2(__ldg(A + d * N + n) * kLog2e * dsum[bd]);
}

// Compose K chunk maps h -> P_k h + H_k (each (batch, D, N), chunk-major) in order,
// starting from h0: carry_in[k] is the state entering chunk k, h_final the state
// after the last.  W lanes (affine_lanes(K)) per (b, d, n).
__global__ void __launch_bounds__(128) compose_kernel(const float* P, const float* H, const float* h0,
                                                      float* carry_in, float* h_final, int64_t K, int64_t BDN,
                                                      int W) {
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / W;
    const bool valid = r < BDN;
    const int64_t w = valid ? r : BDN - 1;
    const float h = affine_carry_warp(
        K, h0 ? __ldg(h0 + w) : 0.f, W, valid,
        [&](int64_t k, float& p, float& q) {
            p = __ldg(P + k * BDN + w);
            q = __ldg(H + k * BDN + w);
        },
        [&](int64_t k, float v) {
            if (carry_in) carry_in[k * BDN + w] = v;
        });
    if (valid && h_final && (threadIdx.x & (W - 1)) == 0) h_final[w] = h;
}

}  // namespace sscan
