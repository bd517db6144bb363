// sscan_step.cu -- one recurrence step for every (batch, channel): the
// constant-time, constant-memory update used for autoregressive generation
// (Mamba technical summary page, sec. 5: each generated token costs one state
// update, with no cache that grows with the context; sec. 2.1 eqs. (2), (3a),
// (3b) at a single t).
//
// One thread per (batch, channel): it reads its N fp32 states (16-byte vector
// loads when N is a multiple of 4), applies h <- Abar h + Bbar x, writes them back
// in place and writes the gated output.  The step moves 8 N bytes of state per
// channel against a handful of exponentials, so it is bound by HBM bandwidth;
// it therefore uses the exact series form of Bbar near delta A = 0 at no cost.
#include <cuda_runtime.h>

#include "sscan_launch.h"
#include "sscan_math.cuh"

namespace sscan {
namespace {

// Load n values of one row into fp32 registers; VEC rows are 16-byte aligned with n a
// multiple of 16 bytes, read as 16-byte vectors.
template <typename T, int NMAX, bool VEC>
__device__ __forceinline__ void load_row(const T* p, int n, float (&v)[NMAX]) {
    if constexpr (VEC) {
        constexpr int PER = 16 / (int)sizeof(T);
#pragma unroll
        for (int k = 0; k < NMAX / PER; ++k) {
            const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p) + k);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                if constexpr (sizeof(T) == 4) {
                    v[k * PER + j] = __uint_as_float(w[j]);
                } else {  // bf16: the high half of an fp32 with the same bits
                    const uint32_t bits = (j & 1) ? (w[j / 2] & 0xffff0000u) : (w[j / 2] << 16);
                    v[k * PER + j] = __uint_as_float(bits);
                }
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < NMAX; ++j) v[j] = j < n ? IO<T>::load(p, j) : 0.f;
    }
}

template <typename T, int NMAX, bool VEC>
__global__ void __launch_bounds__(128) step_kernel(StepArgs a) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= a.batch * a.D) return;
    const int64_t b = row / a.D, d = row - b * a.D;
    const int N = a.N;
    const T* u = static_cast<const T*>(a.u);
    const T* dr = static_cast<const T*>(a.delta_raw);
    const T* z = static_cast<const T*>(a.z);
    float* hp = a.state + row * N;

    // every load first (state, parameters, B and C rows), then the arithmetic
    float h[NMAX], Av[NMAX], Bv[NMAX], Cv[NMAX];
    if (VEC) {
#pragma unroll
        for (int k = 0; k < NMAX / 4; ++k) {
            const float4 v = reinterpret_cast<const float4*>(hp)[k];
            h[4 * k] = v.x;
            h[4 * k + 1] = v.y;
            h[4 * k + 2] = v.z;
            h[4 * k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int n = 0; n < NMAX; ++n) h[n] = n < N ? hp[n] : 0.f;
    }
    load_row<float, NMAX, VEC>(a.A + d * N, N, Av);
    load_row<T, NMAX, VEC>(static_cast<const T*>(a.B) + b * N, N, Bv);
    load_row<T, NMAX, VEC>(static_cast<const T*>(a.C) + b * N, N, Cv);
    const float x = IO<T>::load(u, row);
    const float r = IO<T>::load(dr, row) + (a.bias ? __ldg(a.bias + d) : 0.f);
    const float dsk = a.Dskip ? __ldg(a.Dskip + d) : 0.f;
    const float gz = z ? IO<T>::load(z, row) : 0.f;

    const float delta = a.softplus ? softplus(r) : r;
    float y = 0.f;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        if (VEC || n < N) {
            const float An = Av[n];
            const float abar = ex2(delta * An * kLog2e);
            const float beta = bbar_coef(delta, delta * An, abar, An != 0.f ? 1.f / An : 0.f);
            h[n] = fmaf(abar, h[n], beta * Bv[n] * x);
            y = fmaf(Cv[n], h[n], y);
        }
    }
    y = fmaf(dsk, x, y);
    if (z) y *= silu(gz);
    IO<T>::store(static_cast<T*>(a.out), row, y);
    if (VEC) {
#pragma unroll
        for (int k = 0; k < NMAX / 4; ++k)
            reinterpret_cast<float4*>(hp)[k] = make_float4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3]);
    } else {
#pragma unroll
        for (int n = 0; n < NMAX; ++n)
            if (n < N) hp[n] = h[n];
    }
}

template <typename T>
cudaError_t launch_t(const StepArgs& a, cudaStream_t st) {
    const int64_t rows = a.batch * a.D;
    const unsigned blocks = (unsigned)((rows + 127) / 128);
    // 16-byte vectors need every row (state, A, B, C) to start on a 16-byte boundary
    const bool vec = (a.N * sizeof(T)) % 16 == 0 && (a.N * sizeof(float)) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(a.state) % 16 == 0 && reinterpret_cast<uintptr_t>(a.A) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(a.B) % 16 == 0 && reinterpret_cast<uintptr_t>(a.C) % 16 == 0;
    if (a.N == 16 && vec) step_kernel<T, 16, true><<<blocks, 128, 0, st>>>(a);
    else if (a.N == 8 && vec) step_kernel<T, 8, true><<<blocks, 128, 0, st>>>(a);
    else if (a.N <= 4) step_kernel<T, 4, false><<<blocks, 128, 0, st>>>(a);
    else if (a.N <= 8) step_kernel<T, 8, false><<<blocks, 128, 0, st>>>(a);
    else step_kernel<T, 16, false><<<blocks, 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepArgs& a, int io_bf16, cudaStream_t st) {
    return io_bf16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
}

}  // namespace sscan
