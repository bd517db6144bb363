// sscan_step.cu -- one recurrence step for every (batch, channel): the
// constant-time, constant-memory update used for autoregressive generation
// (Mamba technical summary page, sec. 5: each generated token costs one state
// update, with no cache that grows with the context; sec. 2.1 eqs. (2), (3a),
// (3b) at a single t).
//
// The step moves 8 N bytes of fp32 state per channel against N exponentials, so it
// is bound by HBM bandwidth; it therefore uses the exact series form of Bbar near
// delta A = 0 at no cost.  Two kernels:
//   step_quad_kernel (N = 4, 8 or 16, vector-aligned rows): every lane owns 8 states
//     (4 when N = 4) of one (batch, channel) row -- 16-byte loads and stores of its
//     state, 16-byte loads of A, 4-element loads of B and C -- and the lanes of a row
//     sum their partial readouts with shuffles.  Many small independent lanes keep enough
//     loads in flight to stream the state at full bandwidth.
//   step_kernel (any N <= 16, any alignment): one thread per row, all N states.
#include <cuda_runtime.h>

#include "sscan_launch.h"
#include "sscan_math.cuh"

namespace sscan {
namespace {

// One thread per (batch, channel) row, all N states in registers, scalar loads.
template <typename T, int NMAX>
__global__ void __launch_bounds__(128) step_kernel(StepArgs a) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= a.batch * a.D) return;
    const int64_t b = row / a.D, d = row - b * a.D;
    const int N = a.N;
    const T* Bm = static_cast<const T*>(a.B) + b * N;
    const T* Cm = static_cast<const T*>(a.C) + b * N;
    float* hp = a.state + row * N;

    // every load first (state, parameters, B and C rows), then the arithmetic
    float h[NMAX], Av[NMAX], Bv[NMAX], Cv[NMAX];
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        h[n] = n < N ? hp[n] : 0.f;
        Av[n] = n < N ? __ldg(a.A + d * N + n) : 0.f;
        Bv[n] = n < N ? IO<T>::load(Bm, n) : 0.f;
        Cv[n] = n < N ? IO<T>::load(Cm, n) : 0.f;
    }
    const float uv = IO<T>::load(static_cast<const T*>(a.u), row);
    const float x = a.input_silu ? silu(uv) : uv;
    const float r = IO<T>::load(static_cast<const T*>(a.delta_raw), row) + (a.bias ? __ldg(a.bias + d) : 0.f);
    const float dsk = a.Dskip ? __ldg(a.Dskip + d) : 0.f;
    const float gz = a.z ? IO<T>::load(static_cast<const T*>(a.z), row) : 0.f;

    const float delta = a.softplus ? softplus(r) : r;
    float y = 0.f;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
        if (n < N) {
            const float An = Av[n];
            const float abar = ex2(delta * An * kLog2e);
            const float beta = bbar_coef(delta, delta * An, abar, An != 0.f ? rcp(An) : 0.f);
            h[n] = fmaf(abar, h[n], beta * Bv[n] * x);
            y = fmaf(Cv[n], h[n], y);
        }
    }
    y = fmaf(dsk, x, y);
    if (a.z) y *= silu(gz);
    IO<T>::store(static_cast<T*>(a.out), row, y);
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
        if (n < N) hp[n] = h[n];
}

// Four consecutive values of a B or C row as fp32 (8 bytes of bf16 or 16 of fp32).
template <typename T>
__device__ __forceinline__ float4 load4(const T* p) {
    if constexpr (sizeof(T) == 4) {
        return __ldg(reinterpret_cast<const float4*>(p));
    } else {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    }
}

// Grid: (lane blocks over one batch's D x LPR lanes, batch); no integer division
// by a runtime size anywhere.
// Grid: (lane blocks over one batch's D x LPR lanes, batch); no integer division
// by a runtime size anywhere.  Each lane owns SPL (4 or 8) consecutive states.
template <typename T, int LPR, int SPL>
__global__ void __launch_bounds__(256) step_quad_kernel(StepArgs a) {
    constexpr int N = SPL * LPR, NV = SPL / 4;
    const int64_t b = blockIdx.y;
    const int64_t gl = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // lanes past the last channel still take part in the row shuffles, on the last channel
    const bool valid = gl / LPR < a.D;
    const int64_t d = valid ? gl / LPR : a.D - 1;
    const int q = (int)(gl % LPR);
    const int64_t row = b * a.D + d;
    float4* hp = reinterpret_cast<float4*>(a.state + row * N + q * SPL);

    float hv[SPL], An[SPL], Bn[SPL], Cn[SPL];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        const float4 h = hp[v];
        const float4 Av = __ldg(reinterpret_cast<const float4*>(a.A + d * N + q * SPL) + v);
        const float4 Bv = load4<T>(static_cast<const T*>(a.B) + b * N + q * SPL + 4 * v);
        const float4 Cv = load4<T>(static_cast<const T*>(a.C) + b * N + q * SPL + 4 * v);
        hv[4 * v] = h.x, hv[4 * v + 1] = h.y, hv[4 * v + 2] = h.z, hv[4 * v + 3] = h.w;
        An[4 * v] = Av.x, An[4 * v + 1] = Av.y, An[4 * v + 2] = Av.z, An[4 * v + 3] = Av.w;
        Bn[4 * v] = Bv.x, Bn[4 * v + 1] = Bv.y, Bn[4 * v + 2] = Bv.z, Bn[4 * v + 3] = Bv.w;
        Cn[4 * v] = Cv.x, Cn[4 * v + 1] = Cv.y, Cn[4 * v + 2] = Cv.z, Cn[4 * v + 3] = Cv.w;
    }
    const float uv = IO<T>::load(static_cast<const T*>(a.u), row);
    const float x = a.input_silu ? silu(uv) : uv;
    const float r = IO<T>::load(static_cast<const T*>(a.delta_raw), row) + (a.bias ? __ldg(a.bias + d) : 0.f);
    const float dsk = a.Dskip ? __ldg(a.Dskip + d) : 0.f;
    const float gz = a.z ? IO<T>::load(static_cast<const T*>(a.z), row) : 0.f;

    const float delta = a.softplus ? softplus(r) : r;
    const float dl2 = delta * kLog2e;
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < SPL; ++j) {
        const float abar = ex2(dl2 * An[j]);
        const float beta = bbar_coef(delta, delta * An[j], abar, An[j] != 0.f ? rcp(An[j]) : 0.f);
        hv[j] = fmaf(abar, hv[j], beta * (Bn[j] * x));
        y = fmaf(Cn[j], hv[j], y);
    }
#pragma unroll
    for (int m = 1; m < LPR; m *= 2) y += __shfl_xor_sync(0xffffffffu, y, m);
    if (!valid) return;
#pragma unroll
    for (int v = 0; v < NV; ++v) hp[v] = make_float4(hv[4 * v], hv[4 * v + 1], hv[4 * v + 2], hv[4 * v + 3]);
    if (q == 0) {
        y = fmaf(dsk, x, y);
        if (a.z) y *= silu(gz);
        IO<T>::store(static_cast<T*>(a.out), row, y);
    }
}

template <typename T>
cudaError_t launch_t(const StepArgs& a, cudaStream_t st) {
    const int64_t rows = a.batch * a.D;
    const unsigned blocks = (unsigned)((rows + 127) / 128);
    const bool quad = (a.N == 4 || a.N == 8 || a.N == 16) && reinterpret_cast<uintptr_t>(a.state) % 16 == 0 &&
                      reinterpret_cast<uintptr_t>(a.A) % 16 == 0 &&
                      reinterpret_cast<uintptr_t>(a.B) % (4 * sizeof(T)) == 0 &&
                      reinterpret_cast<uintptr_t>(a.C) % (4 * sizeof(T)) == 0;
    if (quad && a.batch <= 65535) {
        // 8 states per lane where N allows (measured: 10.2 us per step at batch 64,
        // D 5120, N 16, against 11.6 us with 4 states per lane)
        const int spl = a.N >= 8 ? 8 : 4;
        const dim3 grid((unsigned)((a.D * (a.N / spl) + 255) / 256), (unsigned)a.batch);
        if (a.N == 16) step_quad_kernel<T, 2, 8><<<grid, 256, 0, st>>>(a);
        else if (a.N == 8) step_quad_kernel<T, 1, 8><<<grid, 256, 0, st>>>(a);
        else step_quad_kernel<T, 1, 4><<<grid, 256, 0, st>>>(a);
        return cudaGetLastError();
    }
    if (a.N <= 4) step_kernel<T, 4><<<blocks, 128, 0, st>>>(a);
    else if (a.N <= 8) step_kernel<T, 8><<<blocks, 128, 0, st>>>(a);
    else step_kernel<T, 16><<<blocks, 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepArgs& a, int io_bf16, cudaStream_t st) {
    return io_bf16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
}

}  // namespace sscan
