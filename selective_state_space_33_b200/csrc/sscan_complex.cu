// sscan_complex.cu -- forward selective scan with a complex diagonal A (the complex
// initialisation A_n = -1/2 + n i of the A-init ablation table, sec. 6.5 of the
// Mamba technical summary page): eqs. (2) and (3) of sec. 2.1 in complex
// arithmetic, with B and C the real input projections of sec. 3.2 and the output
// the real part of the readout, y_t = Re(sum_n C_tn h_tn) + D_skip x_t, gated by
// SiLU(z) (Fig. 3).
//
// Work decomposition (as the real tiled kernel): a CTA of 4 warps owns one batch
// and DC channels for the whole sequence; the NG lanes of a channel each hold CG
// complex states (CG = 4, or 2 when the grid is small) in registers.  Per 16-step tile all threads
// stage (delta, x) and (gate, D x gate) for the tile's channels and the tile's B
// and C rows in shared memory with coalesced loads (phase P), then every lane
// advances its states through the tile (phase S) and the NG lanes of a channel
// sum their partial readouts with a butterfly; lane 0 of the channel writes out.
//
// One step of one complex state a = ar + i ai, with v = -B x / a:
//   Abar = 2^(delta ar log2 e) (cos(delta ai) + i sin(delta ai))       (eq. 2)
//   h'   = Abar (h - v) + v  = Abar h + (Abar - 1) B x / a             (eq. 3a)
// (the update form of the real kernels).  The angle is reduced to [-pi, pi] with a
// two-part 2 pi before the MUFU sine and cosine.  A CTA whose block holds an
// |a| < 2^-10 (a = 0 included) takes Bbar / B = delta phi1(delta a) with phi1's
// Taylor series in complex arithmetic where |delta a| < 1/16 instead.
#include <cuda_runtime.h>

#include <cstdint>

#include "sscan_launch.h"
#include "sscan_complex_math.cuh"
#include "sscan_math.cuh"
#include "sscan_plan.h"

namespace sscan {
namespace {

constexpr int kCTT = 16;           // steps per tile
constexpr int kCWarps = 4;
constexpr int kCThreads = kCWarps * 32;
constexpr float kCSmallA = 9.765625e-4f;
template <int NG, int CG>
struct CCfg {
    static constexpr int CW = 32 / NG;       // channels per warp
    static constexpr int DC = CW * kCWarps;  // channels per CTA
    static constexpr int NS = NG * CG;       // states covered (>= N)
};

// One step of the lane's CG complex states (eq. (2) and (3a) with complex a; B, x
// real): fast form h' = Abar (h - v) + v with v = -B x / a, or for a block with a
// small |a| Bbar / B = delta phi1(delta a) by its series.  Returns the partial readout
// Re(sum_j C_j h_j) over these states (eq. (3b)).
template <int CG, bool ACC>
__device__ __forceinline__ float cstep(float2 (&h)[CG], const float2 (&aq)[CG], const float2 (&nia)[CG],
                                       const float2 (&ia)[CG], float delta, float x, const float* Bt,
                                       const float* Ct) {
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < CG; ++j) {
        const float e = ex2(delta * aq[j].x);
        const float2 cs = cplx::cis(delta * aq[j].y);
        const float abr = e * cs.x, abi = e * cs.y;
        const float bx = Bt[j] * x;
        float nr, ni;
        if (!ACC) {
            const float vr = bx * nia[j].x, vi = bx * nia[j].y;
            const float tr = h[j].x - vr, ti = h[j].y - vi;
            nr = fmaf(abr, tr, fmaf(-abi, ti, vr));
            ni = fmaf(abr, ti, fmaf(abi, tr, vi));
        } else {
            // Bbar / B = delta phi1(q), q = delta a: series for |q| < 1/16, else (Abar - 1) / a
            const float qr = delta * aq[j].x * kLn2, qi = delta * aq[j].y;
            float cr, ci;
            if (qr * qr + qi * qi < 0.00390625f) {
                // phi1(q) = 1 + q/2 + q^2/6 + q^3/24 + q^4/120, Horner in complex arithmetic
                float pr = 1.f / 120.f, pi = 0.f;
                const float cf[4] = {1.f / 24.f, 1.f / 6.f, 0.5f, 1.f};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float r2 = fmaf(pr, qr, fmaf(-pi, qi, cf[k]));
                    pi = fmaf(pr, qi, pi * qr);
                    pr = r2;
                }
                cr = delta * pr;
                ci = delta * pi;
            } else {
                const float er = abr - 1.f;
                cr = fmaf(er, ia[j].x, -abi * ia[j].y);
                ci = fmaf(er, ia[j].y, abi * ia[j].x);
            }
            nr = fmaf(abr, h[j].x, fmaf(-abi, h[j].y, cr * bx));
            ni = fmaf(abr, h[j].y, fmaf(abi, h[j].x, ci * bx));
        }
        h[j] = make_float2(nr, ni);
        y = fmaf(Ct[j], nr, y);
    }
    return y;
}

// Sum the partial readouts of a channel's NG lanes (lane bits at multiples of CW)
// for NG consecutive steps so that lane g ends with the sum for step g: a transposed
// butterfly, NG - 1 shuffles per NG steps instead of log2(NG) per step.
template <int NG, int CW>
__device__ __forceinline__ float creduce(float (&p)[NG], int g) {
    if constexpr (NG == 1) {
        return p[0];
    } else {
#pragma unroll
        for (int m = NG / 2; m >= 1; m /= 2) {
            const bool up = (g & m) != 0;
#pragma unroll
            for (int j = 0; j < m; ++j) {
                const float keep = up ? p[m + j] : p[j];
                const float send = up ? p[j] : p[m + j];
                p[j] = keep + __shfl_xor_sync(0xffffffffu, send, m * CW);
            }
        }
        return p[0];
    }
}

// Phase S over one tile.  Checkpoint pass: the state before every 8th step, no
// readout.  Output pass: blocks of NG steps whose readouts are reduced together, lane
// g finishing step tb + g; FULL tiles (kCTT steps) are unrolled with no step predicate.
template <typename T, int NG, int CG, bool ACC, bool CKPT, bool FULL>
__device__ __forceinline__ void scan_tile_c(float2 (&h)[CG], const float2 (&aq)[CG], const float2 (&nia)[CG],
                                            const float2 (&ia)[CG], const float2* sdx, const float2* sgd,
                                            const float* sB, const float* sC, int tl, int g, int cw, bool write,
                                            T* out, int64_t out_stride, float* ck, int64_t ck_stride, int nvalid) {
    using C = CCfg<NG, CG>;
    const float* Bg = sB + g * CG;
    const float* Cg = sC + g * CG;
    if constexpr (CKPT) {
        for (int t = 0; t < tl; ++t) {
            if (t % 8 == 0) {
                // the state before step t: a starting point of the backward's recomputation
#pragma unroll
                for (int j = 0; j < CG; ++j)
                    if (j < nvalid) {
                        ck[(t / 8) * ck_stride + 2 * j] = h[j].x;
                        ck[(t / 8) * ck_stride + 2 * j + 1] = h[j].y;
                    }
            }
            const float2 dx = sdx[t * C::DC + cw];  // (delta, x)
            (void)cstep<CG, ACC>(h, aq, nia, ia, dx.x, dx.y, Bg + t * C::NS, Cg + t * C::NS);
        }
    } else {
#pragma unroll(FULL ? kCTT / NG : 1)
        for (int tb = 0; tb < (FULL ? kCTT : tl); tb += NG) {
            float p[NG];
#pragma unroll
            for (int k = 0; k < NG; ++k) {
                const int t = tb + k;
                p[k] = 0.f;
                if (FULL || t < tl) {
                    const float2 dx = sdx[t * C::DC + cw];  // (delta, x)
                    p[k] = cstep<CG, ACC>(h, aq, nia, ia, dx.x, dx.y, Bg + t * C::NS, Cg + t * C::NS);
                }
            }
            const float y = creduce<NG, C::CW>(p, g);
            const int t = tb + g;
            if (write && (FULL || t < tl)) {
                const float2 gd = sgd[t * C::DC + cw];
                IO<T>::store(out, (int64_t)t * out_stride, fmaf(y, gd.x, gd.y));
            }
        }
    }
}

// CKPT: the checkpoint pass of the backward (states before every 8th step, no output);
// otherwise the forward with outputs.  Separate instantiations keep the per-step
// checkpoint test out of the output kernel's loop.
template <typename T, int NG, int CG, bool CKPT>
__global__ void __launch_bounds__(kCThreads) fwd_complex_kernel(ComplexArgs a, float* ckpt, int64_t nck) {
    using C = CCfg<NG, CG>;
    __shared__ float2 sdx[kCTT * C::DC];  // (delta, x)
    __shared__ float2 sgd[kCTT * C::DC];  // (gate, D x gate)
    __shared__ float sB[kCTT * C::NS], sC[kCTT * C::NS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t ncb = (a.D + C::DC - 1) / C::DC;
    const int64_t b = blockIdx.x / ncb;
    const int64_t d0 = (blockIdx.x % ncb) * C::DC;
    const int N = a.N;
    const T* u = static_cast<const T*>(a.u);
    const T* dr = static_cast<const T*>(a.delta_raw);
    const T* zz = static_cast<const T*>(a.z);
    const T* Bg = static_cast<const T*>(a.B);
    const T* Cg = static_cast<const T*>(a.C);

    const int g = lane / C::CW, c = lane % C::CW, cw = warp * C::CW + c;
    const int64_t d = d0 + cw;
    const bool cvalid = d < a.D;
    float2 h[CG], aq[CG], nia[CG], ia[CG];
    bool small_a = false;
#pragma unroll
    for (int j = 0; j < CG; ++j) {
        const int n = g * CG + j;
        const bool ok = cvalid && n < N;
        const float ar = ok ? __ldg(a.A + (d * N + n) * 2) : -1.f;
        const float ai = ok ? __ldg(a.A + (d * N + n) * 2 + 1) : 0.f;
        const float m2 = ar * ar + ai * ai;
        small_a |= ok && m2 < kCSmallA * kCSmallA;
        aq[j] = make_float2(ar * kLog2e, ai);
        const float inv = ok && m2 > 0.f ? 1.f / m2 : 0.f;
        ia[j] = make_float2(ar * inv, -ai * inv);      // 1 / a
        nia[j] = make_float2(-ia[j].x, -ia[j].y);      // -1 / a
        h[j] = make_float2(0.f, 0.f);
        if (ok && a.h0) h[j] = make_float2(__ldg(a.h0 + ((b * a.D + d) * N + n) * 2),
                                           __ldg(a.h0 + ((b * a.D + d) * N + n) * 2 + 1));
    }
    const bool acc = __syncthreads_or(small_a ? 1 : 0) != 0;
    const int nvalid = cvalid ? (N - g * CG < CG ? N - g * CG : CG) : 0;

    for (int64_t t0 = 0; t0 < a.L; t0 += kCTT) {
        const int tl = (int)(a.L - t0 < kCTT ? a.L - t0 : kCTT);
        // phase P: (delta, x), (gate, D x gate), and the tile's B and C rows
        for (int e = tid; e < kCTT * C::DC; e += kCThreads) {
            const int t = e / C::DC, cc = e % C::DC;
            const int64_t dd = d0 + cc;
            float2 dx = make_float2(0.f, 0.f), gd = make_float2(0.f, 0.f);
            if (t < tl && dd < a.D) {
                const int64_t gi = (b * a.L + t0 + t) * a.D + dd;
                const float x = IO<T>::load(u, gi);
                const float r = IO<T>::load(dr, gi) + (a.bias ? __ldg(a.bias + dd) : 0.f);
                const float gate = zz ? silu(IO<T>::load(zz, gi)) : 1.f;
                const float dsk = a.Dskip ? __ldg(a.Dskip + dd) : 0.f;
                dx = make_float2(a.softplus ? softplus(r) : r, x);
                gd = make_float2(gate, dsk * x * gate);
            }
            sdx[e] = dx;
            sgd[e] = gd;
        }
        for (int e = tid; e < kCTT * C::NS; e += kCThreads) {
            const int t = e / C::NS, n = e % C::NS;
            float bv = 0.f, cv = 0.f;
            if (t < tl && n < N) {
                const int64_t gi = (b * a.L + t0 + t) * N + n;
                bv = IO<T>::load(Bg, gi);
                cv = IO<T>::load(Cg, gi);
            }
            sB[e] = bv;
            sC[e] = cv;
        }
        __syncthreads();
        T* out = CKPT ? nullptr : static_cast<T*>(a.out) + (b * a.L + t0) * a.D + d;
        float* ck = CKPT ? ckpt + (((b * nck + t0 / 8) * a.D + d) * N + g * CG) * 2 : nullptr;
        const int64_t ck_stride = a.D * N * 2;
        const bool wr = cvalid;
        if (acc)
            scan_tile_c<T, NG, CG, true, CKPT, false>(h, aq, nia, ia, sdx, sgd, sB, sC, tl, g, cw, wr, out, a.D, ck,
                                                      ck_stride, nvalid);
        else if (tl == kCTT)
            scan_tile_c<T, NG, CG, false, CKPT, true>(h, aq, nia, ia, sdx, sgd, sB, sC, tl, g, cw, wr, out, a.D, ck,
                                                      ck_stride, nvalid);
        else
            scan_tile_c<T, NG, CG, false, CKPT, false>(h, aq, nia, ia, sdx, sgd, sB, sC, tl, g, cw, wr, out, a.D, ck,
                                                       ck_stride, nvalid);
        __syncthreads();
    }
    if (a.h_last && cvalid) {
#pragma unroll
        for (int j = 0; j < CG; ++j) {
            const int n = g * CG + j;
            if (n < N) {
                a.h_last[((b * a.D + d) * N + n) * 2] = h[j].x;
                a.h_last[((b * a.D + d) * N + n) * 2 + 1] = h[j].y;
            }
        }
    }
}

template <typename T, int NG, int CG>
cudaError_t launch_c(const ComplexArgs& a, float* ckpt, int64_t nck, cudaStream_t st) {
    const int64_t blocks = a.batch * ((a.D + CCfg<NG, CG>::DC - 1) / CCfg<NG, CG>::DC);
    if (blocks <= 0) return cudaGetLastError();
    if (ckpt)
        fwd_complex_kernel<T, NG, CG, true><<<(unsigned)blocks, kCThreads, 0, st>>>(a, ckpt, nck);
    else
        fwd_complex_kernel<T, NG, CG, false><<<(unsigned)blocks, kCThreads, 0, st>>>(a, nullptr, 0);
    return cudaGetLastError();
}

// Four complex states per lane, or two (twice the lanes per channel, half the
// channels per CTA) when the four-state grid would leave the GPU short of CTAs:
// measured at batch 8, L 2048, N 16: D 1536 0.90 ms with two states against 1.08 ms
// with four; D 5120 2.34 ms with four against 2.37 ms with two.
template <typename T>
cudaError_t launch_ct(const ComplexArgs& a, float* ckpt, int64_t nck, cudaStream_t st) {
    const int64_t ng4 = a.N <= 4 ? 1 : (a.N <= 8 ? 2 : 4);
    const int64_t ctas4 = a.batch * ((a.D + 4 * (32 / ng4) - 1) / (4 * (32 / ng4)));
    if (ctas4 < 4 * (int64_t)kSmCount) {
        if (a.N <= 2) return launch_c<T, 1, 2>(a, ckpt, nck, st);
        if (a.N <= 4) return launch_c<T, 2, 2>(a, ckpt, nck, st);
        if (a.N <= 8) return launch_c<T, 4, 2>(a, ckpt, nck, st);
        return launch_c<T, 8, 2>(a, ckpt, nck, st);
    }
    if (a.N <= 4) return launch_c<T, 1, 4>(a, ckpt, nck, st);
    if (a.N <= 8) return launch_c<T, 2, 4>(a, ckpt, nck, st);
    return launch_c<T, 4, 4>(a, ckpt, nck, st);
}

}  // namespace

cudaError_t launch_fwd_complex(const ComplexArgs& a, float* ckpt, int64_t nck, int io_bf16, cudaStream_t st) {
    return io_bf16 ? launch_ct<__nv_bfloat16>(a, ckpt, nck, st) : launch_ct<float>(a, ckpt, nck, st);
}

}  // namespace sscan
