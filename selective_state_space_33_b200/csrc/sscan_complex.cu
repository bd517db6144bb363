// sscan_complex.cu -- forward selective scan with a complex diagonal A (the complex
// initialisation A_n = -1/2 + n i of the A-init ablation table, sec. 6.5 of the
// Mamba technical summary page): eqs. (2) and (3) of sec. 2.1 in complex
// arithmetic, with B and C the real input projections of sec. 3.2 and the output
// the real part of the readout, y_t = Re(sum_n C_tn h_tn) + D_skip x_t, gated by
// SiLU(z) (Fig. 3).
//
// Work decomposition (as the real tiled kernel): a CTA of 4 warps owns one batch
// and DC channels for the whole sequence; the NG lanes of a channel each hold CG
// complex states (CG = 4, or 2 when the grid is small) in registers.  Per 32- or 64-step
// tile, TMA 3-D tile copies bring u, delta_raw, z (and the B, C rows) into a one-stage
// shared-memory ring -- the next tile's copy lands while the current one is scanned;
// mbarrier completion, every wait bounded -- or, for tensors whose rows or bases are
// not 16-byte aligned, every thread loads them directly; all threads then stage
// (delta, x) pairs and the gate for the tile's channels and the tile's B and C rows
// in shared memory (phase P), then every lane
// advances its states through the tile (phase S), two states per f32x2 operation, and
// the NG lanes of a channel sum their partial readouts over blocks of NG steps with a
// transposed butterfly, each lane writing one step's output.
//
// One step of one complex state a = ar + i ai, with v = -B x / a:
//   Abar = 2^(delta ar log2 e) (cos(delta ai) + i sin(delta ai))       (eq. 2)
//   h'   = Abar (h - v) + v  = Abar h + (Abar - 1) B x / a             (eq. 3a)
// (the update form of the real kernels).  The angle is reduced to [-pi, pi] with a
// two-part 2 pi before the MUFU sine and cosine.  A CTA whose block holds an
// |a| < 2^-10 (a = 0 included) takes Bbar / B = delta phi1(delta a) with phi1's
// Taylor series in complex arithmetic where |delta a| < 1/16 instead.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <type_traits>

#include "sscan_launch.h"
#include "sscan_act.cuh"
#include "sscan_complex_math.cuh"
#include "sscan_math.cuh"
#include "sscan_plan.h"
#include "sscan_tma.cuh"

namespace sscan {

__device__ unsigned int g_device_error_cx = 0;

namespace {

constexpr int kCWarps = 4;
constexpr int kCThreads = kCWarps * 32;
constexpr float kCSmallA = 9.765625e-4f;
template <int NG, int CG>
struct CCfg {
    static constexpr int CW = 32 / NG;       // channels per warp
    static constexpr int DC = CW * kCWarps;  // channels per CTA
    static constexpr int NS = NG * CG;       // states covered (>= N)
};

// Dynamic shared memory of a TT-step tile: phase P's staging -- (delta, x) pairs and the
// SiLU gate per (step, channel), the tile's B and C rows -- and, on the TMA path, the
// output tile (written back by one TMA store per tile), a 2-stage ring of raw tiles (u,
// delta_raw, z, then B and C when their rows travel by TMA) and its mbarriers;
// 128-byte aligned sections.  One ring stage: phase P empties it before the next tile's
// copy is issued, and the copy lands while the tile is scanned (at the Mamba-130M shape
// 0.496 ms with two stages and 32-step tiles, 0.491 with one; 0.511 and 0.483 ms with
// 64-step tiles).
template <typename T, int NG, int CG, int TT>
struct CSmem {
    static constexpr int DC = CCfg<NG, CG>::DC, NS = CCfg<NG, CG>::NS;
    static constexpr int OFF_DX = 0;                                             // float2 [TT][DC]
    static constexpr int OFF_GT = OFF_DX + TT * DC * 8;                          // float  [TT][DC]
    static constexpr int OFF_B = OFF_GT + (TT * DC * 4 + 127) / 128 * 128;       // float  [TT][NS]
    static constexpr int OFF_C = OFF_B + (TT * NS * 4 + 127) / 128 * 128;        // float  [TT][NS]
    static constexpr int OFF_OUT = OFF_C + (TT * NS * 4 + 127) / 128 * 128;    // T [TT][DC] (TMA path)
    static constexpr int OFF_RING = OFF_OUT + (TT * DC * (int)sizeof(T) + 127) / 128 * 128;
    static constexpr int RAW = TT * DC * (int)sizeof(T);
    static constexpr int RAWBC = (TT * NS * (int)sizeof(T) + 127) / 128 * 128;  // one B or C tile (N <= NS)
    static constexpr int STAGE = (3 * RAW + 2 * RAWBC + 127) / 128 * 128;
    static constexpr int STAGES = 1;  // the next tile's copy lands during this tile's scan
    static constexpr int OFF_BAR = OFF_RING + STAGES * STAGE;
    static constexpr int SMEM_PLAIN = OFF_RING;          // plain loads: no ring
    static constexpr int SMEM_TMA = OFF_BAR + STAGES * 8;
    static constexpr int PAIRS = TT * DC / 2;            // channel pairs of phase P
    static_assert(RAW % 128 == 0 && (TT * DC * 8) % 128 == 0, "sections start 128-byte aligned");
    static_assert(PAIRS % kCThreads == 0, "phase P runs a fixed number of channel pairs per thread");
};

__device__ __forceinline__ float2 to_f32x2(float2 v) { return v; }
__device__ __forceinline__ float2 to_f32x2(__nv_bfloat162 v) { return __bfloat1622float2(v); }

__device__ __forceinline__ float2 ex2x2c(float2 q) { return make_float2(ex2(q.x), ex2(q.y)); }

// A lane's CG complex states and constants, packed over pairs of states so that the
// fast step runs on f32x2 arithmetic: hr[k] = (Re h_2k, Re h_2k+1), and likewise the
// imaginary parts, a log2(e) split into (Re, Im), and -1/a.
template <int CG>
struct CLane {
    static constexpr int P = CG / 2;
    float2 hr[P], hi[P];  // Re h, Im h
    float2 qr[P], qi[P];  // Re a log2 e, Im a
    float2 nr[P], ni[P];  // Re(-1/a), Im(-1/a)
};

// Component j of a pair-packed array (j is a compile-time index after unrolling).
template <int P>
__device__ __forceinline__ float& comp(float2 (&v)[P], int j) {
    return (j & 1) ? v[j >> 1].y : v[j >> 1].x;
}

// cos and sin of a pair of angles (the reduction of cplx::cis, packed).
__device__ __forceinline__ void cis2(float2 th, float2& cs, float2& sn) {
    const float2 m = __fmul2_rn(th, make_float2(-cplx::kInvTwoPi, -cplx::kInvTwoPi));
    const float2 nk = cplx::round2_fma(m);
    float2 r = __ffma2_rn(nk, make_float2(cplx::kTwoPiHi, cplx::kTwoPiHi), th);
    r = __ffma2_rn(nk, make_float2(cplx::kTwoPiLo, cplx::kTwoPiLo), r);
    cs = make_float2(cplx::cos_approx(r.x), cplx::cos_approx(r.y));
    sn = make_float2(cplx::sin_approx(r.x), cplx::sin_approx(r.y));
}

// One step of the lane's CG complex states (eq. (2) and (3a) with complex a; B, x
// real) in the fast form h' = Abar (h - v) + v with v = -B x / a, two states per
// packed operation, in two parts: cprep forms Abar and v (the MUFU work: 2^(delta Re a),
// cos and sin of delta Im a), cupd updates the states and returns the partial readout
// Re(sum_j C_j h_j) (eq. (3b)).  Full output tiles issue the cprep of step t + 1 before
// the cupd of step t.
template <int CG>
struct CPrep {
    float2 abr[CG / 2], abi[CG / 2], vr[CG / 2], vi[CG / 2];
};

template <int CG>
__device__ __forceinline__ CPrep<CG> cprep(const CLane<CG>& s, float delta, float x, const float* Bt) {
    CPrep<CG> P;
    const float2 dd = make_float2(delta, delta), xx = make_float2(x, x);
#pragma unroll
    for (int k = 0; k < CG / 2; ++k) {
        const float2 e = ex2x2c(__fmul2_rn(dd, s.qr[k]));
        float2 cs, sn;
        cis2(__fmul2_rn(dd, s.qi[k]), cs, sn);
        P.abr[k] = __fmul2_rn(e, cs);
        P.abi[k] = __fmul2_rn(e, sn);
        const float2 bx = __fmul2_rn(reinterpret_cast<const float2*>(Bt)[k], xx);
        P.vr[k] = __fmul2_rn(bx, s.nr[k]);
        P.vi[k] = __fmul2_rn(bx, s.ni[k]);
    }
    return P;
}

template <int CG>
__device__ __forceinline__ float cupd(CLane<CG>& s, const CPrep<CG>& P, const float* Ct) {
    float2 y = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < CG / 2; ++k) {
        const float2 tr = __ffma2_rn(P.vr[k], make_float2(-1.f, -1.f), s.hr[k]);   // Re(h - v)
        const float2 ti = __ffma2_rn(P.vi[k], make_float2(-1.f, -1.f), s.hi[k]);   // Im(h - v)
        const float2 mti = __ffma2_rn(s.hi[k], make_float2(-1.f, -1.f), P.vi[k]);  // -Im(h - v)
        s.hr[k] = __ffma2_rn(P.abr[k], tr, __ffma2_rn(P.abi[k], mti, P.vr[k]));
        s.hi[k] = __ffma2_rn(P.abr[k], ti, __ffma2_rn(P.abi[k], tr, P.vi[k]));
        y = __ffma2_rn(reinterpret_cast<const float2*>(Ct)[k], s.hr[k], y);
    }
    return y.x + y.y;
}

template <int CG>
__device__ __forceinline__ float cstep_fast(CLane<CG>& s, float delta, float x, const float* Bt,
                                            const float* Ct) {
    return cupd<CG>(s, cprep<CG>(s, delta, x, Bt), Ct);
}

// The same step for a block with a small |a|: Bbar / B = delta phi1(delta a) with
// phi1's series where |delta a| < 1/16, else (Abar - 1) / a; one state at a time.
template <int CG>
__device__ __forceinline__ float cstep_acc(CLane<CG>& s, float delta, float x, const float* Bt, const float* Ct) {
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < CG; ++j) {
        const float aqr = comp(s.qr, j), aqi = comp(s.qi, j);
        const float e = ex2(delta * aqr);
        const float2 cs = cplx::cis(delta * aqi);
        const float abr = e * cs.x, abi = e * cs.y;
        const float bx = Bt[j] * x;
        const float qr = delta * aqr * kLn2, qi = delta * aqi;
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
            const float er = abr - 1.f, iar = -comp(s.nr, j), iai = -comp(s.ni, j);  // 1 / a
            cr = fmaf(er, iar, -abi * iai);
            ci = fmaf(er, iai, abi * iar);
        }
        float& hr = comp(s.hr, j);
        float& hi = comp(s.hi, j);
        const float nr = fmaf(abr, hr, fmaf(-abi, hi, cr * bx));
        const float ni = fmaf(abr, hi, fmaf(abi, hr, ci * bx));
        hr = nr;
        hi = ni;
        y = fmaf(Ct[j], nr, y);
    }
    return y;
}

template <int CG, bool ACC>
__device__ __forceinline__ float cstep(CLane<CG>& s, float delta, float x, const float* Bt, const float* Ct) {
    if constexpr (ACC)
        return cstep_acc<CG>(s, delta, x, Bt, Ct);
    else
        return cstep_fast<CG>(s, delta, x, Bt, Ct);
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
// g finishing step tb + g (gate (y + D x), with the lane's own skip weight dskc); FULL
// tiles (TT steps) are unrolled with no step predicate.
template <typename T, int NG, int CG, int TT, bool ACC, bool CKPT, bool FULL>
__device__ __forceinline__ void scan_tile_c(CLane<CG>& s, const float2* sdx, const float* sgt, const float* sB,
                                            const float* sC, int tl, int g, int cw, bool write, T* out,
                                            int64_t out_stride, float dskc, float* ck, int64_t ck_stride,
                                            int nvalid) {
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
                        ck[(t / 8) * ck_stride + 2 * j] = comp(s.hr, j);
                        ck[(t / 8) * ck_stride + 2 * j + 1] = comp(s.hi, j);
                    }
            }
            const float2 dx = sdx[t * C::DC + cw];  // (delta, x)
            (void)cstep<CG, ACC>(s, dx.x, dx.y, Bg + t * C::NS, Cg + t * C::NS);
        }
    } else {
#pragma unroll(FULL ? TT / NG : 1)
        for (int tb = 0; tb < (FULL ? TT : tl); tb += NG) {
            float p[NG];
#pragma unroll
            for (int k = 0; k < NG; ++k) {
                const int t = tb + k;
                p[k] = 0.f;
                if (FULL || t < tl) {
                    const float2 dx = sdx[t * C::DC + cw];  // (delta, x)
                    p[k] = cstep<CG, ACC>(s, dx.x, dx.y, Bg + t * C::NS, Cg + t * C::NS);
                }
            }
            const float y = creduce<NG, C::CW>(p, g);
            const int t = tb + g;
            if (write && (FULL || t < tl))
                IO<T>::store(out, (int64_t)t * out_stride, sgt[t * C::DC + cw] * fmaf(dskc, sdx[t * C::DC + cw].y, y));
        }
    }
}

// Full output tiles of the fast form, software-pipelined: the exponentials, cosines and
// sines of step t + 1 (cprep) are issued before the state update of step t (cupd), so
// their MUFU latency overlaps the dependent fmas; the arithmetic is that of cstep_fast.
template <typename T, int NG, int CG, int TT>
__device__ __forceinline__ void scan_tile_c_pipe(CLane<CG>& s, const float2* sdx, const float* sgt, const float* sB,
                                                 const float* sC, int g, int cw, bool write, T* out,
                                                 int64_t out_stride, float dskc) {
    using C = CCfg<NG, CG>;
    const float* Bg = sB + g * CG;
    const float* Cg = sC + g * CG;
    const float2 dx0 = sdx[cw];
    CPrep<CG> P = cprep<CG>(s, dx0.x, dx0.y, Bg);
#pragma unroll
    for (int tb = 0; tb < TT; tb += NG) {
        float p[NG];
#pragma unroll
        for (int k = 0; k < NG; ++k) {
            const int t = tb + k;
            CPrep<CG> Pn = P;
            if (t + 1 < TT) {
                const float2 dx = sdx[(t + 1) * C::DC + cw];
                Pn = cprep<CG>(s, dx.x, dx.y, Bg + (t + 1) * C::NS);
            }
            p[k] = cupd<CG>(s, P, Cg + t * C::NS);
            P = Pn;
        }
        const float y = creduce<NG, C::CW>(p, g);
        const int t = tb + g;
        if (write) IO<T>::store(out, (int64_t)t * out_stride, sgt[t * C::DC + cw] * fmaf(dskc, sdx[t * C::DC + cw].y, y));
    }
}

// CKPT: the checkpoint pass of the backward (states before every 8th step, no output);
// otherwise the forward with outputs.  Separate instantiations keep the per-step
// checkpoint test out of the output kernel's loop.  TMA: the tiles come through the
// TMA ring (maps m[0..4] = u, delta_raw, z, B, C; bc_tma says whether B and C do);
// otherwise every thread loads them directly.
template <typename T, int NG, int CG, int TT, bool CKPT, bool TMA>
__global__ void __launch_bounds__(kCThreads)
    fwd_complex_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_dr,
                       const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_B,
                       const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_out,
                       ComplexArgs a, float* ckpt, int64_t nck, int bc_tma) {
    using C = CCfg<NG, CG>;
    using S = CSmem<T, NG, CG, TT>;
    constexpr bool kTileOut = TMA && !CKPT;  // outputs through a shared tile and a TMA store
    using P2 = typename std::conditional<sizeof(T) == 2, __nv_bfloat162, float2>::type;
    extern __shared__ __align__(128) unsigned char smem[];
    float2* sdx = reinterpret_cast<float2*>(smem + S::OFF_DX);  // (delta, x)
    float* sgt = reinterpret_cast<float*>(smem + S::OFF_GT);    // SiLU gate
    float* sB = reinterpret_cast<float*>(smem + S::OFF_B);
    float* sC = reinterpret_cast<float*>(smem + S::OFF_C);
    unsigned char* ring = smem + S::OFF_RING;
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
    const int ntile = (int)((a.L + TT - 1) / TT);
    const bool has_z = zz != nullptr;
    const uint32_t bar0 = TMA ? smem_u32(smem + S::OFF_BAR) : 0u;
    const uint32_t stage_bytes = (has_z ? 3u : 2u) * S::RAW + (bc_tma ? 2u * (uint32_t)(TT * N * (int)sizeof(T)) : 0u);

    // the TMA copies of tile `it` into its ring stage (elected thread only)
    auto issue = [&](int it) {
        const int st = it % S::STAGES;
        const uint32_t bar = bar0 + 8 * st;
        const uint32_t base = smem_u32(ring + st * S::STAGE);
        const int t0 = it * TT;
        mbar_expect_tx(bar, stage_bytes);
        tma_load_3d(base, &tm_u, (int)d0, t0, (int)b, bar);
        tma_load_3d(base + S::RAW, &tm_dr, (int)d0, t0, (int)b, bar);
        if (has_z) tma_load_3d(base + 2 * S::RAW, &tm_z, (int)d0, t0, (int)b, bar);
        if (bc_tma) {
            tma_load_3d(base + 3 * S::RAW, &tm_B, 0, t0, (int)b, bar);
            tma_load_3d(base + 3 * S::RAW + S::RAWBC, &tm_C, 0, t0, (int)b, bar);
        }
    };
    int bad = 0;
    if constexpr (TMA) {
        if (tid == 0) {
            for (int st = 0; st < S::STAGES; ++st) mbar_init(bar0 + 8 * st, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            for (int it = 0; it < S::STAGES && it < ntile; ++it) issue(it);
        }
    }

    const int g = lane / C::CW, c = lane % C::CW, cw = warp * C::CW + c;
    const int64_t d = d0 + cw;
    const bool cvalid = d < a.D;
    CLane<CG> s;
    bool small_a = false;
#pragma unroll
    for (int j = 0; j < CG; ++j) {
        const int n = g * CG + j;
        const bool ok = cvalid && n < N;
        const float ar = ok ? __ldg(a.A + (d * N + n) * 2) : -1.f;
        const float ai = ok ? __ldg(a.A + (d * N + n) * 2 + 1) : 0.f;
        const float m2 = ar * ar + ai * ai;
        small_a |= ok && m2 < kCSmallA * kCSmallA;
        comp(s.qr, j) = ar * kLog2e;
        comp(s.qi, j) = ai;
        const float inv = ok && m2 > 0.f ? 1.f / m2 : 0.f;
        comp(s.nr, j) = -ar * inv;  // -1 / a = (-ar + i ai) / |a|^2
        comp(s.ni, j) = ai * inv;
        const bool h0v = ok && a.h0;
        comp(s.hr, j) = h0v ? __ldg(a.h0 + ((b * a.D + d) * N + n) * 2) : 0.f;
        comp(s.hi, j) = h0v ? __ldg(a.h0 + ((b * a.D + d) * N + n) * 2 + 1) : 0.f;
    }
    // skip weight D of this lane's channel (the epilogue forms gate (y + D x))
    const float dskc = (!CKPT && a.Dskip && cvalid) ? __ldg(a.Dskip + d) : 0.f;
    if (TMA && tid == 0 && ntile > 0) bad = !mbar_wait(bar0, 0);
    const int flags = __syncthreads_or((small_a ? 1 : 0) | (bad ? 2 : 0));
    const bool acc = (flags & 1) != 0;
    bool failed = (flags & 2) != 0;
    const int nvalid = cvalid ? (N - g * CG < CG ? N - g * CG : CG) : 0;
    // phase-P channel pair of this thread (fixed: PAIRS is a multiple of the thread count)
    const int pc = 2 * (tid % (C::DC / 2));
    const int64_t pd = d0 + pc;
    const float2 pbias = make_float2((a.bias && pd < a.D) ? __ldg(a.bias + pd) : 0.f,
                                     (a.bias && pd + 1 < a.D) ? __ldg(a.bias + pd + 1) : 0.f);

    for (int it = 0; it < ntile && !failed; ++it) {
        const int64_t t0 = (int64_t)it * TT;
        const int tl = (int)(a.L - t0 < TT ? a.L - t0 : TT);
        const unsigned char* raw = ring + (it % S::STAGES) * S::STAGE;
        // phase P: (delta, x) pairs and the gate of two channels per thread and row, packed
#pragma unroll
        for (int qi = 0; qi < S::PAIRS / kCThreads; ++qi) {
            const int q = tid + qi * kCThreads;
            const int t = q / (C::DC / 2);
            float2 uv, rv, zv = make_float2(0.f, 0.f);
            if constexpr (TMA) {
                uv = to_f32x2(reinterpret_cast<const P2*>(raw)[q]);
                rv = to_f32x2(reinterpret_cast<const P2*>(raw + S::RAW)[q]);
                if (has_z) zv = to_f32x2(reinterpret_cast<const P2*>(raw + 2 * S::RAW)[q]);
            } else {
                const int64_t gi = (b * a.L + t0 + t) * a.D + pd;
                const bool v0 = t < tl && pd < a.D, v1 = t < tl && pd + 1 < a.D;
                uv = make_float2(v0 ? IO<T>::load(u, gi) : 0.f, v1 ? IO<T>::load(u, gi + 1) : 0.f);
                rv = make_float2(v0 ? IO<T>::load(dr, gi) : 0.f, v1 ? IO<T>::load(dr, gi + 1) : 0.f);
                if (has_z) zv = make_float2(v0 ? IO<T>::load(zz, gi) : 0.f, v1 ? IO<T>::load(zz, gi + 1) : 0.f);
            }
            const float2 x = a.input_silu ? silu_x2(uv) : uv;
            float2 dl = __fadd2_rn(rv, pbias);
            if (a.softplus) dl = softplus_x2(dl);
            const float2 gt = has_z ? silu_x2(zv) : make_float2(1.f, 1.f);
            reinterpret_cast<float4*>(sdx)[(t * C::DC + pc) / 2] = make_float4(dl.x, x.x, dl.y, x.y);
            reinterpret_cast<float2*>(sgt)[(t * C::DC + pc) / 2] = gt;
        }
        for (int e = tid; e < TT * C::NS; e += kCThreads) {
            const int t = e / C::NS, n = e % C::NS;
            float bv = 0.f, cv = 0.f;
            if (t < tl && n < N) {
                if (TMA && bc_tma) {
                    bv = to_f32<T>(reinterpret_cast<const T*>(raw + 3 * S::RAW)[t * N + n]);
                    cv = to_f32<T>(reinterpret_cast<const T*>(raw + 3 * S::RAW + S::RAWBC)[t * N + n]);
                } else {
                    const int64_t gi = (b * a.L + t0 + t) * N + n;
                    bv = IO<T>::load(Bg, gi);
                    cv = IO<T>::load(Cg, gi);
                }
            }
            sB[e] = bv;
            sC[e] = cv;
        }
        if constexpr (TMA) fence_proxy_async();
        // the previous tile's output store must have read the output tile
        if (kTileOut && tid == 0) tma_store_wait_read_0();
        __syncthreads();
        // the stage just consumed takes the tile two ahead
        if (TMA && tid == 0 && it + S::STAGES < ntile) issue(it + S::STAGES);
        T* const otile = reinterpret_cast<T*>(smem + S::OFF_OUT);
        T* out = CKPT ? nullptr : kTileOut ? otile + cw : static_cast<T*>(a.out) + (b * a.L + t0) * a.D + d;
        const int64_t ostride = kTileOut ? C::DC : a.D;
        float* ck = CKPT ? ckpt + (((b * nck + t0 / 8) * a.D + d) * N + g * CG) * 2 : nullptr;
        const int64_t ck_stride = a.D * N * 2;
        const bool wr = kTileOut || cvalid;  // the TMA store drops columns past D
        if (acc)
            scan_tile_c<T, NG, CG, TT, true, CKPT, false>(s, sdx, sgt, sB, sC, tl, g, cw, wr, out, ostride, dskc, ck,
                                                          ck_stride, nvalid);
        else if (!CKPT && tl == TT)
            scan_tile_c_pipe<T, NG, CG, TT>(s, sdx, sgt, sB, sC, g, cw, wr, out, ostride, dskc);
        else if (tl == TT)
            scan_tile_c<T, NG, CG, TT, false, CKPT, true>(s, sdx, sgt, sB, sC, tl, g, cw, wr, out, ostride, dskc, ck,
                                                          ck_stride, nvalid);
        else
            scan_tile_c<T, NG, CG, TT, false, CKPT, false>(s, sdx, sgt, sB, sC, tl, g, cw, wr, out, ostride, dskc, ck,
                                                           ck_stride, nvalid);
        if constexpr (kTileOut) fence_proxy_async();
        // the next tile's raw data (or a wait that gave up); shared memory free again
        if (TMA && tid == 0 && it + 1 < ntile)
            bad = !mbar_wait(bar0 + 8 * ((it + 1) % S::STAGES), ((it + 1) / S::STAGES) & 1);
        failed = __syncthreads_or(bad) != 0;
        if (kTileOut && tid == 0) tma_store_3d(&tm_out, (int)d0, (int)t0, (int)b, smem_u32(otile));
    }
    if (kTileOut && tid == 0) tma_store_wait_all();
    if (failed) {
        if (tid == 0) {
            atomicOr(&g_device_error_cx, 1u);
            // let the copies still in flight land before the CTA's shared memory is released
            for (int st = 0; st < S::STAGES; ++st) (void)mbar_wait(bar0 + 8 * st, 0), (void)mbar_wait(bar0 + 8 * st, 1);
        }
        return;
    }
    if (a.h_last && cvalid) {
#pragma unroll
        for (int j = 0; j < CG; ++j) {
            const int n = g * CG + j;
            if (n < N) {
                a.h_last[((b * a.D + d) * N + n) * 2] = comp(s.hr, j);
                a.h_last[((b * a.D + d) * N + n) * 2 + 1] = comp(s.hi, j);
            }
        }
    }
}

// 3-D map over a (batch, L, W) tensor, box [1][rows][box_w], zero fill outside.
template <typename T>
bool make_map_c(CUtensorMap* m, const void* base, int64_t batch, int64_t L, int64_t W, int box_w, int rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)(W * sizeof(T)), (cuuint64_t)(L * W * sizeof(T))};
    const cuuint32_t box[3] = {(cuuint32_t)box_w, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType ty =
        sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    return fn(m, ty, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16c(const void* q) { return q == nullptr || reinterpret_cast<uintptr_t>(q) % 16 == 0; }

template <typename T, int NG, int CG, int TT, bool CKPT, bool TMA>
cudaError_t launch_ck(const CUtensorMap (&m)[6], const ComplexArgs& a, float* ckpt, int64_t nck, int bc_tma,
                      int64_t blocks, cudaStream_t st) {
    using S = CSmem<T, NG, CG, TT>;
    auto kern = fwd_complex_kernel<T, NG, CG, TT, CKPT, TMA>;
    const int smem = TMA ? S::SMEM_TMA : S::SMEM_PLAIN;
    // function attributes are per device: set them once on each device used
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        configured[dev] = true;
    }
    kern<<<(unsigned)blocks, kCThreads, smem, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], a, ckpt, nck, bc_tma);
    return cudaGetLastError();
}

template <typename T, int NG, int CG, int TT>
cudaError_t launch_c_tt(const ComplexArgs& a, float* ckpt, int64_t nck, cudaStream_t st) {
    using C = CCfg<NG, CG>;
    const int64_t blocks = a.batch * ((a.D + C::DC - 1) / C::DC);
    if (blocks <= 0) return cudaGetLastError();
    // the TMA ring and the output store need 16-byte aligned bases and row pitches of the
    // (batch, L, D) tensors
    CUtensorMap m[6];
    bool tma = (a.D * (int64_t)sizeof(T)) % 16 == 0 && aligned16c(a.u) && aligned16c(a.delta_raw) &&
               aligned16c(a.z) && (ckpt != nullptr || aligned16c(a.out)) && a.L < (int64_t(1) << 31) &&
               a.D < (int64_t(1) << 31);
    int bc_tma = 0;
    if (tma) {
        tma = make_map_c<T>(&m[0], a.u, a.batch, a.L, a.D, C::DC, TT) &&
              make_map_c<T>(&m[1], a.delta_raw, a.batch, a.L, a.D, C::DC, TT) &&
              make_map_c<T>(&m[2], a.z ? a.z : a.u, a.batch, a.L, a.D, C::DC, TT) &&
              make_map_c<T>(&m[5], ckpt ? a.u : a.out, a.batch, a.L, a.D, C::DC, TT);
        // B and C rows by TMA when a row of N values is a whole number of 16-byte units
        if (tma && (a.N * (int64_t)sizeof(T)) % 16 == 0 && aligned16c(a.B) && aligned16c(a.C) &&
            make_map_c<T>(&m[3], a.B, a.batch, a.L, a.N, a.N, TT) && make_map_c<T>(&m[4], a.C ? a.C : a.B, a.batch, a.L, a.N, a.N, TT))
            bc_tma = 1;
        else
            m[3] = m[4] = m[0];
    }
    if (!tma) {
        std::memset(m, 0, sizeof m);
        return ckpt ? launch_ck<T, NG, CG, TT, true, false>(m, a, ckpt, nck, 0, blocks, st)
                    : launch_ck<T, NG, CG, TT, false, false>(m, a, nullptr, 0, 0, blocks, st);
    }
    return ckpt ? launch_ck<T, NG, CG, TT, true, true>(m, a, ckpt, nck, bc_tma, blocks, st)
                : launch_ck<T, NG, CG, TT, false, true>(m, a, nullptr, 0, bc_tma, blocks, st);
}

// Steps per tile: 64 when the whole grid fits the GPU at once with 64-step tiles, else 32
// (at the Mamba-130M shape, one ring stage: 0.491 ms with 32-step tiles, 0.483 with 64;
// with two stages 0.592 / 0.572 / 0.597 ms for 16 / 32 / 64 before the output tile).
template <typename T, int NG, int CG>
cudaError_t launch_c(const ComplexArgs& a, float* ckpt, int64_t nck, cudaStream_t st) {
    using C = CCfg<NG, CG>;
    const int64_t blocks = a.batch * ((a.D + C::DC - 1) / C::DC);
    const int64_t fit64 = kSmemPerSm / (CSmem<T, NG, CG, 64>::SMEM_TMA + kSmemPerCtaReserved);
    if (blocks <= fit64 * kSmCount) return launch_c_tt<T, NG, CG, 64>(a, ckpt, nck, st);
    return launch_c_tt<T, NG, CG, 32>(a, ckpt, nck, st);
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

cudaError_t read_device_error_cx(unsigned int* value, int clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error_cx, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error_cx, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace sscan
