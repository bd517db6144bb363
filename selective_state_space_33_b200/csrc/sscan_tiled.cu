// sscan_tiled.cu -- the fast forward kernel of the selective scan for sm_100a.
//
// Work decomposition.  A CTA owns one batch b, a block of DC consecutive channels
// and one sequence chunk; it walks the chunk in tiles of TT steps (16, 32 or 64:
// longer tiles where the grid leaves few CTAs per SM, see launch_geom).  Its four
// warps each own CW = 32/NG channels; the NG lanes of a channel each hold G = 4
// of the N <= 4*NG fp32 states in registers for the whole chunk (lane =
// g*CW + c), so the recurrence h_t = Abar h_{t-1} + Bbar x_t (sec. 2.1, eq. (3a))
// runs sequentially in t with no state ever leaving the SM (sec. 4.1).
//
// Per tile:
//   TMA 3-D loads bring the u, delta_raw (and z) tiles [TT x DC] into a 2-stage
//   shared-memory ring (mbarrier completion, one elected thread issues and waits,
//   every wait bounded);
//   phase P: all threads turn the raw tile into fp32 (delta, x) pairs and the SiLU
//   gate (softplus of sec. 3.2, Fig. 3), and stage the tile's B and C rows;
//   phase S: each lane advances its 4 states through the tile with packed f32x2
//   arithmetic (Abar = exp(delta A) on the MUFU pipe, Bbar from the same
//   exponential, eq. (2)); the partial readouts C.h of the NG lanes of a channel
//   are summed by a transposed butterfly so each lane finishes one step's output
//   (skip term and gate) into a shared tile that one TMA 3-D store writes back.
//
// Modes: kOut writes out (and h_last from the last chunk), kAgg writes each
// chunk's end state from zero plus its sum of delta (for the cross-chunk carry),
// kLast writes only h_last, kCkpt writes the state before every 8th step (the
// backward pass's recomputation starting points).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "sscan_check.cuh"
#include "sscan_launch.h"
#include "sscan_act.cuh"
#include "sscan_math.cuh"
#include "sscan_plan.h"
#include "sscan_tma.cuh"

namespace sscan {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kWarps = 4;     // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr float kSmallA = 9.765625e-4f;  // |A| below 2^-10 takes the series form of Bbar

enum { kOut = 0, kAgg = 1, kLast = 2, kCkpt = 3 };
constexpr int kCkStep = 8;  // steps between checkpoints written by kCkpt

template <typename T> struct Pair;
template <> struct Pair<float> {
    using type = float2;
    static __device__ __forceinline__ float2 f(float2 v) { return v; }
};
template <> struct Pair<__nv_bfloat16> {
    using type = __nv_bfloat162;
    static __device__ __forceinline__ float2 f(__nv_bfloat162 v) { return __bfloat1622float2(v); }
};

// Tile geometry for NG lanes per channel, G states per lane.  Raw-tile ring depth:
// one stage (the next tile's copy is issued once phase P has consumed the stage and
// lands during phase S), except for the backward's bf16 checkpoint pass, which runs
// beside other kernels and keeps two.  Measured, bf16: one stage 0.583 against
// 0.592 ms at the 2.8B-layer shape and 0.254 against 0.259 ms at the 130M shape;
// two stages for the checkpoint pass 1.374 against 1.386 ms per backward call.
template <typename T, int NG, int G, int MODE, int TT>
struct Cfg {
    static constexpr int CW = 32 / NG;                     // channels per warp
    static constexpr int DC = CW * kWarps;                 // channels per CTA
    static constexpr int NS = NG * G;                      // states covered (>= N)
    static constexpr int STAGES = (sizeof(T) == 2 && MODE == kCkpt) ? 2 : 1;
    static constexpr int RAW = TT * DC * (int)sizeof(T);  // bytes of one raw (batch, L, D) tile
    static constexpr int RAWBC = TT * NS * (int)sizeof(T);  // bytes reserved for one raw B or C tile
    static constexpr int STAGE = 3 * RAW + 2 * RAWBC;      // u, delta_raw, z, B, C
    static constexpr int BC_ENTRIES = TT * NS;
    static constexpr int PAIRS = TT * DC / 2;             // channel pairs of phase P
    static_assert(PAIRS % kThreads == 0, "phase P runs a fixed number of pairs per thread");
    // shared-memory layout (byte offsets, all 128-aligned)
    static constexpr int OFF_RAW = 0;                                     // [STAGES][STAGE]
    static constexpr int OFF_DX = OFF_RAW + STAGES * STAGE;               // float2 (delta, x) [TT][DC]
    static constexpr int OFF_GD = OFF_DX + TT * DC * 8;                  // float  gate [TT][DC]
    static constexpr int OFF_B = OFF_GD + TT * DC * 4;                   // float  [TT][NS]
    static constexpr int OFF_C = OFF_B + TT * NS * 4;                    // float  [TT][NS]
    static constexpr int OFF_OUT = OFF_C + TT * NS * 4;                  // [RAW] output tile
    static constexpr int OFF_BAR = OFF_OUT + RAW;                         // uint64 [STAGES]
    static constexpr int SMEM = OFF_BAR + STAGES * 8;
};

// Per lane: G states of one channel as G/2 f32x2 pairs, with A log2(e) and -1/A.
template <int G>
struct LaneG {
    float2 h[G / 2], A2[G / 2], niA[G / 2];
};

__device__ __forceinline__ float2 ex2x2(float2 q) { return f2(ex2(q.x), ex2(q.y)); }

// One step for the lane's G states, eq. (2) and (3a).  With v = -B x / A the update
// h' = Abar h + (Abar - 1) B x / A is Abar (h - v) + v: two packed fmas per pair
// (h - v as fma(v, -1, h), exact), no negated operand.  dx = (delta, x);
// Bp, Cp point at the lane's G values of B_t, C_t.  Returns the partial readout
// sum_j C_j h_j over these states (eq. (3b)).
template <int G, bool WANT_Y>
__device__ __forceinline__ float step_fast(LaneG<G>& s, float2 dx, const float* Bp, const float* Cp) {
    const float2 dd = f2(dx.x, dx.x), xx = f2(dx.y, dx.y);
    float2 y = f2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < G / 2; ++k) {
        const float2 Bv = reinterpret_cast<const float2*>(Bp)[k];
        const float2 a = ex2x2(__fmul2_rn(dd, s.A2[k]));
        const float2 v = __fmul2_rn(Bv, __fmul2_rn(xx, s.niA[k]));
        s.h[k] = __ffma2_rn(a, __ffma2_rn(v, f2(-1.f, -1.f), s.h[k]), v);
        if (WANT_Y) y = __ffma2_rn(reinterpret_cast<const float2*>(Cp)[k], s.h[k], y);
    }
    return WANT_Y ? y.x + y.y : 0.f;
}

// Accurate form for blocks with a small |A| (or A = 0): Bbar / B = delta phi1(delta A)
// with phi1's series near 0, as in the general kernels.
template <int G, bool WANT_Y>
__device__ __forceinline__ float step_acc(LaneG<G>& s, float2 dx, const float* Bp, const float* Cp) {
    const float delta = dx.x, x = dx.y;
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < G; ++j) {
        float2& hp = s.h[j / 2];
        const float A2 = (j & 1) ? s.A2[j / 2].y : s.A2[j / 2].x;
        const float iA = -((j & 1) ? s.niA[j / 2].y : s.niA[j / 2].x);
        const float q2 = delta * A2;
        const float abar = ex2(q2);
        const float beta = bbar_coef(delta, q2 * kLn2, abar, iA);
        float& hv = (j & 1) ? hp.y : hp.x;
        hv = fmaf(abar, hv, beta * Bp[j] * x);
        if (WANT_Y) y = fmaf(Cp[j], hv, y);
    }
    return WANT_Y ? y : 0.f;
}

// Sum the partial readouts of the NG lanes of a channel for NG consecutive steps
// so that lane g ends with the full sum for step g (transposed butterfly: each
// round halves the values a lane holds).
template <int NG, int CW>
__device__ __forceinline__ float transpose_reduce(float (&p)[NG], int g) {
    if constexpr (NG == 1) {
        return p[0];
    } else {
        float cur[NG];
#pragma unroll
        for (int j = 0; j < NG; ++j) cur[j] = p[j];
#pragma unroll
        for (int m = NG / 2; m >= 1; m /= 2) {
            const bool up = (g & m) != 0;
#pragma unroll
            for (int j = 0; j < m; ++j) {
                const float keep = up ? cur[m + j] : cur[j];
                const float send = up ? cur[j] : cur[m + j];
                cur[j] = keep + __shfl_xor_sync(0xffffffffu, send, m * CW);
            }
        }
        return cur[0];
    }
}

// Phase S over one tile, NG steps per block (the readouts of a block are reduced
// together); with outputs, two blocks per loop iteration so that one block's
// reduction overlaps the next block's steps.  FULL tiles (TT valid steps) need no per-step predicate;
// the last, partial tile of a chunk takes the predicated form.
template <typename T, int NG, int G, int MODE, int TT, bool ACC, bool FULL>
__device__ __forceinline__ void scan_tile(LaneG<G>& s, unsigned char* smem, int tile_len, int g, int cw, T* sout,
                                          float dskc, float& dsum, float* ck, int64_t ck_stride, int nvalid,
                                          const float* ck_base, int64_t ck_extent) {
    using C = Cfg<T, NG, G, MODE, TT>;
    constexpr bool WANT_Y = MODE == kOut;
    const float2* sdx = reinterpret_cast<const float2*>(smem + C::OFF_DX) + cw;
    const float* sgt = reinterpret_cast<const float*>(smem + C::OFF_GD) + cw;
    const float* sB = reinterpret_cast<const float*>(smem + C::OFF_B) + g * G;
    const float* sC = reinterpret_cast<const float*>(smem + C::OFF_C) + g * G;
#pragma unroll(MODE == kOut ? 2 : 1)
    for (int tb = 0; tb < TT; tb += NG) {
        if (MODE == kCkpt && tb % kCkStep == 0 && (FULL || tb < tile_len)) {
            // state before step tb, the starting point of one backward recomputation
            float* dst = ck + (tb / kCkStep) * ck_stride;
#pragma unroll
            for (int j = 0; j < G; ++j)
                if (j < nvalid && in_range(dst + j - ck_base, ck_extent)) dst[j] = (j & 1) ? s.h[j / 2].y : s.h[j / 2].x;
        }
        float p[NG];
#pragma unroll
        for (int k = 0; k < NG; ++k) {
            const int t = tb + k;
            p[k] = 0.f;
            if (FULL || t < tile_len) {
                const float2 dx = sdx[t * C::DC];
                if (MODE == kAgg) dsum += dx.x;
                p[k] = ACC ? step_acc<G, WANT_Y>(s, dx, sB + t * C::NS, sC + t * C::NS)
                           : step_fast<G, WANT_Y>(s, dx, sB + t * C::NS, sC + t * C::NS);
            }
        }
        if constexpr (WANT_Y) {
            const float y = transpose_reduce<NG, C::CW>(p, g);
            const int t = tb + g;
            if (FULL || t < tile_len) {
                sout[t * C::DC + cw] = from_f32<T>(sgt[t * C::DC] * fmaf(dskc, sdx[t * C::DC].y, y));
            }
        }
    }
}

// Full tiles of the fast form with outputs, software-pipelined: the exponentials and
// the v terms of step t+1 are issued before the state update of step t, so the MUFU
// latency of one step overlaps the dependent fmas of the previous one (measured
// 0.633 -> 0.620 ms at the 2.8B-layer shape, bf16; identical results).
template <int G>
struct Prep { float2 a[G / 2]; float2 v[G / 2]; };

template <int G>
__device__ __forceinline__ Prep<G> prep_step(const LaneG<G>& s, float2 dx, const float* Bp) {
    Prep<G> P;
    const float2 dd = f2(dx.x, dx.x), xx = f2(dx.y, dx.y);
#pragma unroll
    for (int k = 0; k < G / 2; ++k) {
        P.a[k] = ex2x2(__fmul2_rn(dd, s.A2[k]));
        P.v[k] = __fmul2_rn(reinterpret_cast<const float2*>(Bp)[k], __fmul2_rn(xx, s.niA[k]));
    }
    return P;
}

template <int G>
__device__ __forceinline__ float upd_step(LaneG<G>& s, const Prep<G>& P, const float* Cp) {
    float2 y = f2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < G / 2; ++k) {
        s.h[k] = __ffma2_rn(P.a[k], __ffma2_rn(P.v[k], f2(-1.f, -1.f), s.h[k]), P.v[k]);
        y = __ffma2_rn(reinterpret_cast<const float2*>(Cp)[k], s.h[k], y);
    }
    return y.x + y.y;
}

template <typename T, int NG, int G, int TT>
__device__ __forceinline__ void scan_tile_pipe(LaneG<G>& s, unsigned char* smem, int g, int cw, T* sout,
                                               float dskc) {
    using C = Cfg<T, NG, G, kOut, TT>;
    const float2* sdx = reinterpret_cast<const float2*>(smem + C::OFF_DX) + cw;
    const float* sgt = reinterpret_cast<const float*>(smem + C::OFF_GD) + cw;
    const float* sB = reinterpret_cast<const float*>(smem + C::OFF_B) + g * G;
    const float* sC = reinterpret_cast<const float*>(smem + C::OFF_C) + g * G;
    Prep<G> P = prep_step<G>(s, sdx[0], sB);
#pragma unroll
    for (int tb = 0; tb < TT; tb += NG) {
        float p[NG];
#pragma unroll
        for (int k = 0; k < NG; ++k) {
            const int t = tb + k;
            Prep<G> Pn = P;
            if (t + 1 < TT) Pn = prep_step<G>(s, sdx[(t + 1) * C::DC], sB + (t + 1) * C::NS);
            p[k] = upd_step<G>(s, P, sC + t * C::NS);
            P = Pn;
        }
        const float y = transpose_reduce<NG, C::CW>(p, g);
        const int t = tb + g;
        sout[t * C::DC + cw] = from_f32<T>(sgt[t * C::DC] * fmaf(dskc, sdx[t * C::DC].y, y));
    }
}
template <typename T, int NG, int G, int MODE, int TT, bool ACC>
__device__ __forceinline__ void scan_tile_any(LaneG<G>& s, unsigned char* smem, int tile_len, int g, int cw, T* sout,
                                              float dskc, float& dsum, float* ck, int64_t ck_stride, int nvalid,
                                              const float* ck_base, int64_t ck_extent) {
    if constexpr (MODE == kOut && !ACC) {
        if (tile_len == TT) {
            scan_tile_pipe<T, NG, G, TT>(s, smem, g, cw, sout, dskc);
            return;
        }
    }
    if (tile_len == TT)
        scan_tile<T, NG, G, MODE, TT, ACC, true>(s, smem, tile_len, g, cw, sout, dskc, dsum, ck, ck_stride, nvalid,
                                                 ck_base, ck_extent);
    else
        scan_tile<T, NG, G, MODE, TT, ACC, false>(s, smem, tile_len, g, cw, sout, dskc, dsum, ck, ck_stride, nvalid,
                                                  ck_base, ck_extent);
}

// Register budget (resident CTAs per SM the launch bound asks for): 9 for 4-state lanes,
// except with 64-step tiles, which are launched only when at most 4 CTAs per SM are needed
// and then get the registers of 4 (117, no spills: 0.2070 against 0.2107 ms at the
// Mamba-130M shape); 5 for the 8-state lanes.
template <int G, int TT> struct Occupancy { static constexpr int kCtas = G == 4 ? (TT == 64 ? 4 : 9) : 5; };

template <typename T, int NG, int G, int MODE, int TT>
__global__ void __launch_bounds__(kThreads, Occupancy<G, TT>::kCtas)
    fwd_tiled_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_dr,
                     const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_out,
                     const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                     TiledArgs a) {
    using C = Cfg<T, NG, G, MODE, TT>;
    using P2 = typename Pair<T>::type;
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t ncb = (a.D + C::DC - 1) / C::DC;
    const int64_t blk = blockIdx.x;
    const int cb = (int)(blk % ncb);
    const int64_t bc = blk / ncb;
    const int chunk = (int)(bc % a.nchunks);
    const int b = (int)(bc / a.nchunks);
    const int64_t t_begin = (int64_t)chunk * a.chunk_len;
    const int64_t t_end = min(a.L, t_begin + a.chunk_len);
    const int ntile = (int)((t_end - t_begin + TT - 1) / TT);
    const int N = a.N;
    const int d0 = cb * C::DC;
    constexpr bool want_out = MODE == kOut;
    // extents of the arrays indexed below (checked in the debug build only)
    const int64_t ext_state = a.batch * a.D * N, ext_chunks = a.batch * a.nchunks * a.D * N;
    const int64_t ext_ckpt = a.batch * a.nck * a.D * N;
    const bool has_z = want_out && a.has_z;
    const bool bc_tma = a.bc_tma != 0;
    const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
    const uint32_t raw_bytes = (has_z ? 3u : 2u) * C::RAW;
    const uint32_t bc_bytes = (uint32_t)(TT * N * (int)sizeof(T));
    const uint32_t stage_bytes = raw_bytes + (bc_tma ? (want_out ? 2u : 1u) * bc_bytes : 0u);

    // issue the TMA copies of tile `it` into its ring stage (elected thread only)
    auto issue = [&](int it) {
        const int st = it % C::STAGES;
        const uint32_t bar = bar0 + 8 * st;
        const uint32_t base = smem_u32(smem + C::OFF_RAW + st * C::STAGE);
        const int tt = (int)(t_begin + (int64_t)it * TT);
        mbar_expect_tx(bar, stage_bytes);
        tma_load_3d(base, &tm_u, d0, tt, b, bar);
        tma_load_3d(base + C::RAW, &tm_dr, d0, tt, b, bar);
        if (has_z) tma_load_3d(base + 2 * C::RAW, &tm_z, d0, tt, b, bar);
        if (bc_tma) {
            tma_load_3d(base + 3 * C::RAW, &tm_B, 0, tt, b, bar);
            if (want_out) tma_load_3d(base + 3 * C::RAW + C::RAWBC, &tm_C, 0, tt, b, bar);
        }
    };

    int bad = 0;
    if (tid == 0) {
        for (int st = 0; st < C::STAGES; ++st) mbar_init(bar0 + 8 * st, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int it = 0; it < C::STAGES && it < ntile; ++it) issue(it);
    }

    // per-lane state: channel cw of this CTA, states g*G .. g*G+G-1
    const int g = lane / C::CW, c = lane % C::CW, cw = warp * C::CW + c;
    const int64_t d = d0 + cw;
    const bool cvalid = d < a.D;
    LaneG<G> s;
    bool small_a = false;
#pragma unroll
    for (int j = 0; j < G; ++j) {
        const int n = g * G + j;
        const bool ok = cvalid && n < N;
        const float An = ok && in_range(d * N + n, a.D * N) ? __ldg(a.A + d * N + n) : -1.f;
        small_a |= ok && fabsf(An) < kSmallA;
        float h = 0.f;
        if (ok && MODE != kAgg) {
            const int64_t ic = (((int64_t)b * a.nchunks + chunk) * a.D + d) * N + n;
            const int64_t is = ((int64_t)b * a.D + d) * N + n;
            if (a.nchunks > 1) h = in_range(ic, ext_chunks) ? a.ws_state[ic] : 0.f;
            else if (a.h0) h = in_range(is, ext_state) ? __ldg(a.h0 + is) : 0.f;
        }
        const float A2 = ok ? An * kLog2e : 0.f;
        const float niA = ok && An != 0.f ? -1.f / An : 0.f;
        if (j & 1) {
            s.h[j / 2].y = h;
            s.A2[j / 2].y = A2;
            s.niA[j / 2].y = niA;
        } else {
            s.h[j / 2].x = h;
            s.A2[j / 2].x = A2;
            s.niA[j / 2].x = niA;
        }
    }
    // the first tile's data; one CTA-wide choice of the Bbar form (block-uniform branch)
    if (tid == 0 && ntile > 0) bad = !mbar_wait(bar0, 0);
    const int flags = __syncthreads_or((small_a ? 1 : 0) | (bad ? 2 : 0));
    const bool acc = (flags & 1) != 0;
    bool failed = (flags & 2) != 0;

    // phase-P channel pair of this thread (fixed, since kThreads is a multiple of DC/2)
    const int pc = 2 * (tid % (C::DC / 2));
    const int64_t pd = d0 + pc;
    // skip weight D of this lane's channel (the epilogue forms gate * (y + D x))
    const float dskc = (want_out && a.Dskip && cvalid) ? __ldg(a.Dskip + d) : 0.f;
    const T* Bg = static_cast<const T*>(a.B);
    const T* Cg = static_cast<const T*>(a.C);
    float dsum = 0.f;
    const float2 pbias = f2((a.bias && pd < a.D) ? __ldg(a.bias + pd) : 0.f,
                            (a.bias && pd + 1 < a.D) ? __ldg(a.bias + pd + 1) : 0.f);

    for (int it = 0; it < ntile && !failed; ++it) {
        const int st = it % C::STAGES;
        const int64_t tt = t_begin + (int64_t)it * TT;
        const int tile_len = (int)(t_end - tt < TT ? t_end - tt : TT);
        // phase P: raw tile -> (delta, x) pairs and (gate, D x gate); B and C rows as fp32
        {
            const unsigned char* raw = smem + C::OFF_RAW + st * C::STAGE;
            const P2* ru = reinterpret_cast<const P2*>(raw);
            const P2* rd = reinterpret_cast<const P2*>(raw + C::RAW);
            const P2* rz = reinterpret_cast<const P2*>(raw + 2 * C::RAW);
            float4* sdx = reinterpret_cast<float4*>(smem + C::OFF_DX);
            float2* sgt = reinterpret_cast<float2*>(smem + C::OFF_GD);
            // a fixed trip count (PAIRS is a multiple of kThreads for every geometry)
#pragma unroll
            for (int qi = 0; qi < C::PAIRS / kThreads; ++qi) {
                const int q = tid + qi * kThreads;
                const int t = q / (C::DC / 2);
                float2 x = Pair<T>::f(ru[q]);
                if (a.input_silu) x = silu_x2(x);
                float2 dl = __fadd2_rn(Pair<T>::f(rd[q]), pbias);
                if (a.softplus) dl = softplus_x2(dl);
                sdx[(t * C::DC + pc) / 2] = make_float4(dl.x, x.x, dl.y, x.y);
                if (want_out) {
                    const float2 gt = has_z ? silu_x2(Pair<T>::f(rz[q])) : f2(1.f, 1.f);
                    sgt[(t * C::DC + pc) / 2] = gt;
                }
            }
            float* sBf = reinterpret_cast<float*>(smem + C::OFF_B);
            float* sCf = reinterpret_cast<float*>(smem + C::OFF_C);
            const T* rB = reinterpret_cast<const T*>(raw + 3 * C::RAW);
            const T* rC = reinterpret_cast<const T*>(raw + 3 * C::RAW + C::RAWBC);
            if (bc_tma && N == C::NS) {
                // dense [TT][N] tiles: 4-value groups, those of B (0 .. V-1) then of C
                // (V .. 2V-1), one per thread per round
                constexpr int V = C::BC_ENTRIES / 4;
                static_assert((2 * V) % kThreads == 0 || 2 * V < kThreads, "whole rounds of 4-value groups");
#pragma unroll
                for (int gq = tid; gq < 2 * V; gq += kThreads) {
                const int which = gq / V, v = gq % V;
                if (which == 0 || (which == 1 && want_out)) {
                    const T* src = which ? rC : rB;
                    float4 f;
                    if constexpr (sizeof(T) == 4) {
                        f = reinterpret_cast<const float4*>(src)[v];
                    } else {
                        const uint2 w = reinterpret_cast<const uint2*>(src)[v];
                        f = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                                        __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
                    }
                    reinterpret_cast<float4*>(which ? sCf : sBf)[v] = f;
                }
                }
            } else {
#pragma unroll
                for (int ei = 0; ei < (C::BC_ENTRIES + kThreads - 1) / kThreads; ++ei) {
                    const int e = tid + ei * kThreads;
                    if (C::BC_ENTRIES % kThreads != 0 && e >= C::BC_ENTRIES) break;
                    const int t = e / C::NS, n = e % C::NS;
                    float bv = 0.f, cv = 0.f;
                    if (n < N) {
                        if (bc_tma) {
                            bv = to_f32<T>(rB[t * N + n]);
                            if (want_out) cv = to_f32<T>(rC[t * N + n]);
                        } else if (tt + t < t_end) {
                            const int64_t gi = ((int64_t)b * a.L + tt + t) * N + n;
                            if (in_range(gi, a.batch * a.L * N)) {
                                bv = to_f32<T>(Bg[gi]);
                                if (want_out) cv = to_f32<T>(Cg[gi]);
                            }
                        }
                    }
                    sBf[e] = bv;
                    if (want_out) sCf[e] = cv;
                }
            }
        }
        fence_proxy_async();
        // the previous tile's output store must have read the one output tile
        if (want_out && tid == 0) tma_store_wait_read_0();
        __syncthreads();
        if (tid == 0 && it + C::STAGES < ntile) issue(it + C::STAGES);
        // phase S
        T* sout = reinterpret_cast<T*>(smem + C::OFF_OUT);
        float* ck = nullptr;
        if (MODE == kCkpt)
            ck = a.ws_ckpt + ((((int64_t)b * a.nck) + tt / kCkStep) * a.D + d) * N + g * G;
        const int64_t ck_stride = (int64_t)a.D * N;
        const int nvalid = cvalid ? min(G, N - g * G) : 0;
        if (acc)
            scan_tile_any<T, NG, G, MODE, TT, true>(s, smem, tile_len, g, cw, sout, dskc, dsum, ck, ck_stride, nvalid,
                                                a.ws_ckpt, ext_ckpt);
        else
            scan_tile_any<T, NG, G, MODE, TT, false>(s, smem, tile_len, g, cw, sout, dskc, dsum, ck, ck_stride, nvalid,
                                                 a.ws_ckpt, ext_ckpt);
        if (want_out) fence_proxy_async();
        // the next tile's data, then one barrier for: outputs complete, tile buffers free,
        // next raw tile landed (or a wait that gave up)
        if (tid == 0 && it + 1 < ntile)
            bad = !mbar_wait(bar0 + 8 * ((it + 1) % C::STAGES), ((it + 1) / C::STAGES) & 1);
        failed = __syncthreads_or(bad) != 0;
        if (want_out && tid == 0) tma_store_3d(&tm_out, d0, (int)tt, b, smem_u32(sout));
    }
    if (tid == 0 && want_out) tma_store_wait_all();
    if (failed) {
        if (tid == 0) {
            atomicOr(&g_device_error, 1u);
            // let the loads still in flight land before the CTA's shared memory is released
            for (int st = 0; st < C::STAGES; ++st) (void)mbar_wait(bar0 + 8 * st, 0), (void)mbar_wait(bar0 + 8 * st, 1);
        }
        return;
    }
    // final state of this chunk
#pragma unroll
    for (int j = 0; j < G; ++j) {
        const int n = g * G + j;
        if (!cvalid || n >= N) continue;
        const float hf = (j & 1) ? s.h[j / 2].y : s.h[j / 2].x;
        const int64_t ic = (((int64_t)b * a.nchunks + chunk) * a.D + d) * N + n;
        const int64_t is = ((int64_t)b * a.D + d) * N + n;
        if (MODE == kAgg) {
            if (in_range(ic, ext_chunks)) a.ws_state[ic] = hf;
        } else if (a.h_last && chunk == a.nchunks - 1) {
            if (in_range(is, ext_state)) a.h_last[is] = hf;
        }
    }
    const int64_t idsum = ((int64_t)b * a.nchunks + chunk) * a.D + d;
    if (MODE == kAgg && g == 0 && cvalid && in_range(idsum, a.batch * a.nchunks * a.D)) a.ws_dsum[idsum] = dsum;
}

// --------------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D map over a (batch, L, D) tensor, box [1][TT][DC], zero fill outside.
template <typename T>
bool make_map(CUtensorMap* m, const void* base, int64_t batch, int64_t L, int64_t D, int DC, int TT) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)(D * sizeof(T)), (cuuint64_t)(L * D * sizeof(T))};
    const cuuint32_t box[3] = {(cuuint32_t)DC, (cuuint32_t)TT, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType ty =
        sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    return fn(m, ty, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B and C (batch, L, N) travel by TMA when a row of N values is a whole number of
// 16-byte units; otherwise phase P reads them with plain loads.
template <typename T>
bool bc_by_tma(const TiledArgs& a) {
    return (a.N * sizeof(T)) % 16 == 0 && reinterpret_cast<uintptr_t>(a.B) % 16 == 0 &&
           (a.C == nullptr || reinterpret_cast<uintptr_t>(a.C) % 16 == 0);
}

template <typename T, int NG, int G, int MODE, int TT>
cudaError_t launch_mode(const TiledArgs& args, const TiledPtrs& p, cudaStream_t st) {
    using C = Cfg<T, NG, G, MODE, TT>;
    TiledArgs a = args;
    a.bc_tma = bc_by_tma<T>(a) ? 1 : 0;
    CUtensorMap mu, md, mz, mo, mb, mc;
    const void* zsrc = p.z ? p.z : p.u;      // an unused map still needs a valid address
    const void* osrc = p.out ? p.out : p.u;
    if (!make_map<T>(&mu, p.u, a.batch, a.L, a.D, C::DC, TT) || !make_map<T>(&md, p.delta_raw, a.batch, a.L, a.D, C::DC, TT) ||
        !make_map<T>(&mz, zsrc, a.batch, a.L, a.D, C::DC, TT) || !make_map<T>(&mo, osrc, a.batch, a.L, a.D, C::DC, TT))
        return cudaErrorInvalidValue;
    if (a.bc_tma) {
        if (!make_map<T>(&mb, a.B, a.batch, a.L, a.N, a.N, TT) ||
            !make_map<T>(&mc, a.C ? a.C : a.B, a.batch, a.L, a.N, a.N, TT))
            return cudaErrorInvalidValue;
    } else {
        mb = mu;
        mc = mu;
    }
    auto kern = fwd_tiled_kernel<T, NG, G, MODE, TT>;
    // function attributes are per device: set them once on each device used
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        configured[dev] = true;
    }
    const int64_t ncb = (a.D + C::DC - 1) / C::DC;
    const int64_t blocks = a.batch * a.nchunks * ncb;
    kern<<<(unsigned)blocks, kThreads, C::SMEM, st>>>(mu, md, mz, mo, mb, mc, a);
    return cudaGetLastError();
}

// Steps per tile.  Each tile costs two CTA-wide barriers and one phase P whose latency
// the other CTAs of the SM must hide; longer tiles halve that per step but need more
// shared memory, so fewer CTAs fit an SM.  Measured (bf16 / fp32 I/O, ms per launch,
// tiles of 16 / 32 / 64 steps): Mamba-130M layer 0.255 / 0.225 / 0.214 and 0.252 / 0.223 /
// 0.299; Mamba-2.8B layer 0.587 / 0.556 / 0.622 and 0.573 / 0.565 / 0.774; the million-step
// split 20.9 / 19.6 / 21.6.  So 64 when the whole grid fits the GPU at once with 64-step
// tiles, else 32.  The backward's checkpoint pass runs beside the reverse kernel's summary
// pass; launched before it, it takes 32 (backward call 1.254 ms with 16-step tiles, 1.204 ms
// with 32; 64-step tiles of the two-stage checkpoint ring need 76 KB).
template <typename T, int NG, int G>
cudaError_t launch_geom(const TiledArgs& a, const TiledPtrs& p, int mode, cudaStream_t st) {
    if (mode == kTiledCkpt) return launch_mode<T, NG, G, kCkpt, 32>(a, p, st);
    const int64_t ctas = a.batch * a.nchunks * ((a.D + 32 / NG * kWarps - 1) / (32 / NG * kWarps));
    const int64_t fit64_smem = kSmemPerSm / (Cfg<T, NG, G, kOut, 64>::SMEM + kSmemPerCtaReserved);
    const int64_t fit64 = fit64_smem < Occupancy<G, 64>::kCtas ? fit64_smem : Occupancy<G, 64>::kCtas;
    if (ctas <= fit64 * kSmCount) {
        if (mode == kTiledOut) return launch_mode<T, NG, G, kOut, 64>(a, p, st);
        if (mode == kTiledAgg) return launch_mode<T, NG, G, kAgg, 64>(a, p, st);
        return launch_mode<T, NG, G, kLast, 64>(a, p, st);
    }
    if (mode == kTiledOut) return launch_mode<T, NG, G, kOut, 32>(a, p, st);
    if (mode == kTiledAgg) return launch_mode<T, NG, G, kAgg, 32>(a, p, st);
    return launch_mode<T, NG, G, kLast, 32>(a, p, st);
}

template <typename T>
cudaError_t launch_t(const TiledArgs& a, const TiledPtrs& p, const TiledGeom& geo, int mode, cudaStream_t st) {
    if (geo.NG == 1) return launch_geom<T, 1, 4>(a, p, mode, st);
    if (geo.NG == 2) return launch_geom<T, 2, 4>(a, p, mode, st);
    return launch_geom<T, 4, 4>(a, p, mode, st);
}

}  // namespace

// Lane geometry: four states per lane, NG = ceil(N / 4) lanes per channel.  (Eight
// states per lane halve the per-step overheads but halve the warps; at the Mamba
// layer shapes that left too few warps per sub-partition to hide latency, and it
// measured slower.  Two states per lane double the warps, more than the 2.8B-layer
// grid can hold in one wave, and measured slower at both layer shapes.)
TiledGeom tiled_geometry(int64_t batch, int64_t L, int64_t D, int64_t N) {
    (void)batch;
    (void)L;
    (void)D;
    const int ng = N <= 4 ? 1 : (N <= 8 ? 2 : 4);
    return TiledGeom{ng, 4, 32 / ng * kWarps};
}

cudaError_t launch_fwd_tiled(const TiledArgs& a, const TiledPtrs& p, const TiledGeom& geo, int io_bf16, int mode,
                             cudaStream_t st) {
    if (!encode_fn()) return cudaErrorNotSupported;
    return io_bf16 ? launch_t<__nv_bfloat16>(a, p, geo, mode, st) : launch_t<float>(a, p, geo, mode, st);
}

namespace {
// The failure path of a bounded wait, exercised on purpose: an mbarrier with one
// expected arrival that never comes.  Nothing is in flight on it, so giving up
// leaves nothing behind.
__global__ void wait_probe_kernel(unsigned int polls) {
    __shared__ __align__(8) unsigned long long bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait(b, 0, polls)) atomicOr(&g_device_error, 4u);
}
}  // namespace

cudaError_t launch_wait_probe(unsigned int polls, cudaStream_t st) {
    wait_probe_kernel<<<1, 32, 0, st>>>(polls);
    return cudaGetLastError();
}

cudaError_t read_device_error(unsigned int* value, int clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace sscan
