// sscan_bwd_tiled.cu -- backward of the selective scan for sm_100a, with the states
// recomputed on chip (Mamba technical summary page, sec. 4.1 item 3).
//
// A forward pass in checkpoint mode (sscan_tiled.cu) first stores the state before
// every 8th step.  This kernel then walks each (batch, 32-channel) block through
// the sequence in reverse, 8 steps (one tile) at a time:
//   TMA brings u, delta_raw, z, dout and the B, C rows of the tile into a 2-stage
//   ring (bounded mbarrier waits);
//   phase P turns them into fp32 operand pairs (delta, delta, x, x) and (dy, dy)
//   plus the epilogue terms -- dy = dout SiLU(z),
//   dz factor = dout SiLU'(z), softplus' = sigmoid(r), SiLU'(u) with the input
//   activation -- with packed f32x2 arithmetic;
//   each lane recomputes its 4 states through the tile from the checkpoint,
//   keeping h_t in shared memory, then runs the adjoint recurrence backwards:
//     lam_t = C_t dy_t + Abar_{t+1} lam_{t+1}
//     w     = delta^2 psi(delta A),  psi(q) = (q e^q - expm1(q)) / q^2
//             (its Taylor series for |q| < 1/2, where the closed form cancels;
//             (1 + Abar (q - 1)) / A^2 elsewhere)
//     lam beta = delta lam Abar - A lam w        (beta = Bbar / B = delta Abar - A w)
//     dx   += lam beta B,   dB += lam beta x,   dC += dy h_t
//     d delta += lam Abar (A h_{t-1} + B x)
//     dA   += delta lam Abar h_{t-1} + lam w B x
//   so one evaluation of w per state gives both beta and the A-gradient term;
//   the per-element sums over a channel's lanes use transposed shuffle butterflies,
//   and the (t, n) sums of dB, dC over a warp's channels a padded shared-memory
//   transpose, before anything touches global memory.
// dB and dC of a tile are summed across the CTA's warps in shared memory (shared
// atomic adds) and then added to fp32 accumulators in global memory; dA, dD and the bias
// gradient are per-channel sums added once at the end.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "sscan_launch.h"
#include "sscan_affine.cuh"
#include "sscan_check.cuh"
#include "sscan_math.cuh"
#include "sscan_tma.cuh"

namespace sscan {

__device__ unsigned int g_device_error_bwd = 0;

namespace {

constexpr int kTB = 8;  // steps per tile (= checkpoint spacing of the forward kernel)
constexpr float kSmallAB = 9.765625e-4f;  // |A| below 2^-10: the recomputation takes the series form
constexpr int kWarpsB = 4;
constexpr int kThreadsB = kWarpsB * 32;

__device__ __forceinline__ float2 g2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 ex2p(float2 q) { return g2(ex2(q.x), ex2(q.y)); }

template <typename T> struct BPair;
template <> struct BPair<float> {
    using type = float2;
    static __device__ __forceinline__ float2 f(float2 v) { return v; }
};
template <> struct BPair<__nv_bfloat16> {
    using type = __nv_bfloat162;
    static __device__ __forceinline__ float2 f(__nv_bfloat162 v) { return __bfloat1622float2(v); }
};

template <typename T, int NG>
struct BCfg {
    static constexpr int CW = 32 / NG;                    // channels per warp
    static constexpr int DC = CW * kWarpsB;               // channels per CTA
    static constexpr int NS = NG * 4;                     // states covered
    static constexpr int RAW = kTB * DC * (int)sizeof(T);
    static constexpr int RAWBC = kTB * NS * (int)sizeof(T);
    static constexpr int STAGE = 4 * RAW + 2 * RAWBC;     // u, delta_raw, z, dout, B, C
    static constexpr int STAGES = 2;
    static constexpr int PAIRS = kTB * DC / 2;
    static_assert(PAIRS % kThreadsB == 0, "phase P runs a fixed number of channel pairs per thread");
    // dB / dC transpose (NG == 4): per warp, NG rows of CW lanes x 8 values, rows padded to
    // 8 (CW + 1) floats so that the column reads of a warp hit 32 distinct banks
    static constexpr int TR_ROW = 8 * (CW + 1);
    static constexpr int TR_WARP = NG * TR_ROW;
    static constexpr int OFF_RAW = 0;
    static constexpr int OFF_DX = OFF_RAW + STAGES * STAGE;     // float4 (d, d, x, x)      [kTB][DC]
    static constexpr int OFF_DY = OFF_DX + kTB * DC * 16;       // float2 (dy, dy)          [kTB][DC]
    static constexpr int OFF_EP = OFF_DY + kTB * DC * 8;        // float4 (D dy, dzf, sr, D x) [kTB][DC]
    static constexpr int OFF_SU = OFF_EP + kTB * DC * 16;       // float  SiLU'(u)          [kTB][DC]
    static constexpr int OFF_B = OFF_SU + kTB * DC * 4;         // float [kTB][NS]
    static constexpr int OFF_C = OFF_B + kTB * NS * 4;          // float [kTB][NS]
    static constexpr int OFF_HS = OFF_C + kTB * NS * 4;         // float4 [kTB][kThreadsB] recomputed states
    static constexpr int OFF_TR = OFF_HS + kTB * kThreadsB * 16;  // float [warp][TR_WARP]
    static constexpr int OFF_ACC = OFF_TR + (NG == 4 ? kWarpsB * TR_WARP * 4 : 0);  // float [kTB][NS][2]
    static constexpr int OFF_OUT = OFF_ACC + kTB * NS * 2 * 4;  // [2 buffers][3 tensors][RAW]
    static constexpr int OFF_BAR = OFF_OUT + 2 * 3 * RAW;
    static constexpr int SMEM = OFF_BAR + STAGES * 8;
    // the summary pass uses the ring, the (delta, dy) operands and C only: its barriers
    // follow C and its launch asks for that much shared memory
    static constexpr int OFF_BAR_SUM = OFF_HS;
    static constexpr int SMEM_SUM = OFF_BAR_SUM + STAGES * 8;
};

// Transposed butterfly over the NG lanes of a channel (lane bits at multiples of CW),
// as in the forward kernel: lane g ends with the full sum for step g of the block.
template <int NG, int CW>
__device__ __forceinline__ float treduce_g(float (&p)[NG], int g) {
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

// Sum 8 values over the CW channel lanes of a warp (the low lane bits): three
// transposed rounds leave value (c & 7) in lane c summed over 8 lanes, then plain
// rounds fold the remaining channel bits.
template <int CW>
__device__ __forceinline__ float treduce_c8(float (&v)[8], int c) {
    float cur[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) cur[j] = v[j];
#pragma unroll
    for (int m = 4; m >= 1; m /= 2) {
        const bool up = (c & m) != 0;
#pragma unroll
        for (int j = 0; j < m; ++j) {
            const float keep = up ? cur[m + j] : cur[j];
            const float send = up ? cur[j] : cur[m + j];
            cur[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    float r = cur[0];
#pragma unroll
    for (int m = 8; m < CW; m *= 2) r += __shfl_xor_sync(0xffffffffu, r, m);
    return r;
}

// beta = Bbar / B = expm1(delta A) / A for two states: delta phi1(q) by its series
// for |q| < 1/16, (Abar - 1) / A otherwise (the same regions as sscan::bbar_coef).
__device__ __forceinline__ float2 bbar2(float2 dd, float2 A2, float2 iA) {
    const float2 q2 = __fmul2_rn(dd, A2);
    const float2 q = __fmul2_rn(q2, g2(kLn2, kLn2));
    const float2 bl = __fmul2_rn(__fadd2_rn(ex2p(q2), g2(-1.f, -1.f)), iA);
    float2 ph = __ffma2_rn(q, g2(1.f / 120.f, 1.f / 120.f), g2(1.f / 24.f, 1.f / 24.f));
    ph = __ffma2_rn(ph, q, g2(1.f / 6.f, 1.f / 6.f));
    ph = __ffma2_rn(ph, q, g2(0.5f, 0.5f));
    ph = __ffma2_rn(ph, q, g2(1.f, 1.f));
    const float2 bs = __fmul2_rn(dd, ph);
    return g2(fabsf(q.x) < 0.0625f ? bs.x : bl.x, fabsf(q.y) < 0.0625f ? bs.y : bl.y);
}

// softplus(r) and its derivative sigmoid(r) for two values, from one exponential
// u = e^r each, in the three regions of sscan::softplus: r > 20: r; u < 2^-5: the
// log1p series u - u^2/2 + ... + u^5/5 (lg2.approx near 1 carries an absolute,
// not a relative, error); else ln2 log2(1 + u).  sigmoid(r) = u / (1 + u).
__device__ __forceinline__ void softplus_sig_x2(float2 r, float2& sp, float2& sg) {
    const float2 u = ex2p(g2(fminf(r.x, 20.f) * kLog2e, fminf(r.y, 20.f) * kLog2e));
    float2 ser = __ffma2_rn(u, g2(0.2f, 0.2f), g2(-0.25f, -0.25f));
    ser = __ffma2_rn(ser, u, g2(1.f / 3.f, 1.f / 3.f));
    ser = __ffma2_rn(ser, u, g2(-0.5f, -0.5f));
    ser = __ffma2_rn(ser, u, g2(1.f, 1.f));
    ser = __fmul2_rn(ser, u);
    const float2 w = __fadd2_rn(u, g2(1.f, 1.f));
    const float2 lg = __fmul2_rn(g2(lg2(w.x), lg2(w.y)), g2(kLn2, kLn2));
    const float vx = u.x < 0.03125f ? ser.x : lg.x, vy = u.y < 0.03125f ? ser.y : lg.y;
    sp = g2(r.x > 20.f ? r.x : vx, r.y > 20.f ? r.y : vy);
    sg = __fmul2_rn(u, g2(rcp(w.x), rcp(w.y)));
}

__device__ __forceinline__ float2 sigmoid_x2(float2 z) {
    const float2 d = __fadd2_rn(ex2p(__fmul2_rn(z, g2(-kLog2e, -kLog2e))), g2(1.f, 1.f));
    return g2(rcp(d.x), rcp(d.y));
}

// w = delta^2 psi(q) for two states, q = delta A = q2 ln 2, psi(q) = (q e^q - expm1(q)) / q^2.
//   |q| < 1/2 : the Taylor series sum_k (k+1)/(k+2)! q^k through q^6 (dropped tail below
//               2e-7 q^7, ~5e-7 relative), written in q2 = q log2(e);
//   otherwise : (1 + Abar (q - 1)) / A^2 from Abar = e^q; 1 + Abar (q - 1) = q^2 psi(q)
//               >= 0.09 there, so the subtraction costs about 1e-6 relative.
__device__ __forceinline__ float2 wpsi_x2(float2 q2, float2 ab, float2 d2, float2 iA2) {
    constexpr float l1 = 0.6931471805599453f, l2 = l1 * l1, l3 = l2 * l1, l4 = l3 * l1, l5 = l4 * l1, l6 = l5 * l1;
    float2 ps = __ffma2_rn(q2, g2(l6 / 5760.f, l6 / 5760.f), g2(l5 / 840.f, l5 / 840.f));
    ps = __ffma2_rn(ps, q2, g2(l4 / 144.f, l4 / 144.f));
    ps = __ffma2_rn(ps, q2, g2(l3 / 30.f, l3 / 30.f));
    ps = __ffma2_rn(ps, q2, g2(l2 / 8.f, l2 / 8.f));
    ps = __ffma2_rn(ps, q2, g2(l1 / 3.f, l1 / 3.f));
    ps = __ffma2_rn(ps, q2, g2(0.5f, 0.5f));
    const float2 ws = __fmul2_rn(d2, ps);
    const float2 qm1 = __ffma2_rn(q2, g2(l1, l1), g2(-1.f, -1.f));
    const float2 wc = __fmul2_rn(__ffma2_rn(ab, qm1, g2(1.f, 1.f)), iA2);
    constexpr float kT = 0.5f * 1.4426950408889634f;  // |q| = 1/2 in log2 units
    return g2(fabsf(q2.x) < kT ? ws.x : wc.x, fabsf(q2.y) < kT ? ws.y : wc.y);
}

// Per-lane constants and accumulators of the reverse sweep for its 4 states (2 pairs).
struct RevLane {
    float2 A2[2];    // A log2(e)
    float2 niA[2];   // -1 / A (0 when A == 0)
    float2 nA[2];    // -A
    float2 iA2[2];   // 1 / A^2 (0 when A == 0)
    float2 lam[2];   // Abar_{t+1} lam_{t+1}
    float2 P1[2];    // sum_t delta lam Abar h_{t-1}
    float2 P2[2];    // sum_t lam w B x
};

// One reverse step for the lane's 4 states.  dx = (d, d, x, x), dy2 = (dy, dy),
// Bv / Cv the lane's 4 values of B_t / C_t, hc = h_t, hp = h_{t-1}.  Returns the
// lane's partial sums for du, d delta, and the readout y_t; writes its dB, dC values.
__device__ __forceinline__ void rev_step(RevLane& s, float4 dx, float2 dyy, float4 Bv, float4 Cv, float4 hc,
                                         float4 hp, float& pdu, float& pdd, float& py, float (&vbc)[8]) {
    const float2 dd = g2(dx.x, dx.y), xx = g2(dx.z, dx.w), d2 = __fmul2_rn(dd, dd);
    const float2 Bp[2] = {g2(Bv.x, Bv.y), g2(Bv.z, Bv.w)};
    const float2 Cp[2] = {g2(Cv.x, Cv.y), g2(Cv.z, Cv.w)};
    const float2 hcv[2] = {g2(hc.x, hc.y), g2(hc.z, hc.w)};
    const float2 hpv[2] = {g2(hp.x, hp.y), g2(hp.z, hp.w)};
    float2 du2 = g2(0.f, 0.f), S1 = g2(0.f, 0.f), S2 = g2(0.f, 0.f), y2 = g2(0.f, 0.f);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const float2 q2 = __fmul2_rn(dd, s.A2[p]);
        const float2 ab = ex2p(q2);
        const float2 l = __ffma2_rn(Cp[p], dyy, s.lam[p]);
        const float2 la = __fmul2_rn(l, ab);
        const float2 w = wpsi_x2(q2, ab, d2, s.iA2[p]);
        const float2 m = __fmul2_rn(l, w);
        const float2 lb = __ffma2_rn(s.nA[p], m, __fmul2_rn(dd, la));  // lam beta
        du2 = __ffma2_rn(lb, Bp[p], du2);
        const float2 dBv = __fmul2_rn(lb, xx);
        const float2 dCv = __fmul2_rn(dyy, hcv[p]);
        vbc[2 * p] = dBv.x;
        vbc[2 * p + 1] = dBv.y;
        vbc[4 + 2 * p] = dCv.x;
        vbc[4 + 2 * p + 1] = dCv.y;
        const float2 lah = __fmul2_rn(la, hpv[p]);
        S1 = __ffma2_rn(s.A2[p], lah, S1);
        S2 = __ffma2_rn(la, Bp[p], S2);
        s.P1[p] = __ffma2_rn(dd, lah, s.P1[p]);
        s.P2[p] = __ffma2_rn(m, __fmul2_rn(Bp[p], xx), s.P2[p]);
        y2 = __ffma2_rn(Cp[p], hcv[p], y2);
        s.lam[p] = la;
    }
    pdu = du2.x + du2.y;
    pdd = fmaf(kLn2, S1.x + S1.y, dx.z * (S2.x + S2.y));
    py = y2.x + y2.y;
}

// Sum 8 values over the 8 channel lanes (low lane bits) of each state group of a warp
// through a padded shared-memory transpose: lane (g, c) leaves with value c of its
// group summed over the group's lanes.  tr is the warp's scratch of TR_WARP floats.
template <int CW>
__device__ __forceinline__ float tr_reduce8(const float (&v)[8], float* tr, int g, int c) {
    constexpr int ROW = 8 * (CW + 1);
    float* mine = tr + g * ROW + c * 8;
    reinterpret_cast<float4*>(mine)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(mine)[1] = make_float4(v[4], v[5], v[6], v[7]);
    __syncwarp();
    const float* col = tr + g * ROW + c;
    float r = col[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) r += col[8 * k];
    __syncwarp();
    return r;
}

template <typename T, int NG, int MODE>
__global__ void __launch_bounds__(kThreadsB, 5)
    bwd_tiled_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_dr,
                     const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_g,
                     const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                     const __grid_constant__ CUtensorMap tm_du, const __grid_constant__ CUtensorMap tm_ddr,
                     const __grid_constant__ CUtensorMap tm_dz, BwdTiledArgs a) {
    using C = BCfg<T, NG>;
    using P2 = typename BPair<T>::type;
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t ncb = (a.D + C::DC - 1) / C::DC;
    const int cb = (int)(blockIdx.x % ncb);
    // segment of the sequence (the summary pass skips segment 0, whose summary no
    // segment needs)
    const int64_t nsl = MODE == kBwdSummary ? a.nseg - 1 : a.nseg;
    const int64_t rest = blockIdx.x / ncb;
    const int seg = (int)(rest % nsl) + (MODE == kBwdSummary ? 1 : 0);
    const int b = (int)(rest / nsl);
    const int N = a.N;
    const int d0 = cb * C::DC;
    // extents of the arrays indexed below (checked in the debug build only)
    const int64_t ext_seg = a.batch * a.nseg * a.D * N, ext_ckpt = a.batch * a.nck * a.D * N;
    const int64_t ext_bln = a.batch * a.L * N;
    const int tiles_all = (int)((a.L + kTB - 1) / kTB);
    const int tile_lo = seg * (int)(a.seg_len / kTB);
    const int tile_hi = min(tiles_all, tile_lo + (int)((a.seg_len + kTB - 1) / kTB));
    const int ntb = tile_hi - tile_lo;  // tiles of this segment
    const bool has_z = a.has_z != 0;
    constexpr bool kSum = MODE == kBwdSummary;  // the summary pass reads neither u nor B
    const uint32_t bar0 = smem_u32(smem + (kSum ? C::OFF_BAR_SUM : C::OFF_BAR));
    const uint32_t stage_bytes = ((has_z ? 4u : 3u) - (kSum ? 1u : 0u)) * C::RAW +
                                 (kSum ? 1u : 2u) * (uint32_t)(kTB * N * (int)sizeof(T));

    // tiles are taken in reverse: processing index k covers tile tile_hi - 1 - k
    auto issue = [&](int k) {
        const int st = k % C::STAGES;
        const uint32_t bar = bar0 + 8 * st;
        const uint32_t base = smem_u32(smem + C::OFF_RAW + st * C::STAGE);
        const int t0 = (tile_hi - 1 - k) * kTB;
        mbar_expect_tx(bar, stage_bytes);
        if (!kSum) tma_load_3d(base, &tm_u, d0, t0, b, bar);
        tma_load_3d(base + C::RAW, &tm_dr, d0, t0, b, bar);
        if (has_z) tma_load_3d(base + 2 * C::RAW, &tm_z, d0, t0, b, bar);
        tma_load_3d(base + 3 * C::RAW, &tm_g, d0, t0, b, bar);
        if (!kSum) tma_load_3d(base + 4 * C::RAW, &tm_B, 0, t0, b, bar);
        tma_load_3d(base + 4 * C::RAW + C::RAWBC, &tm_C, 0, t0, b, bar);
    };

    int bad = 0;
    if (tid == 0) {
        for (int st = 0; st < C::STAGES; ++st) mbar_init(bar0 + 8 * st, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int k = 0; k < C::STAGES && k < ntb; ++k) issue(k);
    }
    // the tile's dB, dC summed over the CTA's channels: zero here, and zeroed again by
    // the thread that drains each entry into global memory
    float* sacc = reinterpret_cast<float*>(smem + C::OFF_ACC);
    if (!kSum)
        for (int e = tid; e < kTB * C::NS * 2; e += kThreadsB) sacc[e] = 0.f;

    // lane state: channel cw, states g*4 .. g*4+3
    const int g = lane / C::CW, c = lane % C::CW, cw = warp * C::CW + c;
    const int64_t d = d0 + cw;
    const bool cvalid = d < a.D;
    RevLane s;
    bool small_a = false;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        float av[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int n = g * 4 + 2 * k + j;
            const bool ok = cvalid && n < N;
            av[j] = ok && in_range(d * N + n, a.D * N) ? __ldg(a.A + d * N + n) : 0.f;
            small_a |= ok && fabsf(av[j]) < kSmallAB;
        }
        s.A2[k] = g2(av[0] * kLog2e, av[1] * kLog2e);
        s.niA[k] = g2(av[0] != 0.f ? -1.f / av[0] : 0.f, av[1] != 0.f ? -1.f / av[1] : 0.f);
        s.nA[k] = g2(-av[0], -av[1]);
        s.iA2[k] = g2(av[0] != 0.f ? 1.f / (av[0] * av[0]) : 0.f, av[1] != 0.f ? 1.f / (av[1] * av[1]) : 0.f);
        s.lam[k] = s.P1[k] = s.P2[k] = g2(0.f, 0.f);
    }
    if (MODE == kBwdFull && a.nseg > 1) {
        // the adjoint state the segments to the right pass in
        float lv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = g * 4 + j;
            const int64_t il = (((int64_t)b * a.nseg + seg) * a.D + d) * N + n;
            lv[j] = cvalid && n < N && in_range(il, ext_seg) ? a.ws_lam[il] : 0.f;
        }
        s.lam[0] = g2(lv[0], lv[1]);
        s.lam[1] = g2(lv[2], lv[3]);
    }
    float dsum = 0.f;
    const int nvalid = cvalid ? min(4, N - g * 4) : 0;
    float dbias_acc = 0.f;
    // phase-P channel pair of this thread (fixed: PAIRS is a multiple of the thread count)
    const int pc = 2 * (tid % (C::DC / 2));
    const int64_t pd = d0 + pc;
    const float2 pbias = g2((a.bias && pd < a.D) ? __ldg(a.bias + pd) : 0.f,
                            (a.bias && pd + 1 < a.D) ? __ldg(a.bias + pd + 1) : 0.f);
    const float2 pdsk = g2((a.Dskip && pd < a.D) ? __ldg(a.Dskip + pd) : 0.f,
                           (a.Dskip && pd + 1 < a.D) ? __ldg(a.Dskip + pd + 1) : 0.f);
    float2 dD_acc = g2(0.f, 0.f);
    float* tr = reinterpret_cast<float*>(smem + C::OFF_TR) + warp * C::TR_WARP;

    if (tid == 0 && ntb > 0) bad = !mbar_wait(bar0, 0);
    // one CTA-wide choice of the recomputation's Bbar form (block-uniform branch)
    const int flags = __syncthreads_or((small_a ? 1 : 0) | (bad ? 2 : 0));
    const bool acc = (flags & 1) != 0;
    bool failed = (flags & 2) != 0;

    for (int k = 0; k < ntb && !failed; ++k) {
        const int it = tile_hi - 1 - k;
        const int st = k % C::STAGES;
        const int t0 = it * kTB;
        const int tile_len = (int)(a.L - t0 < kTB ? a.L - t0 : kTB);
        const unsigned char* raw = smem + C::OFF_RAW + st * C::STAGE;
        // ---- phase P: operand pairs of every (step, channel) of the tile
        {
            const P2* ru = reinterpret_cast<const P2*>(raw);
            const P2* rd = reinterpret_cast<const P2*>(raw + C::RAW);
            const P2* rz = reinterpret_cast<const P2*>(raw + 2 * C::RAW);
            const P2* rg = reinterpret_cast<const P2*>(raw + 3 * C::RAW);
            float4* sdx = reinterpret_cast<float4*>(smem + C::OFF_DX);
            float2* sdy = reinterpret_cast<float2*>(smem + C::OFF_DY);
            float4* sep = reinterpret_cast<float4*>(smem + C::OFF_EP);
            float2* ssu = reinterpret_cast<float2*>(smem + C::OFF_SU);
#pragma unroll
            for (int qi = 0; qi < C::PAIRS / kThreadsB; ++qi) {
                const int q = tid + qi * kThreadsB;
                const int t = q / (C::DC / 2);
                const bool tv = t < tile_len;
                if constexpr (kSum) {
                    // the summary pass needs delta and dy only
                    const float2 r = __fadd2_rn(BPair<T>::f(rd[q]), pbias);
                    float2 dl = r, sr;
                    if (a.softplus) softplus_sig_x2(r, dl, sr);
                    float2 dy = BPair<T>::f(rg[q]);
                    if (has_z) {
                        const float2 zz = BPair<T>::f(rz[q]);
                        dy = __fmul2_rn(__fmul2_rn(dy, sigmoid_x2(zz)), zz);
                    }
                    if (!tv) dy = g2(0.f, 0.f);
                    const int e = t * C::DC + pc;
                    sdx[e] = make_float4(dl.x, dl.x, 0.f, 0.f);
                    sdx[e + 1] = make_float4(dl.y, dl.y, 0.f, 0.f);
                    reinterpret_cast<float4*>(sdy)[e / 2] = make_float4(dy.x, dy.x, dy.y, dy.y);
                    continue;
                }
                const float2 uv = BPair<T>::f(ru[q]);
                float2 x = uv;
                if (a.input_silu) {
                    const float2 su = sigmoid_x2(uv);
                    x = __fmul2_rn(uv, su);
                    // SiLU'(u) = s (1 + u (1 - s))
                    const float2 om = __ffma2_rn(su, g2(-1.f, -1.f), g2(1.f, 1.f));
                    ssu[(t * C::DC + pc) / 2] = __fmul2_rn(su, __ffma2_rn(uv, om, g2(1.f, 1.f)));
                }
                const float2 r = __fadd2_rn(BPair<T>::f(rd[q]), pbias);
                float2 dl = r, sr = g2(1.f, 1.f);
                if (a.softplus) softplus_sig_x2(r, dl, sr);
                const float2 go = BPair<T>::f(rg[q]);
                float2 dy = go, dzf = g2(0.f, 0.f);
                if (has_z) {
                    const float2 zz = BPair<T>::f(rz[q]);
                    const float2 sz = sigmoid_x2(zz);
                    const float2 gs = __fmul2_rn(go, sz);
                    dy = __fmul2_rn(gs, zz);
                    // dz factor: dout s (1 + z (1 - s))
                    dzf = __fmul2_rn(gs, __ffma2_rn(zz, __ffma2_rn(sz, g2(-1.f, -1.f), g2(1.f, 1.f)), g2(1.f, 1.f)));
                }
                if (!tv) dy = dzf = g2(0.f, 0.f);
                const int e = t * C::DC + pc;
                sdx[e] = make_float4(dl.x, dl.x, x.x, x.x);
                sdx[e + 1] = make_float4(dl.y, dl.y, x.y, x.y);
                reinterpret_cast<float4*>(sdy)[e / 2] = make_float4(dy.x, dy.x, dy.y, dy.y);
                const float2 kdy = __fmul2_rn(pdsk, dy), kx = __fmul2_rn(pdsk, x);
                sep[e] = make_float4(kdy.x, dzf.x, sr.x, kx.x);
                sep[e + 1] = make_float4(kdy.y, dzf.y, sr.y, kx.y);
                dD_acc = __ffma2_rn(dy, x, dD_acc);
            }
            const T* rB = reinterpret_cast<const T*>(raw + 4 * C::RAW);
            const T* rC = reinterpret_cast<const T*>(raw + 4 * C::RAW + C::RAWBC);
            float* sBf = reinterpret_cast<float*>(smem + C::OFF_B);
            float* sCf = reinterpret_cast<float*>(smem + C::OFF_C);
            for (int e = tid; e < kTB * C::NS; e += kThreadsB) {
                const int t = e / C::NS, n = e % C::NS;
                if (!kSum) sBf[e] = n < N ? to_f32<T>(rB[t * N + n]) : 0.f;
                sCf[e] = n < N ? to_f32<T>(rC[t * N + n]) : 0.f;
            }
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0 && k + C::STAGES < ntb) issue(k + C::STAGES);

        const float4* sdx = reinterpret_cast<const float4*>(smem + C::OFF_DX) + cw;
        const float2* sdy = reinterpret_cast<const float2*>(smem + C::OFF_DY) + cw;
        const float4* sB = reinterpret_cast<const float4*>(smem + C::OFF_B) + g;
        const float4* sC = reinterpret_cast<const float4*>(smem + C::OFF_C) + g;
        if constexpr (MODE == kBwdSummary) {
            // adjoint only: lam <- Abar_t (C_t dy_t + lam), from the right end of the segment
            for (int t = tile_len - 1; t >= 0; --t) {
                const float4 dx = sdx[t * C::DC];
                const float dy = sdy[t * C::DC].x;
                const float4 Cv = sC[t * NG];
                const float2 dd = g2(dx.x, dx.y), dyy = g2(dy, dy);
                const float2 Cp[2] = {g2(Cv.x, Cv.y), g2(Cv.z, Cv.w)};
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    s.lam[p] = __fmul2_rn(__ffma2_rn(Cp[p], dyy, s.lam[p]), ex2p(__fmul2_rn(dd, s.A2[p])));
                dsum += dx.x;
            }
            if (tid == 0 && k + 1 < ntb)
                bad = !mbar_wait(bar0 + 8 * ((k + 1) % C::STAGES), ((k + 1) / C::STAGES) & 1);
            failed = __syncthreads_or(bad) != 0;
            continue;
        }

        // ---- recompute the tile's states from the checkpoint
        float4* shs = reinterpret_cast<float4*>(smem + C::OFF_HS) + tid;
        float4 hk;
        {
            const int64_t ic = (((int64_t)b * a.nck + it) * a.D + d) * N + g * 4;
            float hv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) hv[j] = j < nvalid && in_range(ic + j, ext_ckpt) ? a.ws_ckpt[ic + j] : 0.f;
            hk = make_float4(hv[0], hv[1], hv[2], hv[3]);
        }
        {
            float2 h0 = g2(hk.x, hk.y), h1 = g2(hk.z, hk.w);
            // the forward kernel's form: h' = Abar (h - v) + v with v = -B x / A; the
            // exponentials and v of step t + 1 are prepared before the update of step t
            auto prep = [&](int t, float2& a0, float2& a1, float2& v0, float2& v1) {
                const float4 dx = sdx[t * C::DC];
                const float4 Bv = sB[t * NG];
                const float2 dd = g2(dx.x, dx.y), xx = g2(dx.z, dx.w);
                a0 = ex2p(__fmul2_rn(dd, s.A2[0]));
                a1 = ex2p(__fmul2_rn(dd, s.A2[1]));
                v0 = __fmul2_rn(g2(Bv.x, Bv.y), __fmul2_rn(xx, s.niA[0]));
                v1 = __fmul2_rn(g2(Bv.z, Bv.w), __fmul2_rn(xx, s.niA[1]));
            };
            if (!acc && tile_len == kTB) {
                float2 a0, a1, v0, v1;
                prep(0, a0, a1, v0, v1);
#pragma unroll
                for (int t = 0; t < kTB; ++t) {
                    float2 b0 = a0, b1 = a1, w0 = v0, w1 = v1;
                    if (t + 1 < kTB) prep(t + 1, b0, b1, w0, w1);
                    h0 = __ffma2_rn(a0, __ffma2_rn(v0, g2(-1.f, -1.f), h0), v0);
                    h1 = __ffma2_rn(a1, __ffma2_rn(v1, g2(-1.f, -1.f), h1), v1);
                    shs[t * kThreadsB] = make_float4(h0.x, h0.y, h1.x, h1.y);
                    a0 = b0, a1 = b1, v0 = w0, v1 = w1;
                }
            } else if (!acc) {
                for (int t = 0; t < tile_len; ++t) {
                    float2 a0, a1, v0, v1;
                    prep(t, a0, a1, v0, v1);
                    h0 = __ffma2_rn(a0, __ffma2_rn(v0, g2(-1.f, -1.f), h0), v0);
                    h1 = __ffma2_rn(a1, __ffma2_rn(v1, g2(-1.f, -1.f), h1), v1);
                    shs[t * kThreadsB] = make_float4(h0.x, h0.y, h1.x, h1.y);
                }
            } else {
                // |A| < 2^-10 somewhere in the block: Bbar from phi1's series where delta A is small
                const float2 iA[2] = {g2(-s.niA[0].x, -s.niA[0].y), g2(-s.niA[1].x, -s.niA[1].y)};
                for (int t = 0; t < tile_len; ++t) {
                    const float4 dx = sdx[t * C::DC];
                    const float4 Bv = sB[t * NG];
                    const float2 dd = g2(dx.x, dx.y), xx = g2(dx.z, dx.w);
                    const float2 Bx0 = __fmul2_rn(g2(Bv.x, Bv.y), xx), Bx1 = __fmul2_rn(g2(Bv.z, Bv.w), xx);
                    h0 = __ffma2_rn(ex2p(__fmul2_rn(dd, s.A2[0])), h0, __fmul2_rn(bbar2(dd, s.A2[0], iA[0]), Bx0));
                    h1 = __ffma2_rn(ex2p(__fmul2_rn(dd, s.A2[1])), h1, __fmul2_rn(bbar2(dd, s.A2[1], iA[1]), Bx1));
                    shs[t * kThreadsB] = make_float4(h0.x, h0.y, h1.x, h1.y);
                }
            }
        }
        // ---- reverse sweep in blocks of NG steps (last block first); the state loaded as
        // h_{t-1} at step t is the h_t of step t-1, so it is carried in registers
        T* so = reinterpret_cast<T*>(smem + C::OFF_OUT + (k & 1) * 3 * C::RAW);
        const float4* sep = reinterpret_cast<const float4*>(smem + C::OFF_EP) + cw;
        const float* ssu = reinterpret_cast<const float*>(smem + C::OFF_SU) + cw;
        float4 hnext = tile_len > 0 ? shs[(tile_len - 1) * kThreadsB] : make_float4(0.f, 0.f, 0.f, 0.f);
        auto step = [&](int t, float& pdu, float& pdd, float& py) {
            float vbc[8];
            const float4 hc = hnext;
            hnext = t > 0 ? shs[(t - 1) * kThreadsB] : hk;
            rev_step(s, sdx[t * C::DC], sdy[t * C::DC], sB[t * NG], sC[t * NG], hc, hnext, pdu, pdd, py, vbc);
            // dB, dC of step t summed over this warp's channels, then over the CTA in smem
            float v;
            if constexpr (NG == 4) v = tr_reduce8<C::CW>(vbc, tr, g, c);
            else v = treduce_c8<C::CW>(vbc, c);
            if (c < 8) {
                const int which = c >> 2, j = c & 3;
                atomicAdd(&sacc[(t * C::NS + g * 4 + j) * 2 + which], v);
            }
        };
        auto finish = [&](int tb, float (&pdu)[NG], float (&pdd)[NG], float (&py)[NG]) {
            const float sdu = treduce_g<NG, C::CW>(pdu, g);
            const float sdd_ = treduce_g<NG, C::CW>(pdd, g);
            const float sy = treduce_g<NG, C::CW>(py, g);
            const int t = tb + g;
            if (t < tile_len && g < NG) {
                const float4 ep = sep[t * C::DC];  // (D dy, dz factor, softplus', D x)
                float du = sdu + ep.x;
                if (a.input_silu) du *= ssu[t * C::DC];
                const float ddr = sdd_ * ep.z;
                so[t * C::DC + cw] = from_f32<T>(du);
                so[C::RAW / (int)sizeof(T) + t * C::DC + cw] = from_f32<T>(ddr);
                so[2 * C::RAW / (int)sizeof(T) + t * C::DC + cw] = from_f32<T>(ep.y * (sy + ep.w));
                if (cvalid) dbias_acc += ddr;
            }
        };
        if (tile_len == kTB) {
#pragma unroll
            for (int tb = kTB - NG; tb >= 0; tb -= NG) {
                float pdu[NG], pdd[NG], py[NG];
#pragma unroll
                for (int kk = NG - 1; kk >= 0; --kk) step(tb + kk, pdu[kk], pdd[kk], py[kk]);
                finish(tb, pdu, pdd, py);
            }
        } else {
            // the sequence's last, partial tile
            for (int tb = ((tile_len - 1) / NG) * NG; tb >= 0; tb -= NG) {
                float pdu[NG], pdd[NG], py[NG];
#pragma unroll
                for (int kk = NG - 1; kk >= 0; --kk) {
                    pdu[kk] = pdd[kk] = py[kk] = 0.f;
                    if (tb + kk < tile_len) step(tb + kk, pdu[kk], pdd[kk], py[kk]);
                }
                finish(tb, pdu, pdd, py);
            }
        }
        fence_proxy_async();
        if (tid == 0 && k + 1 < ntb)
            bad = !mbar_wait(bar0 + 8 * ((k + 1) % C::STAGES), ((k + 1) / C::STAGES) & 1);
        failed = __syncthreads_or(bad) != 0;
        if (tid == 0) {
            const uint32_t o = smem_u32(so);
            tma_store_3d_nocommit(&tm_du, d0, t0, b, o);
            tma_store_3d_nocommit(&tm_ddr, d0, t0, b, o + C::RAW);
            if (has_z) tma_store_3d_nocommit(&tm_dz, d0, t0, b, o + 2 * C::RAW);
            tma_commit();
            tma_store_wait_read_1();
        }
        // the tile's dB, dC into the fp32 accumulators (the next tile adds into sacc only
        // after its phase-P barrier)
        for (int e = tid; e < tile_len * C::NS; e += kThreadsB) {
            const int t = e / C::NS, n = e % C::NS;
            float2* slot = reinterpret_cast<float2*>(sacc) + e;
            if (n < N) {
                const float2 v = *slot;
                const int64_t gi = ((int64_t)b * a.L + t0 + t) * N + n;
                if (in_range(gi, ext_bln)) {
                    atomicAdd(a.dB32 + gi, v.x);
                    atomicAdd(a.dC32 + gi, v.y);
                }
            }
            *slot = make_float2(0.f, 0.f);
        }
    }
    if (tid == 0) tma_store_wait_all();
    if (failed) {
        if (tid == 0) {
            atomicOr(&g_device_error_bwd, 2u);
            for (int st = 0; st < C::STAGES; ++st) (void)mbar_wait(bar0 + 8 * st, 0), (void)mbar_wait(bar0 + 8 * st, 1);
        }
        return;
    }
    const float lamv[4] = {s.lam[0].x, s.lam[0].y, s.lam[1].x, s.lam[1].y};
    if constexpr (MODE == kBwdSummary) {
        // the segment's summary: adjoint state passed on from zero, and its sum of delta
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t il = (((int64_t)b * a.nseg + seg) * a.D + d) * N + g * 4 + j;
            if (j < nvalid && in_range(il, ext_seg)) a.ws_lam[il] = lamv[j];
        }
        const int64_t idsum = ((int64_t)b * a.nseg + seg) * a.D + d;
        if (g == 0 && cvalid && in_range(idsum, a.batch * a.nseg * a.D)) a.ws_dsum[idsum] = dsum;
        return;
    }
    // per-channel sums
    const float dAv[4] = {s.P1[0].x + s.P2[0].x, s.P1[0].y + s.P2[0].y, s.P1[1].x + s.P2[1].x, s.P1[1].y + s.P2[1].y};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j >= nvalid) continue;
        const int n = g * 4 + j;
        const int64_t is = ((int64_t)b * a.D + d) * N + n;
        if (a.dh0 && seg == 0 && in_range(is, a.batch * a.D * N)) a.dh0[is] = lamv[j];
        // dA = sum_t [delta lam Abar h_{t-1} + lam B x delta^2 psi(delta A)]
        if (in_range(d * N + n, a.D * N)) atomicAdd(a.dA + d * N + n, dAv[j]);
    }
    if (a.dbias && cvalid && in_range(d, a.D)) atomicAdd(a.dbias + d, dbias_acc);
    if (a.dD && pd < a.D) {
        if (in_range(pd, a.D)) atomicAdd(a.dD + pd, dD_acc.x);
        if (pd + 1 < a.D && in_range(pd + 1, a.D)) atomicAdd(a.dD + pd + 1, dD_acc.y);
    }
}

// 3-D map over a (batch, L, W) tensor, box [1][kTB][box_w].
template <typename T>
bool make_map_b(CUtensorMap* m, const void* base, int64_t batch, int64_t L, int64_t W, int box_w) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)(W * sizeof(T)), (cuuint64_t)(L * W * sizeof(T))};
    const cuuint32_t box[3] = {(cuuint32_t)box_w, (cuuint32_t)kTB, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType ty =
        sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    return fn(m, ty, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int NG, int MODE>
cudaError_t launch_bwd_kernel(const CUtensorMap (&m)[9], const BwdTiledArgs& a, cudaStream_t st) {
    using C = BCfg<T, NG>;
    auto kern = bwd_tiled_kernel<T, NG, MODE>;
    // function attributes are per device: set them once on each device used
    static bool configured[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    constexpr int smem = MODE == kBwdSummary ? C::SMEM_SUM : C::SMEM;
    if (!configured[dev]) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        configured[dev] = true;
    }
    const int64_t segs = MODE == kBwdSummary ? a.nseg - 1 : a.nseg;
    const int64_t blocks = a.batch * segs * ((a.D + C::DC - 1) / C::DC);
    if (blocks > 0)
        kern<<<(unsigned)blocks, kThreadsB, smem, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], m[8], a);
    return cudaGetLastError();
}

template <typename T, int NG>
cudaError_t launch_bwd_t(const BwdTiledArgs& a, const BwdTiledPtrs& p, int mode, cudaStream_t st) {
    using C = BCfg<T, NG>;
    CUtensorMap m[9];
    const void* zsrc = p.z ? p.z : p.u;
    void* dzdst = p.dz ? p.dz : p.du;
    if (!make_map_b<T>(&m[0], p.u, a.batch, a.L, a.D, C::DC) || !make_map_b<T>(&m[1], p.delta_raw, a.batch, a.L, a.D, C::DC) ||
        !make_map_b<T>(&m[2], zsrc, a.batch, a.L, a.D, C::DC) || !make_map_b<T>(&m[3], p.dout, a.batch, a.L, a.D, C::DC) ||
        !make_map_b<T>(&m[4], p.B, a.batch, a.L, a.N, a.N) || !make_map_b<T>(&m[5], p.C, a.batch, a.L, a.N, a.N) ||
        !make_map_b<T>(&m[6], p.du, a.batch, a.L, a.D, C::DC) || !make_map_b<T>(&m[7], p.ddelta_raw, a.batch, a.L, a.D, C::DC) ||
        !make_map_b<T>(&m[8], dzdst, a.batch, a.L, a.D, C::DC))
        return cudaErrorInvalidValue;
    return mode == kBwdSummary ? launch_bwd_kernel<T, NG, kBwdSummary>(m, a, st)
                               : launch_bwd_kernel<T, NG, kBwdFull>(m, a, st);
}

// W lanes per (batch, channel, state): compose the segments right to left with
// the warp-shuffle affine-pair scan, leaving in ws_lam the adjoint state that enters each
// segment from its right.  A segment maps an entering adjoint state lam to
// P lam + H, with P = exp(A * its sum of delta) (the product of its Abar) and H its
// summary; segment nseg-1 is entered with zero, and segment 0's own map is never
// needed.
__global__ void __launch_bounds__(128) bwd_carry_kernel(BwdTiledArgs a, int W) {
    const int64_t total = a.batch * a.D * a.N;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / W;
    const bool valid = r < total;
    const int64_t w = valid ? r : total - 1;
    const int64_t n = w % a.N, bd = w / a.N;
    const int64_t d = bd % a.D, b = bd / a.D;
    const float A2 = __ldg(a.A + d * a.N + n) * kLog2e;
    // map j (j = 0 .. nseg-2) is segment s = nseg-1-j
    const float lam0 = affine_carry_warp(
        a.nseg - 1, 0.f, W, valid,
        [&](int64_t j, float& p, float& q) {
            const int64_t s = a.nseg - 1 - j;
            const int64_t id = (b * a.nseg + s) * a.D + d, il = id * a.N + n;
            p = in_range(id, a.batch * a.nseg * a.D) ? ex2(A2 * a.ws_dsum[id]) : 0.f;
            q = in_range(il, a.batch * a.nseg * a.D * a.N) ? a.ws_lam[il] : 0.f;
        },
        [&](int64_t j, float v) {
            const int64_t il = ((b * a.nseg + (a.nseg - 1 - j)) * a.D + d) * a.N + n;
            if (in_range(il, a.batch * a.nseg * a.D * a.N)) a.ws_lam[il] = v;
        });
    const int64_t i0 = ((b * a.nseg) * a.D + d) * a.N + n;
    if (valid && (threadIdx.x & (W - 1)) == 0 && in_range(i0, a.batch * a.nseg * a.D * a.N)) a.ws_lam[i0] = lam0;
}

}  // namespace

cudaError_t read_device_error_bwd(unsigned int* value, int clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error_bwd, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error_bwd, &zero, sizeof(unsigned int));
    }
    return e;
}

cudaError_t launch_bwd_tiled(const BwdTiledArgs& a, const BwdTiledPtrs& p, int io_bf16, int mode, cudaStream_t st) {
    if (io_bf16) {
        if (a.N <= 4) return launch_bwd_t<__nv_bfloat16, 1>(a, p, mode, st);
        if (a.N <= 8) return launch_bwd_t<__nv_bfloat16, 2>(a, p, mode, st);
        return launch_bwd_t<__nv_bfloat16, 4>(a, p, mode, st);
    }
    if (a.N <= 4) return launch_bwd_t<float, 1>(a, p, mode, st);
    if (a.N <= 8) return launch_bwd_t<float, 2>(a, p, mode, st);
    return launch_bwd_t<float, 4>(a, p, mode, st);
}

cudaError_t launch_bwd_carry(const BwdTiledArgs& a, cudaStream_t st) {
    const int W = affine_lanes(a.nseg - 1);
    const int64_t n = a.batch * a.D * a.N * W;  // W lanes per (batch, channel, state)
    if (n > 0) bwd_carry_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(a, W);
    return cudaGetLastError();
}

}  // namespace sscan
