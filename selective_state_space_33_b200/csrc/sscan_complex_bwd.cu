// sscan_complex_bwd.cu -- backward of the complex-A selective scan (sscan_complex.cu),
// with the states recomputed on chip (Mamba technical summary page, sec. 4.1 item 3).
//
// The complex forward kernel, in checkpoint mode, stores the state before every 8th
// step.  This kernel walks each (batch, channel block) through the sequence in
// reverse, 8 steps (one tile) at a time: phase P stages (delta, x), (dy, the dz
// factor, softplus') and the tile's B and C rows in shared memory; each lane
// recomputes its 2 complex states through the tile from the checkpoint (kept in
// shared memory), then runs the adjoint recurrence backwards.  The adjoint of a
// complex state is dL/dRe h + i dL/dIm h; the product Abar h maps it by conj(Abar):
//   lam_t    = C_t dy_t + conj(Abar_{t+1}) lam_{t+1}
//   dx      += Re(conj(lam) beta) B,   dB += Re(conj(lam) beta) x,   dC += dy Re(h_t)
//   d delta += Re(conj(lam) Abar (a h_{t-1} + B x))
//   dA      += conj(conj(lam) (delta Abar h_{t-1} + delta^2 psi(delta a) B x))
// with beta = (Abar - 1)/a and psi(q) = (q e^q - (e^q - 1)) / q^2; for |delta a| < 1/2 the
// reverse step takes psi's series and beta = delta (Abar - delta a psi).  The
// recomputation follows the forward kernel's form h' = Abar (h - v) + v, v = -B x / a,
// or, in a block holding an |a| < 2^-10, phi1's series for |delta a| < 1/16.
// Per-element sums over a channel's lanes use transposed shuffle butterflies over
// blocks of steps; dB and dC (t, n) are summed over the
// warp's channels with shuffles, over the CTA's warps in shared memory, and added to
// fp32 accumulators in global memory.
#include <cuda_runtime.h>

#include <cstdint>

#include "sscan_complex_math.cuh"
#include "sscan_launch.h"
#include "sscan_math.cuh"

namespace sscan {
namespace {

constexpr int kXTB = 8;  // steps per tile (= the checkpoint spacing)
constexpr int kXWarps = 4;
constexpr int kXThreads = kXWarps * 32;
constexpr int kXCG = 2;  // complex states per lane
constexpr float kXSmallA = 9.765625e-4f;  // |a| below 2^-10: the block recomputes with phi1's series

template <int NG>
struct XCfg {
    static constexpr int CW = 32 / NG;
    static constexpr int DC = CW * kXWarps;
    static constexpr int NS = NG * kXCG;
};

__device__ __forceinline__ float2 cmul(float2 p, float2 q) {
    return make_float2(fmaf(p.x, q.x, -p.y * q.y), fmaf(p.x, q.y, p.y * q.x));
}

// Sum per-element values over a channel's NG lanes (lane bits at multiples of CW)
// for BLK consecutive steps: a transposed butterfly over the high BLK state-group
// bits (lane group ghi ends with step ghi of the block), then plain rounds over the
// remaining LO = NG / BLK groups.
template <int BLK, int LO, int CW>
__device__ __forceinline__ float xreduce(float (&p)[BLK], int ghi) {
#pragma unroll
    for (int m = BLK / 2; m >= 1; m /= 2) {
        const bool up = (ghi & m) != 0;
#pragma unroll
        for (int j = 0; j < m; ++j) {
            const float keep = up ? p[m + j] : p[j];
            const float send = up ? p[j] : p[m + j];
            p[j] = keep + __shfl_xor_sync(0xffffffffu, send, m * LO * CW);
        }
    }
    float v = p[0];
#pragma unroll
    for (int m = 1; m < LO; m <<= 1) v += __shfl_xor_sync(0xffffffffu, v, m * CW);
    return v;
}

template <typename T, int NG>
__global__ void __launch_bounds__(kXThreads, 6) bwd_complex_kernel(ComplexBwdArgs g) {
    const ComplexArgs& a = g.f;
    using C = XCfg<NG>;
    __shared__ float2 sdx[kXTB * C::DC];   // (delta, x)
    __shared__ float4 sq[kXTB * C::DC];    // (dy, dz factor, softplus', -)
    __shared__ float sB[kXTB * C::NS], sC[kXTB * C::NS];
    __shared__ float4 shs[kXTB * kXThreads];                 // recomputed h_t of each lane
    __shared__ float sacc[kXWarps][kXTB * C::NS][2];         // per-warp dB, dC of the tile
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t ncb = (a.D + C::DC - 1) / C::DC;
    const int64_t b = blockIdx.x / ncb;
    const int64_t d0 = (blockIdx.x % ncb) * C::DC;
    const int N = a.N;
    const T* u = static_cast<const T*>(a.u);
    const T* dr = static_cast<const T*>(a.delta_raw);
    const T* zz = static_cast<const T*>(a.z);
    const T* go = static_cast<const T*>(g.dout);
    const T* Bg = static_cast<const T*>(a.B);
    const T* Cg = static_cast<const T*>(a.C);

    const int gq = lane / C::CW, c = lane % C::CW, cw = warp * C::CW + c;
    const int64_t d = d0 + cw;
    const bool cvalid = d < a.D;
    const int nvalid = cvalid ? (N - gq * kXCG < kXCG ? N - gq * kXCG : kXCG) : 0;
    float2 av[kXCG], aq[kXCG], ia[kXCG], lam[kXCG], gA[kXCG];
    bool small_a = false;
#pragma unroll
    for (int j = 0; j < kXCG; ++j) {
        const int n = gq * kXCG + j;
        const bool ok = j < nvalid;
        const float ar = ok ? __ldg(a.A + (d * N + n) * 2) : -1.f;
        const float ai = ok ? __ldg(a.A + (d * N + n) * 2 + 1) : 0.f;
        const float m2 = ar * ar + ai * ai;
        small_a |= ok && m2 < kXSmallA * kXSmallA;
        av[j] = make_float2(ar, ai);
        aq[j] = make_float2(ar * kLog2e, ai);
        const float inv = m2 > 0.f ? 1.f / m2 : 0.f;
        ia[j] = make_float2(ar * inv, -ai * inv);
        lam[j] = gA[j] = make_float2(0.f, 0.f);
    }
    // one CTA-wide choice of the recomputation's form (block-uniform branch)
    const bool acc = __syncthreads_or(small_a ? 1 : 0) != 0;
    const float dsk = (cvalid && a.Dskip) ? __ldg(a.Dskip + d) : 0.f;
    float dD_acc = 0.f, db_acc = 0.f;
    const int ntile = (int)((a.L + kXTB - 1) / kXTB);

    for (int k = 0; k < ntile; ++k) {
        const int it = ntile - 1 - k;
        const int64_t t0 = (int64_t)it * kXTB;
        const int tl = (int)(a.L - t0 < kXTB ? a.L - t0 : kXTB);
        __syncthreads();  // the previous tile is done with shared memory
        // ---- phase P
        for (int e = tid; e < kXTB * C::DC; e += kXThreads) {
            const int t = e / C::DC;
            const int64_t dd = d0 + e % C::DC;
            float2 dx = make_float2(0.f, 0.f);
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < tl && dd < a.D) {
                const int64_t gi = (b * a.L + t0 + t) * a.D + dd;
                const float uv = IO<T>::load(u, gi);
                const float x = a.input_silu ? silu(uv) : uv;
                const float r = IO<T>::load(dr, gi) + (a.bias ? __ldg(a.bias + dd) : 0.f);
                const float o = IO<T>::load(go, gi);
                float dy = o, dzf = 0.f;
                if (zz) {
                    const float zv = IO<T>::load(zz, gi), s = sigmoid(zv);
                    dy = o * zv * s;
                    dzf = o * s * fmaf(zv, 1.f - s, 1.f);
                }
                dx = make_float2(a.softplus ? softplus(r) : r, x);
                q = make_float4(dy, dzf, a.softplus ? sigmoid(r) : 1.f, a.input_silu ? dsilu(uv) : 1.f);
            }
            sdx[e] = dx;
            sq[e] = q;
        }
        for (int e = tid; e < kXTB * C::NS; e += kXThreads) {
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

        // ---- recompute the tile's states from its checkpoint
        float2 hk[kXCG];
#pragma unroll
        for (int j = 0; j < kXCG; ++j) {
            const int n = gq * kXCG + j;
            hk[j] = j < nvalid ? make_float2(g.ckpt[(((b * g.nck + it) * a.D + d) * N + n) * 2],
                                             g.ckpt[(((b * g.nck + it) * a.D + d) * N + n) * 2 + 1])
                               : make_float2(0.f, 0.f);
        }
        if (!acc) {
            // the forward kernel's form: h' = Abar (h - v) + v with v = -B x / a
            float2 h[kXCG] = {hk[0], hk[1]};
            for (int t = 0; t < tl; ++t) {
                const float2 dx = sdx[t * C::DC + cw];
#pragma unroll
                for (int j = 0; j < kXCG; ++j) {
                    const float2 cs = cplx::cis(dx.x * aq[j].y);
                    const float e = ex2(dx.x * aq[j].x);
                    const float2 ab = make_float2(e * cs.x, e * cs.y);
                    const float bx = sB[t * C::NS + gq * kXCG + j] * dx.y;
                    const float2 nh = cmul(ab, make_float2(fmaf(bx, ia[j].x, h[j].x), fmaf(bx, ia[j].y, h[j].y)));
                    h[j] = make_float2(fmaf(-bx, ia[j].x, nh.x), fmaf(-bx, ia[j].y, nh.y));
                }
                shs[t * kXThreads + tid] = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            }
        } else {
            // |a| < 2^-10 somewhere in the block: Bbar from phi1's series where delta a is small
            float2 h[kXCG] = {hk[0], hk[1]};
            for (int t = 0; t < tl; ++t) {
                const float2 dx = sdx[t * C::DC + cw];
#pragma unroll
                for (int j = 0; j < kXCG; ++j) {
                    const float2 cs = cplx::cis(dx.x * aq[j].y);
                    const float e = ex2(dx.x * aq[j].x);
                    const float2 ab = make_float2(e * cs.x, e * cs.y);
                    const float2 q = make_float2(dx.x * av[j].x, dx.x * av[j].y);
                    float2 beta;
                    if (q.x * q.x + q.y * q.y < 0.00390625f) {
                        float2 p = make_float2(1.f / 120.f, 0.f);
                        const float cf[4] = {1.f / 24.f, 1.f / 6.f, 0.5f, 1.f};
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            p = cmul(p, q);
                            p.x += cf[m];
                        }
                        beta = make_float2(dx.x * p.x, dx.x * p.y);
                    } else {
                        beta = cmul(make_float2(ab.x - 1.f, ab.y), ia[j]);
                    }
                    const float bx = sB[t * C::NS + gq * kXCG + j] * dx.y;
                    const float2 nh = cmul(ab, h[j]);
                    h[j] = make_float2(fmaf(beta.x, bx, nh.x), fmaf(beta.y, bx, nh.y));
                }
                shs[t * kXThreads + tid] = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
            }
        }

        // ---- reverse sweep, in blocks of BLK steps whose per-element sums are reduced together
        constexpr int BLK = NG > 4 ? 4 : NG, LO = NG / BLK;
        const int ghi = gq / LO, glo = gq % LO;
        for (int tb = ((tl - 1) / BLK) * BLK; tb >= 0; tb -= BLK) {
          float p1[BLK], p2[BLK], p3[BLK];
#pragma unroll
          for (int kk = BLK - 1; kk >= 0; --kk) {
            const int t = tb + kk;
            p1[kk] = p2[kk] = p3[kk] = 0.f;
            if (t >= tl) continue;
            const float2 dx = sdx[t * C::DC + cw];
            const float4 q4 = sq[t * C::DC + cw];
            const float delta = dx.x, x = dx.y, dy = q4.x;
            const float4 hc4 = shs[t * kXThreads + tid];
            const float4 hp4 = t > 0 ? shs[(t - 1) * kXThreads + tid] : make_float4(hk[0].x, hk[0].y, hk[1].x, hk[1].y);
            const float2 hc[kXCG] = {make_float2(hc4.x, hc4.y), make_float2(hc4.z, hc4.w)};
            const float2 hp[kXCG] = {make_float2(hp4.x, hp4.y), make_float2(hp4.z, hp4.w)};
            float dxp = 0.f, ddp = 0.f, yp = 0.f, dbv[kXCG], dcv[kXCG];
#pragma unroll
            for (int j = 0; j < kXCG; ++j) {
                const float Bn = sB[t * C::NS + gq * kXCG + j], Cn = sC[t * C::NS + gq * kXCG + j];
                const float2 cs = cplx::cis(delta * aq[j].y);
                const float e = ex2(delta * aq[j].x);
                const float2 ab = make_float2(e * cs.x, e * cs.y);
                const float2 q = make_float2(delta * av[j].x, delta * av[j].y);
                const float qq = q.x * q.x + q.y * q.y;
                // beta = Bbar / B and the dA term delta^2 psi(q), psi(q) = (q e^q - (e^q - 1)) / q^2.
                // |q| < 1/2: psi by its series, beta = delta phi1(q) = delta (Abar - q psi) (no
                // cancellation); else beta = (Abar - 1) / a and delta^2 psi = (delta Abar - beta) / a,
                // whose cancellation costs at most a few 1e-6 relative there.  One branch per state.
                float2 beta, d2psi;
                if (qq < 0.25f) {
                    float2 p = make_float2(1.f / 840.f, 0.f);
                    const float cf[5] = {1.f / 144.f, 1.f / 30.f, 0.125f, 1.f / 3.f, 0.5f};
#pragma unroll
                    for (int m = 0; m < 5; ++m) {
                        p = cmul(p, q);
                        p.x += cf[m];
                    }
                    const float2 qp = cmul(q, p);
                    beta = make_float2(delta * (ab.x - qp.x), delta * (ab.y - qp.y));
                    const float dd2 = delta * delta;
                    d2psi = make_float2(dd2 * p.x, dd2 * p.y);
                } else {
                    beta = cmul(make_float2(ab.x - 1.f, ab.y), ia[j]);
                    d2psi = cmul(make_float2(fmaf(delta, ab.x, -beta.x), fmaf(delta, ab.y, -beta.y)), ia[j]);
                }
                const float2 l = make_float2(fmaf(Cn, dy, lam[j].x), lam[j].y);
                const float lb = fmaf(l.x, beta.x, l.y * beta.y);  // Re(conj(l) beta)
                const float bx = Bn * x;
                dxp = fmaf(lb, Bn, dxp);
                dbv[j] = lb * x;
                // dh/d delta = Abar (a h_{t-1} + B x)
                const float2 ah = cmul(av[j], hp[j]);
                const float2 dhd = cmul(ab, make_float2(ah.x + bx, ah.y));
                ddp = fmaf(l.x, dhd.x, fmaf(l.y, dhd.y, ddp));
                // dh/da = delta Abar h_{t-1} + delta^2 psi B x
                const float2 abh = cmul(ab, hp[j]);
                const float2 dha = make_float2(fmaf(delta, abh.x, bx * d2psi.x), fmaf(delta, abh.y, bx * d2psi.y));
                // conj(conj(l) dha): (Re, -Im) of conj(l) dha
                gA[j].x = fmaf(l.x, dha.x, fmaf(l.y, dha.y, gA[j].x));
                gA[j].y = fmaf(-l.x, dha.y, fmaf(l.y, dha.x, gA[j].y));
                dcv[j] = dy * hc[j].x;
                yp = fmaf(Cn, hc[j].x, yp);
                lam[j] = make_float2(fmaf(ab.x, l.x, ab.y * l.y), fmaf(ab.x, l.y, -ab.y * l.x));  // conj(ab) l
            }
            p1[kk] = dxp;
            p2[kk] = ddp;
            p3[kk] = yp;
            // dB, dC of step t summed over the warp's channels (the low lane bits)
#pragma unroll
            for (int j = 0; j < kXCG; ++j) {
#pragma unroll
                for (int m = 1; m < C::CW; m <<= 1) {
                    dbv[j] += __shfl_xor_sync(0xffffffffu, dbv[j], m);
                    dcv[j] += __shfl_xor_sync(0xffffffffu, dcv[j], m);
                }
                if (c == 0) {
                    sacc[warp][t * C::NS + gq * kXCG + j][0] = dbv[j];
                    sacc[warp][t * C::NS + gq * kXCG + j][1] = dcv[j];
                }
            }
          }
          // the block's per-element sums: lane group ghi finishes step tb + ghi
          const float sdu = xreduce<BLK, LO, C::CW>(p1, ghi);
          const float sdd = xreduce<BLK, LO, C::CW>(p2, ghi);
          const float syp = xreduce<BLK, LO, C::CW>(p3, ghi);
          const int t = tb + ghi;
          if (glo == 0 && t < tl && cvalid) {
              const float2 dx = sdx[t * C::DC + cw];
              const float4 q4 = sq[t * C::DC + cw];
              const int64_t gi = (b * a.L + t0 + t) * a.D + d;
              const float ddr = sdd * q4.z;
              IO<T>::store(static_cast<T*>(g.du), gi, fmaf(dsk, q4.x, sdu) * q4.w);
              IO<T>::store(static_cast<T*>(g.ddelta_raw), gi, ddr);
              if (g.dz) IO<T>::store(static_cast<T*>(g.dz), gi, q4.y * fmaf(dsk, dx.y, syp));
              dD_acc = fmaf(q4.x, dx.y, dD_acc);
              db_acc += ddr;
          }
        }
        __syncthreads();
        // the tile's dB, dC: the warps' sums into the fp32 accumulators
        for (int e = tid; e < tl * C::NS; e += kXThreads) {
            const int t = e / C::NS, n = e % C::NS;
            if (n < N) {
                float sb = 0.f, sc = 0.f;
#pragma unroll
                for (int w = 0; w < kXWarps; ++w) {
                    sb += sacc[w][e][0];
                    sc += sacc[w][e][1];
                }
                const int64_t gi = (b * a.L + t0 + t) * N + n;
                atomicAdd(g.dB32 + gi, sb);
                atomicAdd(g.dC32 + gi, sc);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kXCG; ++j) {
        if (j >= nvalid) continue;
        const int n = gq * kXCG + j;
        if (g.dh0) {
            g.dh0[((b * a.D + d) * N + n) * 2] = lam[j].x;
            g.dh0[((b * a.D + d) * N + n) * 2 + 1] = lam[j].y;
        }
        atomicAdd(g.dA + (d * N + n) * 2, gA[j].x);
        atomicAdd(g.dA + (d * N + n) * 2 + 1, gA[j].y);
    }
    // dD and the bias gradient: each lane group holds the steps it finished
#pragma unroll
    for (int m = 1; m < NG; m <<= 1) {
        dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m * C::CW);
        db_acc += __shfl_xor_sync(0xffffffffu, db_acc, m * C::CW);
    }
    if (gq == 0 && cvalid) {
        if (g.dD) atomicAdd(g.dD + d, dD_acc);
        if (g.dbias) atomicAdd(g.dbias + d, db_acc);
    }
}

template <typename T, int NG>
cudaError_t launch_xb(const ComplexBwdArgs& a, cudaStream_t st) {
    const int64_t blocks = a.f.batch * ((a.f.D + XCfg<NG>::DC - 1) / XCfg<NG>::DC);
    if (blocks > 0) bwd_complex_kernel<T, NG><<<(unsigned)blocks, kXThreads, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_xbt(const ComplexBwdArgs& a, cudaStream_t st) {
    if (a.f.N <= 2) return launch_xb<T, 1>(a, st);
    if (a.f.N <= 4) return launch_xb<T, 2>(a, st);
    if (a.f.N <= 8) return launch_xb<T, 4>(a, st);
    return launch_xb<T, 8>(a, st);
}

}  // namespace

cudaError_t launch_bwd_complex(const ComplexBwdArgs& a, int io_bf16, cudaStream_t st) {
    return io_bf16 ? launch_xbt<__nv_bfloat16>(a, st) : launch_xbt<float>(a, st);
}

}  // namespace sscan
