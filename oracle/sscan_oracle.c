/*
 * sscan_oracle.c -- plain, slow, fp64 CPU oracle for the selective state-space
 * scan (S6) of "Mamba: Linear-Time Sequence Modeling with Selective State
 * Spaces" (Gu & Dao).  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline leg call it to check the CUDA library; nothing
 * in the product path links, imports or executes this file.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * Source of every formula (technical summary page "Mamba 状态空间模型原理与
 * Transformer 对比", kb.agiseed.tech):
 *   sec. 2.1 eq. (1a)/(1b)  continuous SSM h' = A h + B x, y = C h
 *   sec. 2.1 eq. (2)        zero-order hold: Abar = exp(dA),
 *                           Bbar = (dA)^-1 (exp(dA) - I) dB
 *   sec. 2.1 eq. (3a)/(3b)  recurrence h_t = Abar h_{t-1} + Bbar x_t, y_t = C h_t
 *   sec. 3.2                delta, B, C are functions of the input; delta passes
 *                           through softplus
 *   Fig. 3 caption          the block's gate uses SiLU, and the block replaces
 *                           the first multiplicative gate with an activation
 *                           (SiLU) on the input branch ahead of the SSM
 *   sec. 4.1                the scan reads (delta, A, B, C) and writes only
 *                           (B, L, D) outputs
 * Readings where the pages are silent (all marked again at the use site):
 *   - A is diagonal and stored as a (D, N) matrix, so eq. (2) becomes, per state
 *     n, Abar = exp(d*A_n) and Bbar = expm1(d*A_n)/A_n * B_n; for A_n = 0 the
 *     limit Bbar = d*B_n is taken.
 *   - delta = softplus(delta_raw + bias_d) when the softplus flag is set, else
 *     delta = delta_raw + bias_d.
 *   - a skip term D_skip[d]*x_t is added to y_t, and the result is multiplied
 *     by SiLU(z_t) when a gate input z is given: out = (C.h + D x) * SiLU(z).
 *   - h_{-1} is zero unless an initial state h0 is given.
 *   - with the input-activation flag the scan's input is x_t = SiLU(u_t) (the
 *     activation of the Fig. 3 input branch; the pages give no convolution or
 *     projection around it, so none is applied), used both in Bbar x_t and in
 *     the skip term; otherwise x_t = u_t.
 *   - layouts are dense row-major: u, delta_raw, z, out: (batch, L, D);
 *     B, C: (batch, L, N) shared by all D channels; A: (D, N);
 *     h0 / h_last: (batch, D, N).
 *
 * Everything is computed in IEEE double with libm's exp/expm1/log1p; inputs in
 * float32 or bfloat16 are widened exactly.  No blocking, fusion or reordering:
 * each (batch, channel) row is a plain loop over t and n.
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

typedef struct {
    int64_t batch, seqlen, dim, dstate;
    int32_t io_dtype;       /* element type of u, delta_raw, z, B, C, dout */
    int32_t delta_softplus; /* nonzero: delta = softplus(delta_raw + bias) */
    int32_t input_silu;     /* nonzero: the scan's input is x = SiLU(u)          */
} orc_problem;

/* Widen one element of an input array to double (exact for all three types). */
static double ld(const void* p, int32_t dt, int64_t i)
{
    if (dt == ORC_F64) return ((const double*)p)[i];
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    {
        uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
}

/* softplus(r) = log(1 + e^r), written in the overflow-free form
 * max(r, 0) + log1p(e^{-|r|}); identical in exact arithmetic (sec. 3.2). */
static double softplus(double r) { return (r > 0.0 ? r : 0.0) + log1p(exp(-fabs(r))); }

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* SiLU(v) = v * sigmoid(v) (Fig. 3 caption: the gate activation). */
static double silu(double v) { return v * sigmoid(v); }

/* d SiLU / dv = sigmoid(v) (1 + v (1 - sigmoid(v))). */
static double dsilu(double v)
{
    const double s = sigmoid(v);
    return s * (1.0 + v * (1.0 - s));
}

/* The scan's input x_t for the stored u_t: SiLU(u_t) when the input-branch
 * activation of Fig. 3 is requested, else u_t itself. */
static double scan_input(const orc_problem* p, double uv) { return p->input_silu ? silu(uv) : uv; }

/* dx_t/du_t for scan_input. */
static double scan_input_grad(const orc_problem* p, double uv) { return p->input_silu ? dsilu(uv) : 1.0; }

/* Bbar / B for one state, from eq. (2) with diagonal A: expm1(d*a)/a,
 * and its limit d when a == 0. */
static double bbar_coef(double delta, double a)
{
    if (a == 0.0) return delta;
    return expm1(delta * a) / a;
}

/* psi(q) = (q e^q - expm1(q)) / q^2, so that d/dA [expm1(dA)/A] = d^2 psi(dA).
 * Near 0 the direct form cancels; the Taylor series sum_{m>=2} (m-1)/m! q^(m-2)
 * is used there instead. */
static double psi(double q)
{
    if (fabs(q) < 1e-3)
        return 0.5 + q * (1.0 / 3.0 + q * (1.0 / 8.0 + q * (1.0 / 30.0 + q * (1.0 / 144.0))));
    return (q * exp(q) - expm1(q)) / (q * q);
}

static int check(const orc_problem* p)
{
    if (!p) return 1;
    if (p->batch < 0 || p->seqlen < 0 || p->dim < 0 || p->dstate < 1) return 1;
    if (p->io_dtype < ORC_F32 || p->io_dtype > ORC_F64) return 1;
    return 0;
}

/*
 * Forward scan, eqs. (2)-(3), for all rows or for the listed rows.
 *   rows == NULL: out is (batch, L, D), h_last is (batch, D, N).
 *   rows != NULL: rows[i] = b*D + d; out is (nrows, L), h_last is (nrows, N).
 * out and h_last may each be NULL (h_last only = the "last state" operation).
 * delta_bias, D_skip, z and h0 may be NULL (zero bias, no skip, no gate,
 * zero initial state).  Returns 0, or 1 on a bad argument.
 */
int orc_fwd(const orc_problem* p, const void* u, const void* delta_raw,
            const double* delta_bias, const double* A, const void* B,
            const void* C, const double* D_skip, const void* z,
            const double* h0, const int64_t* rows, int64_t nrows,
            double* out, double* h_last)
{
    if (check(p) || !u || !delta_raw || !A || !B || (out && !C)) return 1;
    const int64_t Bt = p->batch, L = p->seqlen, D = p->dim, N = p->dstate;
    const int32_t dt = p->io_dtype;
    const int64_t total = rows ? nrows : Bt * D;
    if (rows)
        for (int64_t i = 0; i < nrows; ++i)
            if (rows[i] < 0 || rows[i] >= Bt * D) return 1;

    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < total; ++i) {
        const int64_t row = rows ? rows[i] : i;
        const int64_t b = row / D, d = row % D;
        double* h = (double*)malloc((size_t)N * sizeof(double));
        if (!h) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[row * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const int64_t e = (b * L + t) * D + d; /* (batch, L, D) element */
            const int64_t s = (b * L + t) * N;     /* (batch, L, N) row     */
            const double x = scan_input(p, ld(u, dt, e));
            const double r = ld(delta_raw, dt, e) + (delta_bias ? delta_bias[d] : 0.0);
            const double delta = p->delta_softplus ? softplus(r) : r;
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double a = A[d * N + n];
                const double abar = exp(delta * a);                    /* eq. (2) */
                const double bbar = bbar_coef(delta, a) * ld(B, dt, s + n);
                h[n] = abar * h[n] + bbar * x;                         /* eq. (3a) */
                if (out) y += ld(C, dt, s + n) * h[n];                 /* eq. (3b) */
            }
            if (out) {
                if (D_skip) y += D_skip[d] * x;
                if (z) y *= silu(ld(z, dt, e));
                if (rows) out[i * L + t] = y;
                else out[e] = y;
            }
        }
        if (h_last)
            for (int64_t n = 0; n < N; ++n) h_last[(rows ? i : row) * N + n] = h[n];
        free(h);
    }
    return bad;
}

/*
 * Reverse-mode gradient of orc_fwd's `out` (all rows), by hand:
 *   out_t = y_t * SiLU(z_t),  y_t = sum_n C_tn h_tn + Dskip x_t,
 *   h_tn  = Abar_tn h_{t-1,n} + beta_tn B_tn x_t,  beta = expm1(dA)/A,
 *   Abar = exp(delta A),  delta = softplus(delta_raw + bias).
 * The adjoint lam_t = dL/dh_t obeys lam_t = C_t dy_t + Abar_{t+1} lam_{t+1}.
 * With dAbar = lam h_{t-1} and dbeta = lam B x:
 *   d delta += dAbar * A * Abar + dbeta * Abar          (d beta/d delta = Abar)
 *   dA      += dAbar * delta * Abar + dbeta * delta^2 psi(delta A)
 *   dx      += lam * beta * B,   dB += lam * beta * x,   dC += dy * h_t
 * and d delta_raw = d delta * sigmoid(r) under softplus.  States are kept for
 * the whole row (this is a CPU check, memory is not the point).
 * Outputs are overwritten; dB, dC are (batch, L, N); dA (D, N); dD, dbias (D);
 * dh0 (batch, D, N).  ddelta_bias, dD, dz, dh0 may be NULL.
 */
int orc_bwd(const orc_problem* p, const void* u, const void* delta_raw,
            const double* delta_bias, const double* A, const void* B,
            const void* C, const double* D_skip, const void* z,
            const double* h0, const void* dout, double* du,
            double* ddelta_raw, double* ddelta_bias, double* dA, double* dB,
            double* dC, double* dD, double* dz, double* dh0)
{
    if (check(p) || !u || !delta_raw || !A || !B || !C || !dout || !du ||
        !ddelta_raw || !dA || !dB || !dC)
        return 1;
    const int64_t Bt = p->batch, L = p->seqlen, D = p->dim, N = p->dstate;
    const int32_t dt = p->io_dtype;

    /* per-batch partial sums of the parameter gradients, added in fixed order */
    double* pA = (double*)calloc((size_t)(Bt * D * N + 1), sizeof(double));
    double* pD = (double*)calloc((size_t)(Bt * D + 1), sizeof(double));
    double* pbias = (double*)calloc((size_t)(Bt * D + 1), sizeof(double));
    if (!pA || !pD || !pbias) {
        free(pA); free(pD); free(pbias);
        return 1;
    }
    memset(dB, 0, (size_t)(Bt * L * N) * sizeof(double));
    memset(dC, 0, (size_t)(Bt * L * N) * sizeof(double));

    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < Bt; ++b) {
        double* hs = (double*)malloc((size_t)((L + 1) * N) * sizeof(double));
        double* ys = (double*)malloc((size_t)(L + 1) * sizeof(double));
        double* lam = (double*)malloc((size_t)N * sizeof(double));
        if (!hs || !ys || !lam) {
            free(hs); free(ys); free(lam);
#pragma omp atomic write
            bad = 1;
            continue;
        }
        for (int64_t d = 0; d < D; ++d) {
            const int64_t row = b * D + d;
            const double bias = delta_bias ? delta_bias[d] : 0.0;
            /* forward sweep, keeping h_t (hs[(t+1)*N + n]) and y_t */
            for (int64_t n = 0; n < N; ++n) hs[n] = h0 ? h0[row * N + n] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t e = (b * L + t) * D + d, s = (b * L + t) * N;
                const double x = scan_input(p, ld(u, dt, e));
                const double r = ld(delta_raw, dt, e) + bias;
                const double delta = p->delta_softplus ? softplus(r) : r;
                double y = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = A[d * N + n];
                    const double hn = exp(delta * a) * hs[t * N + n] +
                                      bbar_coef(delta, a) * ld(B, dt, s + n) * x;
                    hs[(t + 1) * N + n] = hn;
                    y += ld(C, dt, s + n) * hn;
                }
                ys[t] = y + (D_skip ? D_skip[d] * x : 0.0);
            }
            /* reverse sweep */
            for (int64_t n = 0; n < N; ++n) lam[n] = 0.0; /* Abar_{t+1} lam_{t+1} */
            for (int64_t t = L - 1; t >= 0; --t) {
                const int64_t e = (b * L + t) * D + d, s = (b * L + t) * N;
                const double x = scan_input(p, ld(u, dt, e));
                const double r = ld(delta_raw, dt, e) + bias;
                const double delta = p->delta_softplus ? softplus(r) : r;
                const double g = ld(dout, dt, e);
                double dy = g;
                if (z) {
                    const double zz = ld(z, dt, e), sg = sigmoid(zz);
                    dy = g * zz * sg;
                    if (dz) dz[e] = g * ys[t] * sg * (1.0 + zz * (1.0 - sg));
                }
                double dx = D_skip ? D_skip[d] * dy : 0.0;
                pD[row] += dy * x;
                double ddelta = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = A[d * N + n];
                    const double q = delta * a;
                    const double abar = exp(q);
                    const double beta = bbar_coef(delta, a);
                    const double Bn = ld(B, dt, s + n), Cn = ld(C, dt, s + n);
                    const double l = Cn * dy + lam[n];
                    const double dabar = l * hs[t * N + n];
                    const double dbeta = l * Bn * x;
                    dC[s + n] += dy * hs[(t + 1) * N + n];
                    dB[s + n] += l * beta * x;
                    dx += l * beta * Bn;
                    ddelta += dabar * a * abar + dbeta * abar;
                    pA[(b * D + d) * N + n] += dabar * delta * abar + dbeta * delta * delta * psi(q);
                    lam[n] = abar * l;
                }
                const double dr = p->delta_softplus ? ddelta * sigmoid(r) : ddelta;
                du[e] = dx * scan_input_grad(p, ld(u, dt, e));
                ddelta_raw[e] = dr;
                pbias[row] += dr;
            }
            if (dh0)
                for (int64_t n = 0; n < N; ++n) dh0[row * N + n] = lam[n];
        }
        free(hs); free(ys); free(lam);
    }
    for (int64_t d = 0; d < D; ++d) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t b = 0; b < Bt; ++b) acc += pA[(b * D + d) * N + n];
            dA[d * N + n] = acc;
        }
        double accD = 0.0, accb = 0.0;
        for (int64_t b = 0; b < Bt; ++b) {
            accD += pD[b * D + d];
            accb += pbias[b * D + d];
        }
        if (dD) dD[d] = accD;
        if (ddelta_bias) ddelta_bias[d] = accb;
    }
    free(pA); free(pD); free(pbias);
    return bad;
}

/* Thread control for the CPU-baseline timing (0 = leave OpenMP's default). */
/*
 * Forward scan with a complex diagonal A -- the complex initialisation
 * A_n = -1/2 + n i named in the sec. 6.5 A-init ablation table -- i.e. eqs. (2)
 * and (3) in complex arithmetic.  Readings where the pages are silent:
 *   - A is (D, N) complex, stored interleaved as (re, im) pairs: A[(d*N + n)*2 + k];
 *   - B and C stay the real (batch, L, N) input-dependent projections of sec. 3.2;
 *     the state is complex: h_t = Abar h_{t-1} + Bbar x_t with
 *     Abar = exp(delta a) and Bbar = (exp(delta a) - 1)/a * B (eq. 2; limit
 *     delta*B at a = 0);
 *   - the output is the real part of the readout eq. (3b):
 *     y_t = Re(sum_n C_tn h_tn) + D_skip x_t, then the SiLU gate;
 *   - h0 / h_last are (batch, D, N) complex, interleaved like A.
 * exp(q) - 1 for complex q = x + iy is formed as
 *   (expm1(x) cos y - 2 sin^2(y/2)) + i exp(x) sin y,
 * the same value without the cancellation of e^x cos y - 1 near q = 0.
 * Same argument conventions as orc_fwd (all rows; out, h_last may be NULL).
 */
int orc_fwd_complex(const orc_problem* p, const void* u, const void* delta_raw,
                    const double* delta_bias, const double* A, const void* B,
                    const void* C, const double* D_skip, const void* z,
                    const double* h0, double* out, double* h_last)
{
    if (check(p) || !u || !delta_raw || !A || !B || (out && !C)) return 1;
    const int64_t Bt = p->batch, L = p->seqlen, D = p->dim, N = p->dstate;
    const int32_t dt = p->io_dtype;

    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t row = 0; row < Bt * D; ++row) {
        const int64_t b = row / D, d = row % D;
        double* hr = (double*)malloc((size_t)N * 2 * sizeof(double));
        if (!hr) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        double* hi = hr + N;
        for (int64_t n = 0; n < N; ++n) {
            hr[n] = h0 ? h0[(row * N + n) * 2] : 0.0;
            hi[n] = h0 ? h0[(row * N + n) * 2 + 1] : 0.0;
        }
        for (int64_t t = 0; t < L; ++t) {
            const int64_t e = (b * L + t) * D + d;
            const int64_t s = (b * L + t) * N;
            const double x = scan_input(p, ld(u, dt, e));
            const double r = ld(delta_raw, dt, e) + (delta_bias ? delta_bias[d] : 0.0);
            const double delta = p->delta_softplus ? softplus(r) : r;
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double ar = A[(d * N + n) * 2], ai = A[(d * N + n) * 2 + 1];
                const double qr = delta * ar, qi = delta * ai;
                /* Abar = exp(q), eq. (2) */
                const double ex = exp(qr);
                const double abr = ex * cos(qi), abi = ex * sin(qi);
                /* Bbar / B = (exp(q) - 1) / a, or delta at a = 0 */
                double cr, ci;
                if (ar == 0.0 && ai == 0.0) {
                    cr = delta;
                    ci = 0.0;
                } else {
                    const double sh = sin(0.5 * qi);
                    const double em1r = expm1(qr) * cos(qi) - 2.0 * sh * sh, em1i = ex * sin(qi);
                    const double den = ar * ar + ai * ai;
                    cr = (em1r * ar + em1i * ai) / den;
                    ci = (em1i * ar - em1r * ai) / den;
                }
                const double bx = ld(B, dt, s + n) * x;
                /* eq. (3a) in complex arithmetic */
                const double nr = abr * hr[n] - abi * hi[n] + cr * bx;
                const double ni = abr * hi[n] + abi * hr[n] + ci * bx;
                hr[n] = nr;
                hi[n] = ni;
                if (out) y += ld(C, dt, s + n) * hr[n]; /* Re of eq. (3b) */
            }
            if (out) {
                if (D_skip) y += D_skip[d] * x;
                if (z) y *= silu(ld(z, dt, e));
                out[e] = y;
            }
        }
        if (h_last)
            for (int64_t n = 0; n < N; ++n) {
                h_last[(row * N + n) * 2] = hr[n];
                h_last[(row * N + n) * 2 + 1] = hi[n];
            }
        free(hr);
    }
    return bad;
}

/* exp(q) - 1 for complex q without the cancellation of e^x cos y - 1 near 0. */
static double complex cexpm1_(double complex q)
{
    const double x = creal(q), y = cimag(q), sh = sin(0.5 * y);
    return (expm1(x) * cos(y) - 2.0 * sh * sh) + I * (exp(x) * sin(y));
}

/* psi(q) = (q e^q - (e^q - 1)) / q^2 for complex q (the derivative of (e^q - 1)/q);
 * its Taylor series 1/2 + q/3 + q^2/8 + q^3/30 + q^4/144 near 0. */
static double complex cpsi(double complex q)
{
    if (cabs(q) < 1e-3)
        return 0.5 + q * (1.0 / 3.0 + q * (1.0 / 8.0 + q * (1.0 / 30.0 + q * (1.0 / 144.0))));
    return (q * cexp(q) - cexpm1_(q)) / (q * q);
}

/*
 * Reverse-mode gradient of orc_fwd_complex's `out` (all rows), by hand.  The
 * complex state is a pair of real variables, so the adjoint lam = dL/dRe h +
 * i dL/dIm h; multiplying h by Abar maps the adjoint by conj(Abar):
 *   lam_t = C_t dy_t + conj(Abar_{t+1}) lam_{t+1}        (C dy is real)
 * and for any real parameter p entering h_t through dh/dp, dL/dp += Re(conj(lam) dh/dp):
 *   dx    += Re(conj(lam) beta) B,   dB += Re(conj(lam) beta) x,   dC += dy Re(h_t)
 *   d delta += Re(conj(lam) (a Abar h_{t-1} + Abar B x))     (d beta/d delta = Abar)
 *   dA   : h is holomorphic in a, so with g = conj(lam) (delta Abar h_{t-1} + delta^2
 *          psi(delta a) B x):  dA_re += Re(g),  dA_im += -Im(g)
 *   dh0 = conj(Abar_0) lam_0.
 * A, dA, h0, dh0 are (re, im) interleaved like orc_fwd_complex; the other outputs
 * as orc_bwd (ddelta_bias, dD, dz, dh0 may be NULL).
 */
int orc_bwd_complex(const orc_problem* p, const void* u, const void* delta_raw,
                    const double* delta_bias, const double* A, const void* B,
                    const void* C, const double* D_skip, const void* z,
                    const double* h0, const void* dout, double* du,
                    double* ddelta_raw, double* ddelta_bias, double* dA, double* dB,
                    double* dC, double* dD, double* dz, double* dh0)
{
    if (check(p) || !u || !delta_raw || !A || !B || !C || !dout || !du || !ddelta_raw || !dA || !dB || !dC)
        return 1;
    const int64_t Bt = p->batch, L = p->seqlen, D = p->dim, N = p->dstate;
    const int32_t dt = p->io_dtype;
    memset(dA, 0, (size_t)(D * N * 2) * sizeof(double));
    memset(dB, 0, (size_t)(Bt * L * N) * sizeof(double));
    memset(dC, 0, (size_t)(Bt * L * N) * sizeof(double));
    if (ddelta_bias) memset(ddelta_bias, 0, (size_t)D * sizeof(double));
    if (dD) memset(dD, 0, (size_t)D * sizeof(double));
    int bad = 0;
    /* rows are independent except for the sums over (batch, channel) -- dA, dB, dC,
     * dbias, dD -- so rows run sequentially here (plain, not fast) */
    for (int64_t row = 0; row < Bt * D && !bad; ++row) {
        const int64_t b = row / D, d = row % D;
        double complex* h = (double complex*)malloc((size_t)((L + 1) * N) * sizeof(double complex));
        double complex* lam = (double complex*)malloc((size_t)N * sizeof(double complex));
        if (!h || !lam) {
            free(h);
            free(lam);
            bad = 1;
            break;
        }
        /* forward, keeping every state: h[(t+1)*N + n] = h_t, h[n] = h_{-1} = h0 */
        for (int64_t n = 0; n < N; ++n)
            h[n] = h0 ? h0[(row * N + n) * 2] + I * h0[(row * N + n) * 2 + 1] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const int64_t e = (b * L + t) * D + d, s = (b * L + t) * N;
            const double x = scan_input(p, ld(u, dt, e));
            const double r = ld(delta_raw, dt, e) + (delta_bias ? delta_bias[d] : 0.0);
            const double delta = p->delta_softplus ? softplus(r) : r;
            for (int64_t n = 0; n < N; ++n) {
                const double complex a = A[(d * N + n) * 2] + I * A[(d * N + n) * 2 + 1];
                const double complex abar = cexp(delta * a);
                const double complex beta = (a == 0.0) ? delta : cexpm1_(delta * a) / a;
                h[(t + 1) * N + n] = abar * h[t * N + n] + beta * ld(B, dt, s + n) * x;
            }
        }
        /* reverse */
        for (int64_t n = 0; n < N; ++n) lam[n] = 0.0;
        double dDacc = 0.0, dbacc = 0.0;
        for (int64_t t = L - 1; t >= 0; --t) {
            const int64_t e = (b * L + t) * D + d, s = (b * L + t) * N;
            const double x = scan_input(p, ld(u, dt, e));
            const double r = ld(delta_raw, dt, e) + (delta_bias ? delta_bias[d] : 0.0);
            const double delta = p->delta_softplus ? softplus(r) : r;
            const double go = ld(dout, dt, e);
            double dy = go;
            if (z) {
                double y = D_skip ? D_skip[d] * x : 0.0;
                for (int64_t n = 0; n < N; ++n) y += ld(C, dt, s + n) * creal(h[(t + 1) * N + n]);
                const double zz = ld(z, dt, e), sg = sigmoid(zz);
                dy = go * zz * sg;
                if (dz) dz[e] = go * y * sg * (1.0 + zz * (1.0 - sg));
            }
            double dx = D_skip ? D_skip[d] * dy : 0.0;
            dDacc += dy * x;
            double ddelta = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double complex a = A[(d * N + n) * 2] + I * A[(d * N + n) * 2 + 1];
                const double complex q = delta * a;
                const double complex abar = cexp(q);
                const double complex beta = (a == 0.0) ? delta : cexpm1_(q) / a;
                const double Bn = ld(B, dt, s + n), Cn = ld(C, dt, s + n);
                const double complex l = Cn * dy + lam[n];
                const double complex hp = h[t * N + n];
                dC[s + n] += dy * creal(h[(t + 1) * N + n]);
                const double lb = creal(conj(l) * beta);
                dB[s + n] += lb * x;
                dx += lb * Bn;
                ddelta += creal(conj(l) * (a * abar * hp + abar * Bn * x));
                const double complex g = conj(l) * (delta * abar * hp + delta * delta * cpsi(q) * Bn * x);
                dA[(d * N + n) * 2] += creal(g);
                dA[(d * N + n) * 2 + 1] -= cimag(g);
                lam[n] = conj(abar) * l;
            }
            const double drr = p->delta_softplus ? ddelta * sigmoid(r) : ddelta;
            du[e] = dx * scan_input_grad(p, ld(u, dt, e));
            ddelta_raw[e] = drr;
            dbacc += drr;
        }
        for (int64_t n = 0; n < N; ++n)
            if (dh0) {
                dh0[(row * N + n) * 2] = creal(lam[n]);
                dh0[(row * N + n) * 2 + 1] = cimag(lam[n]);
            }
        if (dD) dD[d] += dDacc;
        if (ddelta_bias) ddelta_bias[d] += dbacc;
        free(h);
        free(lam);
    }
    return bad;
}

int orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
