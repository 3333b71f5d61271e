/*
 * ssm_oracle.c -- fp64 CPU oracle for the selective-scan hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * path.  It is deliberately plain and slow: one (batch, channel) row at a time,
 * time as the outer loop, state index as the inner loop, every quantity in
 * double precision, libm's exp/expm1.
 *
 * What it computes follows the web page "Mamba SSM Nedir? Transformer
 * Alternatifi Rehberi (2026)" (yapayzekasozluk.tr):
 *   - section "State Space Model Temelleri": the continuous system
 *         h'(t) = A h(t) + B x(t),   y(t) = C h(t) + D x(t)
 *   - section "Ayrık Zamana Geçiş": zero-order-hold discretisation with step
 *     size Delta,
 *         Abar = exp(Delta A)
 *         Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B
 *     followed by the recurrence  h_t = Abar h_{t-1} + Bbar x_t,  y_t = C h_t
 *   - section "Mamba'nın Yeniliği: Selective SSM": B, C and Delta are produced
 *     per token (B_t, C_t, Delta_t); A stays a fixed parameter.
 *
 * Readings taken where the pages are silent or disagree, each with the
 * passage it rests on:
 *   - A is diagonal, one value per (channel, state): A[d][n] ("Ayrık Zamana
 *     Geçiş" writes exp(Delta A) and (Delta A)^-1 as matrix functions; with a
 *     diagonal A they act state by state).  The discretised quantities are
 *     then per state: Abar_n = exp(Delta A_n) and
 *     Bbar_n = (Delta A_n)^-1 (exp(Delta A_n) - 1) Delta B_n.
 *   - Delta is per (batch, token, channel); B_t and C_t are per (batch, token,
 *     state) and shared by every channel ("Mamba'nın Yeniliği: Selective SSM"
 *     lists B, C and Delta as the quantities computed from the input; A is
 *     not among them).
 *   - The discrete output keeps the D x_t skip term of the continuous form of
 *     "State Space Model Temelleri": y_t = C_t . h_t + D_d x_t, with h_t the
 *     state AFTER the update at t (the order in which "Ayrık Zamana Geçiş"
 *     writes the two equations).
 *   - The scan starts from h = 0 unless an initial state is given (no page
 *     states an initial state).
 *   - Delta A = 0 lies outside the stable domain A < 0 ("Sınırlılıklar ve
 *     Açık Sorular"); there the limit (e^z - 1)/z -> 1 is used, i.e.
 *     Bbar = Delta B.
 *
 * Layouts (row-major, last index fastest):
 *   u, delta, y   : [batch][len][channels]
 *   B, C          : [batch][len][nstate]
 *   A             : [channels][nstate]
 *   D             : [channels]                (may be NULL: no skip term)
 *   h0, h_final   : [batch][channels][nstate] (h0 may be NULL: zeros)
 */
#include <complex.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One zero-order-hold step for a single state of a diagonal system, exactly
 * as the "Ayrık Zamana Geçiş" section writes it, with z = Delta * A_n:
 *   Abar = exp(z)
 *   Bbar = z^-1 (exp(z) - 1) Delta B_n
 * exp(z) - 1 is evaluated with expm1 so that small z keeps full precision.   */
static void zoh_discretise(double delta, double a, double b, double *abar, double *bbar)
{
    double z = delta * a;
    *abar = exp(z);
    double phi = (z == 0.0) ? 1.0 : expm1(z) / z; /* (Delta A)^-1 (e^{Delta A} - 1) */
    *bbar = phi * delta * b;
}

/* The recurrence of one (batch, channel) row over `len` tokens.
 * h (length nstate) holds the running state in and out.  `stride` is the
 * distance between consecutive tokens in u/delta/y (the channel count).      */
static void scan_row(const double *u, const double *delta, const double *A_row,
                     const double *B, const double *C, double D_d, int has_D,
                     double *y, double *h, int64_t len, int64_t stride, int64_t nstate)
{
    for (int64_t t = 0; t < len; ++t) {
        double x = u[t * stride];
        double dt = delta[t * stride];
        const double *Bt = B + t * nstate;
        const double *Ct = C + t * nstate;
        double acc = 0.0;
        for (int64_t n = 0; n < nstate; ++n) {
            double abar, bbar;
            zoh_discretise(dt, A_row[n], Bt[n], &abar, &bbar);
            h[n] = abar * h[n] + bbar * x;    /* h_t = Abar h_{t-1} + Bbar x_t */
            acc += Ct[n] * h[n];              /* C_t . h_t                     */
        }
        if (has_D)
            acc += D_d * x;                   /* + D x_t                       */
        if (y)
            y[t * stride] = acc;
    }
}

/* Selective scan over whole sequences.  Returns 0 on success, -1 on a bad
 * argument.  nthreads <= 0 uses the OpenMP default.                          */
int oracle_scan(const double *u, const double *delta, const double *A,
                const double *B, const double *C, const double *D,
                const double *h0, double *y, double *h_final,
                int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                int nthreads)
{
    if (batch < 0 || len < 0 || channels < 0 || nstate <= 0)
        return -1;
    if ((len > 0 && (!u || !delta || !B || !C)) || !A)
        return -1;
    int64_t rows = batch * channels;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = 0;
#pragma omp parallel
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)nstate);
        if (!h) {
#pragma omp atomic write
            status = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            if (!h)
                continue;
            int64_t b = r / channels, d = r % channels;
            for (int64_t n = 0; n < nstate; ++n)
                h[n] = h0 ? h0[(b * channels + d) * nstate + n] : 0.0;
            const size_t tok0 = (size_t)(b * len) * (size_t)channels + (size_t)d;
            scan_row(len ? u + tok0 : NULL, len ? delta + tok0 : NULL, A + d * nstate,
                     len ? B + (size_t)(b * len) * (size_t)nstate : NULL,
                     len ? C + (size_t)(b * len) * (size_t)nstate : NULL,
                     D ? D[d] : 0.0, D != NULL, (y && len) ? y + tok0 : NULL, h,
                     len, channels, nstate);
            if (h_final)
                for (int64_t n = 0; n < nstate; ++n)
                    h_final[(b * channels + d) * nstate + n] = h[n];
        }
        free(h);
    }
    return status;
}

/* One recurrent (generation-time) step for every (batch, channel) row: the
 * O(1)-memory update the pages describe for inference ("Karmaşıklık
 * Karşılaştırması": a fixed-size hidden state is updated per token).
 * state [batch][channels][nstate] is updated in place; x, delta and y are
 * [batch][channels]; B, C are [batch][nstate].                              */
int oracle_state_update(double *state, const double *x, const double *delta,
                        const double *A, const double *B, const double *C,
                        const double *D, double *y,
                        int64_t batch, int64_t channels, int64_t nstate, int nthreads)
{
    if (batch < 0 || channels < 0 || nstate <= 0 || !state || !x || !delta || !A || !B || !C)
        return -1;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int64_t rows = batch * channels;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t b = r / channels, d = r % channels;
        scan_row(x + r, delta + r, A + d * nstate, B + b * nstate, C + b * nstate,
                 D ? D[d] : 0.0, D != NULL, y ? y + r : NULL, state + r * nstate,
                 1, channels, nstate);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Discretisations other than zero-order hold.
 *
 * The Mamba-3 page (bitig.info, section "Geliştirilmiş Ayrıklaştırma
 * Şeması") says Mamba-1 and Mamba-2 discretised the continuous system with
 * "the Euler method" and Mamba-3 with the trapezoidal rule, and gives no
 * formula for either.  Readings taken (the plainest forms that keep the
 * transition exp(Delta A) of "Ayrık Zamana Geçiş"):
 *   method 1, exponential Euler: the state transition stays exp(Delta A)
 *     (as in the zero-order hold of "Ayrık Zamana Geçiş"), the input term is
 *     taken to first order, Bbar = Delta B:
 *         h_t = exp(Delta_t A) h_{t-1} + Delta_t B_t x_t
 *   method 2, trapezoidal: the exact step is
 *         h_t = exp(Delta A) h_{t-1} + int_0^Delta exp(A (Delta - s)) B(s) x(s) ds
 *     and the trapezoid rule takes the integral from its two end points, the
 *     previous token at s = 0 and the current one at s = Delta:
 *         h_t = exp(Delta_t A) h_{t-1}
 *               + (Delta_t / 2) (exp(Delta_t A) B_{t-1} x_{t-1} + B_t x_t)
 *     with B_{-1} x_{-1} = 0: the first token of a call has no predecessor,
 *     also when an initial state is given.
 * For every method y_t = C_t . h_t + D x_t.
 * ------------------------------------------------------------------------ */
static void scan_row_method(const double *u, const double *delta, const double *A_row,
                            const double *B, const double *C, double D_d, int has_D,
                            double *y, double *h, int64_t len, int64_t stride, int64_t nstate,
                            int method)
{
    for (int64_t t = 0; t < len; ++t) {
        double x = u[t * stride];
        double dt = delta[t * stride];
        const double *Bt = B + t * nstate;
        const double *Ct = C + t * nstate;
        double acc = 0.0;
        for (int64_t n = 0; n < nstate; ++n) {
            double abar = exp(dt * A_row[n]);
            double input;
            if (method == 1) {
                input = dt * Bt[n] * x;
            } else {
                double previous = 0.0;   /* exp(Delta_t A) B_{t-1} x_{t-1} */
                if (t > 0)
                    previous = abar * B[(t - 1) * nstate + n] * u[(t - 1) * stride];
                input = 0.5 * dt * (previous + Bt[n] * x);
            }
            h[n] = abar * h[n] + input;
            acc += Ct[n] * h[n];
        }
        if (has_D)
            acc += D_d * x;
        if (y)
            y[t * stride] = acc;
    }
}

/* Selective scan with the discretisation `method` (0: zero-order hold, the
 * same as oracle_scan; 1: exponential Euler; 2: trapezoidal).  Returns 0, or
 * -1 on a bad argument.                                                       */
int oracle_scan_method(const double *u, const double *delta, const double *A,
                       const double *B, const double *C, const double *D,
                       const double *h0, double *y, double *h_final,
                       int64_t batch, int64_t len, int64_t channels, int64_t nstate,
                       int method, int nthreads)
{
    if (method == 0)
        return oracle_scan(u, delta, A, B, C, D, h0, y, h_final, batch, len, channels, nstate, nthreads);
    if (method != 1 && method != 2)
        return -1;
    if (batch < 0 || len < 0 || channels < 0 || nstate <= 0)
        return -1;
    if ((len > 0 && (!u || !delta || !B || !C)) || !A)
        return -1;
    int64_t rows = batch * channels;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = 0;
#pragma omp parallel
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)nstate);
        if (!h) {
#pragma omp atomic write
            status = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            if (!h)
                continue;
            int64_t b = r / channels, d = r % channels;
            for (int64_t n = 0; n < nstate; ++n)
                h[n] = h0 ? h0[(b * channels + d) * nstate + n] : 0.0;
            const size_t tok0 = (size_t)(b * len) * (size_t)channels + (size_t)d;
            scan_row_method(len ? u + tok0 : NULL, len ? delta + tok0 : NULL, A + d * nstate,
                            len ? B + (size_t)(b * len) * (size_t)nstate : NULL,
                            len ? C + (size_t)(b * len) * (size_t)nstate : NULL,
                            D ? D[d] : 0.0, D != NULL, (y && len) ? y + tok0 : NULL, h,
                            len, channels, nstate, method);
            if (h_final)
                for (int64_t n = 0; n < nstate; ++n)
                    h_final[(b * channels + d) * nstate + n] = h[n];
        }
        free(h);
    }
    return status;
}

/* ------------------------------------------------------------------------
 * Backward of the zero-order-hold scan (training).  The pages imply training
 * ("Mamba'nın Yeniliği: Selective SSM": Delta, B and C are learned
 * projections of the input) but print no gradient; this is reverse-mode
 * differentiation of exactly the recurrence of oracle_scan, written out by
 * the chain rule.  With lam_t = dL/dh_t (the adjoint), per state n and token
 * t (z = Delta_t A_n, r = exp(z), Bbar = (r - 1)/A_n B_{t,n}):
 *   lam_t     = C_t dy_t + r_{t+1} lam_{t+1}      (+ dh_final at t = L-1)
 *   du_t      = sum_n lam_t Bbar + D dy_t
 *   dDelta_t  = sum_n lam_t r (A_n h_{t-1} + B_{t,n} x_t)
 *   dA_n     += lam_t (Delta_t r h_{t-1} + x_t B_{t,n} Delta_t^2 psi(z))
 *               with psi(z) = (z e^z - (e^z - 1)) / z^2  (d Bbar / d A_n)
 *   dB_{t,n} += lam_t x_t (r - 1)/A_n          (summed over channels)
 *   dC_{t,n} += dy_t h_t                       (summed over channels)
 *   dD       += dy_t x_t
 *   dh0       = r_0 lam_0
 * Single-threaded: dB, dC and dA are sums over rows.
 * ------------------------------------------------------------------------ */
static double psi(double z)
{
    if (fabs(z) < 1e-3)  /* series: 1/2 + z/3 + z^2/8 + z^3/30 */
        return 0.5 + z * (1.0 / 3.0 + z * (1.0 / 8.0 + z / 30.0));
    return (z * exp(z) - expm1(z)) / (z * z);
}

int oracle_scan_backward(const double *u, const double *delta, const double *A,
                         const double *B, const double *C, const double *D,
                         const double *h0, const double *dy, const double *dh_final,
                         double *du, double *ddelta, double *dA, double *dB, double *dC,
                         double *dD, double *dh0,
                         int64_t batch, int64_t len, int64_t channels, int64_t nstate)
{
    if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || !A || !dA || !dB || !dC || !dh0)
        return -1;
    if (len > 0 && (!u || !delta || !B || !C || !dy || !du || !ddelta))
        return -1;
    for (int64_t i = 0; i < channels * nstate; ++i)
        dA[i] = 0.0;
    for (int64_t i = 0; i < batch * len * nstate; ++i)
        dB[i] = dC[i] = 0.0;
    if (dD)
        for (int64_t d = 0; d < channels; ++d)
            dD[d] = 0.0;
    double *hs = (double *)malloc(sizeof(double) * (size_t)((len + 1) * nstate));
    double *lam = (double *)malloc(sizeof(double) * (size_t)nstate);
    if (!hs || !lam) {
        free(hs);
        free(lam);
        return -1;
    }
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < channels; ++d) {
            const double *Ad = A + d * nstate;
            /* forward: hs[(t+1)*N + n] = h_t, hs[n] = h_{-1} */
            for (int64_t n = 0; n < nstate; ++n)
                hs[n] = h0 ? h0[(b * channels + d) * nstate + n] : 0.0;
            for (int64_t t = 0; t < len; ++t) {
                const size_t k = (size_t)(b * len + t);
                double x = u[k * channels + d], dt = delta[k * channels + d];
                for (int64_t n = 0; n < nstate; ++n) {
                    double abar, bbar;
                    zoh_discretise(dt, Ad[n], B[k * nstate + n], &abar, &bbar);
                    hs[(t + 1) * nstate + n] = abar * hs[t * nstate + n] + bbar * x;
                }
            }
            /* reverse */
            for (int64_t n = 0; n < nstate; ++n)
                lam[n] = dh_final ? dh_final[(b * channels + d) * nstate + n] : 0.0;
            for (int64_t t = len - 1; t >= 0; --t) {
                const size_t k = (size_t)(b * len + t);
                double x = u[k * channels + d], dt = delta[k * channels + d], g = dy[k * channels + d];
                double dut = D ? D[d] * g : 0.0, ddt = 0.0;
                if (dD)
                    dD[d] += g * x;
                for (int64_t n = 0; n < nstate; ++n) {
                    double a = Ad[n], bn = B[k * nstate + n];
                    double hprev = hs[t * nstate + n], ht = hs[(t + 1) * nstate + n];
                    dC[k * nstate + n] += g * ht;              /* y_t = C_t . h_t + D x_t      */
                    lam[n] += C[k * nstate + n] * g;           /* lam_t                       */
                    double z = dt * a, r = exp(z);
                    double phi = (z == 0.0) ? 1.0 : expm1(z) / z;
                    double bbar = phi * dt * bn;
                    dut += lam[n] * bbar;
                    ddt += lam[n] * r * (a * hprev + bn * x);
                    dA[d * nstate + n] += lam[n] * (dt * r * hprev + x * bn * dt * dt * psi(z));
                    dB[k * nstate + n] += lam[n] * x * phi * dt;
                    lam[n] *= r;                               /* towards lam_{t-1}           */
                }
                du[k * channels + d] = dut;
                ddelta[k * channels + d] = ddt;
            }
            for (int64_t n = 0; n < nstate; ++n)
                dh0[(b * channels + d) * nstate + n] = lam[n];
        }
    }
    free(hs);
    free(lam);
    return 0;
}

/* Threads the OpenMP runtime would use (for reporting the CPU baseline). */
/* ---------------------------------------------------------------------------
 * Complex-valued state.
 *
 * The Mamba-3 page (bitig.info), section "Karmaşık Değerli Durum
 * Güncellemesi": the state update uses complex numbers; complex eigenvalues
 * of the transition represent oscillation and rotation, and the page relates
 * them to data-dependent rotary embeddings.  It prints no formula.  Reading
 * taken: A stays diagonal with complex entries A[d][n] = A_re + i A_im
 * (A_re < 0); the zero-order hold of "Ayrık Zamana Geçiş" applies unchanged
 * in complex arithmetic,
 *     Abar = exp(Delta A),   Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B,
 * with B and C real as in the selective scan; the state is complex and the
 * output takes its real part,
 *     y_t = sum_n C_t[n] Re(h_t[n]) + D x_t.
 * Each step turns a state by the angle Delta_t A_im: the rotation depends on
 * the input through Delta.
 *
 * Layouts: A_re, A_im [channels][nstate]; h0, h_final
 * [batch][channels][nstate][2] with (re, im) adjacent; the rest as above.
 * ------------------------------------------------------------------------- */
static void scan_row_complex(const double *u, const double *delta, const double *Are_row,
                             const double *Aim_row, const double *B, const double *C, double D_d,
                             int has_D, double *y, double complex *h, int64_t len, int64_t stride,
                             int64_t nstate)
{
    for (int64_t t = 0; t < len; ++t) {
        double x = u[t * stride];
        double dt = delta[t * stride];
        const double *Bt = B + t * nstate;
        const double *Ct = C + t * nstate;
        double acc = 0.0;
        for (int64_t n = 0; n < nstate; ++n) {
            double complex a = Are_row[n] + I * Aim_row[n];
            double complex z = dt * a;
            double complex abar = cexp(z);
            double complex phi = (z == 0.0) ? 1.0 : (abar - 1.0) / z;  /* (Delta A)^-1 (e^{Delta A} - 1) */
            double complex bbar = phi * dt * Bt[n];
            h[n] = abar * h[n] + bbar * x;
            acc += Ct[n] * creal(h[n]);
        }
        if (has_D)
            acc += D_d * x;
        if (y)
            y[t * stride] = acc;
    }
}

int oracle_scan_complex(const double *u, const double *delta, const double *A_re, const double *A_im,
                        const double *B, const double *C, const double *D, const double *h0,
                        double *y, double *h_final, int64_t batch, int64_t len, int64_t channels,
                        int64_t nstate, int nthreads)
{
    if (batch < 0 || len < 0 || channels < 0 || nstate <= 0)
        return -1;
    if ((len > 0 && (!u || !delta || !B || !C)) || !A_re || !A_im)
        return -1;
    int64_t rows = batch * channels;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = 0;
#pragma omp parallel
    {
        double complex *h = (double complex *)malloc(sizeof(double complex) * (size_t)nstate);
        if (!h) {
#pragma omp atomic write
            status = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            if (!h)
                continue;
            int64_t b = r / channels, d = r % channels;
            for (int64_t n = 0; n < nstate; ++n) {
                const double *s0 = h0 ? h0 + ((b * channels + d) * nstate + n) * 2 : NULL;
                h[n] = s0 ? s0[0] + I * s0[1] : 0.0;
            }
            const size_t tok0 = (size_t)(b * len) * (size_t)channels + (size_t)d;
            scan_row_complex(len ? u + tok0 : NULL, len ? delta + tok0 : NULL, A_re + d * nstate,
                             A_im + d * nstate, len ? B + (size_t)(b * len) * (size_t)nstate : NULL,
                             len ? C + (size_t)(b * len) * (size_t)nstate : NULL, D ? D[d] : 0.0,
                             D != NULL, (y && len) ? y + tok0 : NULL, h, len, channels, nstate);
            if (h_final)
                for (int64_t n = 0; n < nstate; ++n) {
                    h_final[((b * channels + d) * nstate + n) * 2] = creal(h[n]);
                    h_final[((b * channels + d) * nstate + n) * 2 + 1] = cimag(h[n]);
                }
        }
        free(h);
    }
    return status;
}

/* ------------------------------------------------------------------------
 * Multi-input multi-output (MIMO) state update.
 *
 * The Mamba-3 page (bitig.info), sections "MIMO Mekanizmasının İşleyişi"
 * and "Seçici Durum Güncellemesindeki İyileştirmeler", says that MIMO
 * updates the hidden state once per step for several outputs at once,
 * widens what the state holds without enlarging the state transition
 * matrix or adding parameters, and gives every output channel its own
 * selective gate deciding how much of the state that output uses; it
 * prints no formula.  Reading taken (the plainest one that keeps the
 * zero-order hold of "Ayrık Zamana Geçiş" as written, with B a matrix):
 * per channel d the continuous system of "State Space Model Temelleri" has
 * R inputs and R outputs,
 *     h'(t) = A h(t) + B x(t),   y(t) = C h(t) + D x(t),
 * x(t), y(t) in R^R, B_t in R^{N x R} (columns B_t^(r)), C_t in R^{R x N}
 * (rows C_t^(r): the per-output selective gates), D = D_d I; A stays the
 * diagonal N x N transition with one step Delta_t per (token, channel), so
 *     Abar = exp(Delta A),
 *     Bbar x = (Delta A)^-1 (exp(Delta A) - I) Delta B x
 *            = sum_r (Delta A)^-1 (exp(Delta A) - I) Delta B^(r) x^(r),
 *     h_t = Abar h_{t-1} + sum_r Bbar^(r) x_t^(r),
 *     y_t^(r) = C_t^(r) . h_t + D_d x_t^(r).
 * B and C are per (batch, token, input/output r, state), shared by all
 * channels, as in the single-input scan.  With R = 1 this is oracle_scan,
 * operation for operation.
 *
 * Layouts: u, y [batch][len][ranks][channels]; delta [batch][len][channels];
 * B, C [batch][len][ranks][nstate]; A [channels][nstate]; D [channels] or
 * NULL; h0, h_final [batch][channels][nstate] (h0 may be NULL).
 * ------------------------------------------------------------------------ */
static void scan_row_mimo(const double *u, const double *delta, const double *A_row,
                          const double *B, const double *C, double D_d, int has_D,
                          double *y, double *h, int64_t len, int64_t channels, int64_t nstate,
                          int64_t ranks)
{
    for (int64_t t = 0; t < len; ++t) {
        const double dt = delta[t * channels];
        const double *xt = u + t * ranks * channels;         /* x_t^(r) = xt[r * channels] */
        const double *Bt = B + t * ranks * nstate;           /* B_t^(r)[n] = Bt[r * nstate + n] */
        const double *Ct = C + t * ranks * nstate;
        for (int64_t n = 0; n < nstate; ++n) {
            double abar = 1.0, in = 0.0;
            for (int64_t r = 0; r < ranks; ++r) {
                double bbar;
                zoh_discretise(dt, A_row[n], Bt[r * nstate + n], &abar, &bbar);
                in += bbar * xt[r * channels];               /* sum_r Bbar^(r) x_t^(r) */
            }
            h[n] = abar * h[n] + in;                         /* h_t = Abar h_{t-1} + Bbar x_t */
        }
        for (int64_t r = 0; r < ranks; ++r) {
            double acc = 0.0;
            for (int64_t n = 0; n < nstate; ++n)
                acc += Ct[r * nstate + n] * h[n];            /* C_t^(r) . h_t */
            if (has_D)
                acc += D_d * xt[r * channels];               /* + D x_t^(r)   */
            if (y)
                y[(t * ranks + r) * channels] = acc;
        }
    }
}

int oracle_scan_mimo(const double *u, const double *delta, const double *A,
                     const double *B, const double *C, const double *D,
                     const double *h0, double *y, double *h_final,
                     int64_t batch, int64_t len, int64_t channels, int64_t nstate, int64_t ranks,
                     int nthreads)
{
    if (batch < 0 || len < 0 || channels < 0 || nstate <= 0 || ranks <= 0)
        return -1;
    if ((len > 0 && (!u || !delta || !B || !C)) || !A)
        return -1;
    int64_t rows = batch * channels;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = 0;
#pragma omp parallel
    {
        double *h = (double *)malloc(sizeof(double) * (size_t)nstate);
        if (!h) {
#pragma omp atomic write
            status = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            if (!h)
                continue;
            int64_t b = r / channels, d = r % channels;
            for (int64_t n = 0; n < nstate; ++n)
                h[n] = h0 ? h0[(b * channels + d) * nstate + n] : 0.0;
            const size_t x0 = (size_t)(b * len) * (size_t)(ranks * channels) + (size_t)d;
            const size_t bc0 = (size_t)(b * len) * (size_t)(ranks * nstate);
            scan_row_mimo(len ? u + x0 : NULL, len ? delta + (size_t)(b * len) * (size_t)channels + (size_t)d : NULL,
                          A + d * nstate, len ? B + bc0 : NULL, len ? C + bc0 : NULL, D ? D[d] : 0.0,
                          D != NULL, (y && len) ? y + x0 : NULL, h, len, channels, nstate, ranks);
            if (h_final)
                for (int64_t n = 0; n < nstate; ++n)
                    h_final[(b * channels + d) * nstate + n] = h[n];
        }
        free(h);
    }
    return status;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
