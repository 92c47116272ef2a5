/*
 * ssm_oracle.c -- plain, slow, fp64 CPU oracle of the selective SSM (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * What it computes, and where each step comes from:
 *
 *  - Discretisation (NL-345, Mamba: Linear-Time Sequence Modeling with
 *    Selective State Spaces, section 2 "Discretization"; 【論文要約】Mamba
 *    notes, 数式解説 3 "ZOH"): Abar = exp(Delta * A), elementwise because A is
 *    diagonal (NL-345 section 2 "Structure and Dimensions").  Bbar is either
 *    the Euler form Delta * B (the library's convention) or the exact
 *    zero-order hold (Delta A)^-1 (exp(Delta A) - 1) Delta B = expm1(Delta A)/A * B
 *    (the notes' ZOH formula); with A == 0 the ZOH limit is Delta * B.
 *  - Recurrence and readout (NL-345 section 2, eq. (2)):
 *        h_t = Abar_t h_{t-1} + Bbar_t x_t,   y_t = C_t h_t,
 *    so y_t reads the state *after* x_t has entered it.
 *  - Selection (【論文要約】Mamba notes, "S6", Algorithm 2): B_t and C_t are
 *    per-token inputs shared by all channels; Delta_t = tau_Delta(bias +
 *    Delta_raw_t) with tau_Delta = softplus (the notes' Theorem 1), or the plain
 *    sum when softplus is off.  A is a static (dim x dstate) parameter.
 *  - Skip and gate (the library's fused block epilogue, not on the pages):
 *        out = (y + D u) * silu(z),  silu(z) = z / (1 + exp(-z));
 *    a NULL D means D = 0 and a NULL z means no gate.
 *  - Each channel (b, d) is an independent SSM (NL-345 section 2 "Structure
 *    and Dimensions"), so channels are distributed over threads; inside a
 *    channel the loop runs in time order and, for each step, in state order,
 *    exactly as written above.  Thread count never changes a result.
 *
 * Layouts (dense, row-major): u, delta, z, out (batch, seqlen, dim);
 * B, C (batch, seqlen, dstate); A (dim, dstate); D, delta_bias (dim);
 * state (batch, dim, dstate).  All values are double.
 */
#include <complex.h>
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2

/* softplus(s) = log(1 + e^s), evaluated as max(s, 0) + log1p(e^-|s|):
 * the same function, without overflow for large s and without the loss of
 * relative precision that log(1 + tiny) would have for very negative s. */
static double oracle_softplus(double s)
{
    double m = s > 0.0 ? s : 0.0;
    return m + log1p(exp(-fabs(s)));
}

static double oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

typedef struct {
    int64_t batch, seqlen, dim, dstate;
    const double *u, *delta, *A, *B, *C, *Dskip, *z, *bias;
    int softplus, zoh_b;
    double *out, *state;
    int64_t c_begin, c_end; /* channel range, channel = b * dim + d */
    int status;
} scan_job;

static void scan_channels(scan_job *j)
{
    const int64_t L = j->seqlen, Dm = j->dim, N = j->dstate;
    double *h = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
    if (!h) { j->status = ORACLE_NO_MEM; return; }
    for (int64_t c = j->c_begin; c < j->c_end; ++c) {
        const int64_t b = c / Dm, d = c % Dm;
        for (int64_t n = 0; n < N; ++n)
            h[n] = j->state ? j->state[(b * Dm + d) * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const int64_t td = (b * L + t) * Dm + d;  /* (b, t, d) */
            const int64_t tn = (b * L + t) * N;       /* (b, t, 0) */
            const double x = j->u[td];
            double s = j->delta[td] + (j->bias ? j->bias[d] : 0.0);
            const double dlt = j->softplus ? oracle_softplus(s) : s;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double an = j->A[d * N + n];
                const double abar = exp(dlt * an);
                double bbar;
                if (j->zoh_b)
                    bbar = (an == 0.0 ? dlt : expm1(dlt * an) / an) * j->B[tn + n];
                else
                    bbar = dlt * j->B[tn + n];
                h[n] = abar * h[n] + bbar * x;
                acc += j->C[tn + n] * h[n];
            }
            double y = acc + (j->Dskip ? j->Dskip[d] * x : 0.0);
            if (j->z) y *= oracle_silu(j->z[td]);
            j->out[td] = y;
        }
        if (j->state)
            for (int64_t n = 0; n < N; ++n)
                j->state[(b * Dm + d) * N + n] = h[n];
    }
    free(h);
    j->status = ORACLE_OK;
}

static void *scan_thread(void *p)
{
    scan_channels((scan_job *)p);
    return NULL;
}

static int resolve_threads(int nthreads, int64_t channels)
{
    if (nthreads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = n > 0 ? (int)n : 1;
    }
    if (nthreads > 1024) nthreads = 1024;
    if ((int64_t)nthreads > channels) nthreads = (int)(channels > 0 ? channels : 1);
    return nthreads;
}

/* Number of threads a call with nthreads <= 0 would use on this host. */
int oracle_default_threads(void)
{
    return resolve_threads(0, INT64_MAX);
}

/*
 * Selective scan over all (batch, dim) channels.
 *   zoh_b = 0: Bbar = Delta * B (Euler);  zoh_b = 1: exact ZOH Bbar.
 *   state: NULL => h0 = 0 and the final state is not returned; otherwise it
 *          holds h0 on entry and h_L on return.
 *   nthreads <= 0 uses every online core.
 * Returns 0 on success.
 */
int oracle_selective_scan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                          const double *u, const double *delta, const double *A,
                          const double *B, const double *C, const double *Dskip,
                          const double *z, const double *delta_bias, int delta_softplus,
                          int zoh_b, double *out, double *state, int nthreads)
{
    if (batch < 0 || seqlen < 0 || dim < 0 || dstate < 0) return ORACLE_BAD_ARG;
    const int64_t channels = batch * dim;
    if (channels == 0) return ORACLE_OK;
    if (seqlen > 0 && (!u || !delta || !B || !C || !out)) return ORACLE_BAD_ARG;
    if (dstate > 0 && !A) return ORACLE_BAD_ARG;
    int nt = resolve_threads(nthreads, channels);
    scan_job *jobs = (scan_job *)calloc((size_t)nt, sizeof(scan_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return ORACLE_NO_MEM; }
    for (int i = 0; i < nt; ++i) {
        scan_job *j = &jobs[i];
        j->batch = batch; j->seqlen = seqlen; j->dim = dim; j->dstate = dstate;
        j->u = u; j->delta = delta; j->A = A; j->B = B; j->C = C;
        j->Dskip = Dskip; j->z = z; j->bias = delta_bias;
        j->softplus = delta_softplus; j->zoh_b = zoh_b;
        j->out = out; j->state = state;
        j->c_begin = channels * i / nt;
        j->c_end = channels * (i + 1) / nt;
        j->status = ORACLE_BAD_ARG;
    }
    int started = 0;
    for (int i = 1; i < nt; ++i) {
        if (pthread_create(&th[i], NULL, scan_thread, &jobs[i]) != 0) break;
        started = i;
    }
    scan_channels(&jobs[0]);
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    for (int i = started + 1; i < nt; ++i) scan_channels(&jobs[i]); /* threads that failed to start */
    int rc = ORACLE_OK;
    for (int i = 0; i < nt; ++i)
        if (jobs[i].status != ORACLE_OK) rc = jobs[i].status;
    free(jobs);
    free(th);
    return rc;
}

/*
 * Selective scan with a complex diagonal A (and complex B, C): the
 * parameterisation the Mamba notes single out for audio (【論文要約】Mamba
 * notes, Figure 10: complex parameters matter there; Table 8, the A
 * initialisation ablation).  The pages give no formula for it, so this is the
 * plain reading of the real recurrence with complex numbers:
 *     Abar = exp(Delta A)            (complex exponential; Delta is real)
 *     Bbar = Delta B                 (Euler form, as for the real scan)
 *     h_t  = Abar h_{t-1} + Bbar x_t (complex state)
 *     y_t  = Re(sum_n C_t,n h_t,n) + D x_t,   out = y silu(z)
 * u, delta, z, out, D, delta_bias are real as before.  Complex arrays hold
 * (re, im) pairs: A (dim, dstate, 2), B and C (batch, seqlen, dstate, 2),
 * state (batch, dim, dstate, 2).  state: NULL => h0 = 0 and the final state
 * is not returned.  Single-threaded.  Returns 0 on success.
 */
int oracle_selective_scan_complex(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                  const double *u, const double *delta, const double *A,
                                  const double *B, const double *C, const double *Dskip,
                                  const double *z, const double *delta_bias, int delta_softplus,
                                  double *out, double *state)
{
    const int64_t L = seqlen, Dm = dim, N = dstate;
    if (batch < 0 || L < 0 || Dm < 0 || N < 0) return ORACLE_BAD_ARG;
    if (batch * Dm == 0) return ORACLE_OK;
    if (L > 0 && (!u || !delta || !B || !C || !out)) return ORACLE_BAD_ARG;
    if (N > 0 && !A) return ORACLE_BAD_ARG;
    double complex *h = (double complex *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double complex));
    if (!h) return ORACLE_NO_MEM;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < Dm; ++d) {
            const int64_t so = (b * Dm + d) * N;
            for (int64_t n = 0; n < N; ++n)
                h[n] = state ? state[2 * (so + n)] + I * state[2 * (so + n) + 1] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t td = (b * L + t) * Dm + d;
                const int64_t tn = (b * L + t) * N;
                const double x = u[td];
                const double s = delta[td] + (delta_bias ? delta_bias[d] : 0.0);
                const double dlt = delta_softplus ? oracle_softplus(s) : s;
                double complex acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double complex an = A[2 * (d * N + n)] + I * A[2 * (d * N + n) + 1];
                    const double complex bn = B[2 * (tn + n)] + I * B[2 * (tn + n) + 1];
                    const double complex cn = C[2 * (tn + n)] + I * C[2 * (tn + n) + 1];
                    const double complex abar = cexp(dlt * an);
                    h[n] = abar * h[n] + (dlt * bn) * x;
                    acc += cn * h[n];
                }
                double y = creal(acc) + (Dskip ? Dskip[d] * x : 0.0);
                if (z) y *= oracle_silu(z[td]);
                out[td] = y;
            }
            if (state)
                for (int64_t n = 0; n < N; ++n) {
                    state[2 * (so + n)] = creal(h[n]);
                    state[2 * (so + n) + 1] = cimag(h[n]);
                }
        }
    }
    free(h);
    return ORACLE_OK;
}

/*
 * Gradient of the selective scan (Euler Bbar) for upstream gradients dout of
 * the output: the chain rule applied to the forward loop of
 * oracle_selective_scan, in reverse time.  Per channel the forward states
 * h_{-1..L-1} are first stored (this is a reference; the library recomputes
 * them instead), then with lambda_t = dL/dh_t:
 *     dy_t      = dout_t silu(z_t)        (dout_t without a gate)
 *     dz_t      = dout_t y_t silu'(z_t),  silu'(z) = s (1 + z (1 - s)), s = sigmoid(z)
 *     lambda_t  = dy_t C_t + Abar_{t+1} lambda_{t+1}
 *     dC_t     += dy_t h_t                (summed over channels)
 *     dDelta_t  = sum_n lambda_t,n (h_{t-1},n Abar_t,n A_n + B_t,n u_t)
 *     dA_n     += lambda_t,n h_{t-1},n Abar_t,n Delta_t
 *     dB_t,n   += lambda_t,n Delta_t u_t  (summed over channels)
 *     du_t      = dy_t D + Delta_t sum_n lambda_t,n B_t,n
 *     dD       += dy_t u_t
 *     ddelta_t  = dDelta_t sigmoid(delta_t + bias) (softplus on) or dDelta_t
 *     dbias    += ddelta_t;   dh0 = Abar_0 lambda_0
 * Every gradient array is overwritten.  dz may be NULL when z is NULL; dh0 may
 * be NULL.  Single-threaded (the channel-shared gradients are plain sums).
 */
int oracle_selective_scan_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                              const double *u, const double *delta, const double *A,
                              const double *B, const double *C, const double *Dskip,
                              const double *z, const double *delta_bias, int delta_softplus,
                              const double *h0, const double *dout, double *du, double *ddelta,
                              double *dA, double *dB, double *dC, double *dD, double *dz,
                              double *ddelta_bias, double *dh0)
{
    const int64_t L = seqlen, Dm = dim, N = dstate;
    if (batch < 0 || L < 0 || Dm < 0 || N < 0) return ORACLE_BAD_ARG;
    if (!du || !ddelta || !dA || !dB || !dC || !dD || !ddelta_bias || (z && !dz)) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < Dm * N; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < batch * L * N; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    for (int64_t i = 0; i < Dm; ++i) { dD[i] = 0.0; ddelta_bias[i] = 0.0; }
    double *hs = (double *)malloc((size_t)((L + 1) * (N > 0 ? N : 1)) * sizeof(double));
    double *dl = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    double *yv = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    double *lam = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
    if (!hs || !dl || !yv || !lam) { free(hs); free(dl); free(yv); free(lam); return ORACLE_NO_MEM; }
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < Dm; ++d) {
            /* forward, keeping every state: hs[(t + 1) N + n] = h_t[n] */
            for (int64_t n = 0; n < N; ++n) hs[n] = h0 ? h0[(b * Dm + d) * N + n] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t td = (b * L + t) * Dm + d, tn = (b * L + t) * N;
                const double s = delta[td] + (delta_bias ? delta_bias[d] : 0.0);
                dl[t] = delta_softplus ? oracle_softplus(s) : s;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double h = exp(dl[t] * A[d * N + n]) * hs[t * N + n] + dl[t] * B[tn + n] * u[td];
                    hs[(t + 1) * N + n] = h;
                    acc += C[tn + n] * h;
                }
                yv[t] = acc + (Dskip ? Dskip[d] * u[td] : 0.0);
            }
            /* reverse */
            for (int64_t n = 0; n < N; ++n) lam[n] = 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const int64_t td = (b * L + t) * Dm + d, tn = (b * L + t) * N;
                double dy = dout[td];
                if (z) {
                    const double sg = 1.0 / (1.0 + exp(-z[td]));
                    dy = dout[td] * z[td] * sg;
                    dz[td] = dout[td] * yv[t] * sg * (1.0 + z[td] * (1.0 - sg));
                }
                if (Dskip) dD[d] += dy * u[td];
                double dut = Dskip ? dy * Dskip[d] : 0.0;
                double ddl = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double an = A[d * N + n];
                    const double abar = exp(dl[t] * an);
                    const double hprev = hs[t * N + n];
                    lam[n] += dy * C[tn + n];
                    dC[tn + n] += dy * hs[(t + 1) * N + n];
                    ddl += lam[n] * (hprev * abar * an + B[tn + n] * u[td]);
                    dA[d * N + n] += lam[n] * hprev * abar * dl[t];
                    dB[tn + n] += lam[n] * dl[t] * u[td];
                    dut += lam[n] * dl[t] * B[tn + n];
                    lam[n] *= abar;
                }
                du[td] = dut;
                double sv = delta[td] + (delta_bias ? delta_bias[d] : 0.0);
                const double dd = delta_softplus ? ddl / (1.0 + exp(-sv)) : ddl;
                ddelta[td] = dd;
                ddelta_bias[d] += dd;
            }
            if (dh0)
                for (int64_t n = 0; n < N; ++n) dh0[(b * Dm + d) * N + n] = lam[n];
        }
    }
    free(hs); free(dl); free(yv); free(lam);
    return ORACLE_OK;
}

/*
 * One recurrent (decode) step for every channel (NL-345 section 1: constant
 * time per generated step; section 2 eq. (2) for one t).  dt is the time step
 * itself (already positive: no bias, no softplus).  state (batch, dim, dstate)
 * is updated in place; x, dt, z, out are (batch, dim); B, C are (batch, dstate).
 */
int oracle_state_update(int64_t batch, int64_t dim, int64_t dstate, double *state,
                        const double *x, const double *dt, const double *A,
                        const double *B, const double *C, const double *Dskip,
                        const double *z, double *out)
{
    if (batch < 0 || dim < 0 || dstate < 0) return ORACLE_BAD_ARG;
    if (batch * dim == 0) return ORACLE_OK;
    if (!state || !x || !dt || !B || !C || !out || (dstate > 0 && !A)) return ORACLE_BAD_ARG;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const double dlt = dt[b * dim + d];
            const double xv = x[b * dim + d];
            double *h = state + (b * dim + d) * dstate;
            double acc = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                const double abar = exp(dlt * A[d * dstate + n]);
                h[n] = abar * h[n] + dlt * B[b * dstate + n] * xv;
                acc += C[b * dstate + n] * h[n];
            }
            double y = acc + (Dskip ? Dskip[d] * xv : 0.0);
            if (z) y *= oracle_silu(z[b * dim + d]);
            out[b * dim + d] = y;
        }
    }
    return ORACLE_OK;
}

/*
 * Mamba-2's structured state space duality (SSD) layer, in its linear
 * (recurrent) form ("Transformers are SSMs" review, nubint.ai: 提案手法 --
 * an SSM is a matrix transformation; the linear recurrence and the quadratic,
 * attention-like form compute the same map).  The review prints no formula;
 * the plain reading, shared with the Mamba notes' selective SSM, is:
 *   heads h = 0..H-1 of P channels each; groups g = 0..G-1 of H/G heads that
 *   share B_t and C_t (the review's grouped-value attention); A is one scalar
 *   per head, so Abar is a scalar times the identity;
 *   Delta_t = softplus(dt[b,t,h] + dt_bias[h]) (or the plain sum), one per head;
 *   for every channel (b, h, p) and state n, in time order:
 *       state[n] = exp(Delta_t A_h) state[n] + Delta_t B[b,t,g,n] x[b,t,h,p]
 *       y        = sum_n C[b,t,g,n] state[n] + D_h x[b,t,h,p]
 *       out      = y * silu(z[b,t,h,p])   (z NULL: no gate; D NULL: no skip)
 * Layouts (dense, row-major): x, z, out (batch, seqlen, heads, headdim);
 * dt (batch, seqlen, heads); A, D, dt_bias (heads); B, C (batch, seqlen,
 * groups, dstate); state (batch, heads, headdim, dstate), h0 in and h_L out
 * (NULL: h0 = 0, not returned).  Single-threaded; returns 0 on success.
 */
int oracle_ssd_scan(int64_t batch, int64_t seqlen, int64_t heads, int64_t headdim, int64_t groups,
                    int64_t dstate, const double *x, const double *dt, const double *A,
                    const double *B, const double *C, const double *D, const double *z,
                    const double *dt_bias, int dt_softplus, double *out, double *state)
{
    if (batch < 0 || seqlen < 0 || heads < 0 || headdim < 0 || groups < 1 || dstate < 0) return ORACLE_BAD_ARG;
    if (heads % groups != 0) return ORACLE_BAD_ARG;
    if (batch * heads * headdim == 0) return ORACLE_OK;
    if (seqlen > 0 && (!x || !dt || !A || !B || !C || !out)) return ORACLE_BAD_ARG;
    const int64_t L = seqlen, H = heads, P = headdim, N = dstate, hpg = heads / groups;
    double *h = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
    if (!h) return ORACLE_NO_MEM;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t hd = 0; hd < H; ++hd) {
            const int64_t g = hd / hpg;
            for (int64_t p = 0; p < P; ++p) {
                double *st = state ? state + ((b * H + hd) * P + p) * N : NULL;
                for (int64_t n = 0; n < N; ++n) h[n] = st ? st[n] : 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    const double s = dt[(b * L + t) * H + hd] + (dt_bias ? dt_bias[hd] : 0.0);
                    const double dlt = dt_softplus ? oracle_softplus(s) : s;
                    const double abar = exp(dlt * A[hd]);
                    const int64_t xi = ((b * L + t) * H + hd) * P + p;
                    const int64_t bi = ((b * L + t) * groups + g) * N;
                    const double xv = x[xi];
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        h[n] = abar * h[n] + dlt * B[bi + n] * xv;
                        acc += C[bi + n] * h[n];
                    }
                    double y = acc + (D ? D[hd] * xv : 0.0);
                    if (z) y *= oracle_silu(z[xi]);
                    out[xi] = y;
                }
                if (st)
                    for (int64_t n = 0; n < N; ++n) st[n] = h[n];
            }
        }
    free(h);
    return ORACLE_OK;
}
