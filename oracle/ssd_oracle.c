/*
 * CPU oracle for the Mamba-2 SSD sequence mixer -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline leg may load this
 * library.  It shares no code, header or constant with the CUDA path; it is the plain, slow,
 * token-by-token definition of what that path computes, in float64, so that the chunked GPU
 * algorithm can be checked against it element by element.
 *
 * What it computes (per batch b, head h, with g = h / (H/G) the group of head h):
 *
 *     a_t      = exp(dt_t * A_h)                               scalar decay of the state
 *     S_t      = a_t * S_{t-1} + dt_t * x_t (outer) B_t        P x N state, S_{-1} = h0 or 0
 *     y_t[p]   = sum_n S_t[p][n] * C_t[n]  +  D_h * x_t[p]
 *
 * Sources, by page and section:
 *   - the selective SSM recurrence h_t = A_t h_{t-1} + B_t x_t, y_t = C_t h_t
 *     (ql.gl "Why Does Mamba-2 Resemble the Transformer?", The Problem; eightmm.github.io
 *     "Mamba-2", Question);
 *   - A_t restricted to a scalar times identity, one scalar per head and token
 *     (chipfoundryservices.com "hybrid attention-SSM", third paragraph; crackai.dev
 *     "Transformers are SSMs", How It Works);
 *   - A-bar = exp(dt A) and the skip term D x (mohakchugh.is-a.dev "Mamba-2", State Space
 *     Models: The Core Abstraction);
 *   - the input enters as dt * x (the same page, Architecture: Multi-Head SSM, which feeds
 *     x * dt to the scan), i.e. B-bar x = dt B x rather than the zero-order-hold B-bar;
 *   - y_t includes the current token: the decay product over j = i+1..t is empty at i = t
 *     (eightmm.github.io "Mamba-2", Matrix Mixer View), so the state is updated before the
 *     readout.
 *
 * The chunked (block-decomposed) algorithm reaches this same result in exact arithmetic
 * (ql.gl, The Core of SSD: chunking preserves the meaning of the sequential state
 * computation), so this recurrence is the reference for every output of the scan and of the
 * decode update, which is the same recurrence run one token per call.
 *
 * Layouts (all row-major, float64):
 *   x  (b, L, H, P)   dt (b, L, H)   A (H)   B, C (b, L, G, N)   D (H)
 *   h0, final state (b, H, P, N)     y (b, L, H, P)
 *   boundary states (b, H, nb, P, N): the state after token (k+1)*every - 1, k = 0..nb-1.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fused multiply-add, so every
 * operation rounds as written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Run the recurrence for one (b, h).  Returns 0, or -1 if the state could not be allocated. */
static int scan_one(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t N,
                    int64_t G, const double *x, const double *dt, const double *A,
                    const double *B, const double *C, const double *D, const double *h0,
                    double *y, double *final_state, double *boundary, int64_t every,
                    int64_t nb)
{
    const int64_t g = h / (H / G);
    double *S = (double *)malloc((size_t)(P * N) * sizeof(double));
    if (!S)
        return -1;
    if (h0)
        memcpy(S, h0 + (b * H + h) * P * N, (size_t)(P * N) * sizeof(double));
    else
        memset(S, 0, (size_t)(P * N) * sizeof(double));

    for (int64_t t = 0; t < L; ++t) {
        const double dtt = dt[(b * L + t) * H + h];
        const double a = exp(dtt * A[h]);
        const double *xt = x + ((b * L + t) * H + h) * P;
        const double *Bt = B + ((b * L + t) * G + g) * N;
        const double *Ct = C + ((b * L + t) * G + g) * N;
        double *yt = y + ((b * L + t) * H + h) * P;
        for (int64_t p = 0; p < P; ++p) {
            double *Sp = S + p * N;
            const double u = dtt * xt[p];
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                Sp[n] = a * Sp[n] + u * Bt[n];
                acc += Sp[n] * Ct[n];
            }
            yt[p] = acc + D[h] * xt[p];
        }
        if (boundary && every > 0 && (t + 1) % every == 0 && (t + 1) / every <= nb) {
            const int64_t k = (t + 1) / every - 1;
            memcpy(boundary + ((b * H + h) * nb + k) * P * N, S,
                   (size_t)(P * N) * sizeof(double));
        }
    }
    if (final_state)
        memcpy(final_state + (b * H + h) * P * N, S, (size_t)(P * N) * sizeof(double));
    free(S);
    return 0;
}

/*
 * Full scan.  bh (nullable) lists n_bh flattened indices b*H + h to compute; when NULL every
 * (b, h) is computed.  Outputs of (b, h) pairs not listed are left untouched.  final_state and
 * boundary are nullable.  Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int oracle_ssd_scan(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                    int64_t dstate, int64_t ngroups, const double *x, const double *dt,
                    const double *A, const double *B, const double *C, const double *D,
                    const double *h0, double *y, double *final_state, double *boundary,
                    int64_t every, int64_t nb, const int64_t *bh, int64_t n_bh)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 ||
        ngroups <= 0 || nheads % ngroups != 0)
        return -1;
    const int64_t total = bh ? n_bh : batch * nheads;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int64_t i = 0; i < total; ++i) {
        const int64_t f = bh ? bh[i] : i;
        if (f < 0 || f >= batch * nheads) {
            failed |= 1;
            continue;
        }
        failed |= scan_one(f / nheads, f % nheads, seqlen, nheads, headdim, dstate, ngroups, x,
                           dt, A, B, C, D, h0, y, final_state, boundary, every, nb) != 0;
    }
    return failed ? -1 : 0;
}

/*
 * Gradients of  loss = sum_t <dy_t, y_t> + <dfinal, S_{L-1}>  through the recurrence above, for
 * one (b, h): reverse-mode differentiation of the token loop.  The pages give no backward; this
 * is the derivative of the forward definition, written out step by step:
 *
 *     G_t      = dy_t (outer) C_t + a_{t+1} G_{t+1}        adjoint of S_t (P x N);
 *                G_{L-1} = dy_{L-1} (outer) C_{L-1} + dfinal
 *     dx_t     = D_h dy_t + dt_t G_t B_t                   (S_t depends on x_t through dt_t x_t B_t)
 *     dB_t    += dt_t G_t^T x_t                            (this head's share of its group's dB)
 *     dC_t    += S_t^T dy_t                                (this head's share of its group's dC)
 *     dl_t     = a_t <G_t, S_{t-1}>                        (adjoint of l_t = dt_t A_h, a_t = exp(l_t))
 *     ddt_t    = <G_t B_t, x_t> + A_h dl_t
 *     dA_h    += dt_t dl_t,     dD_h += <dy_t, x_t>,        dinit = a_0 G_0
 *
 * The backward sweep needs S_{t-1} at every t.  Instead of keeping all L states, the forward
 * sweep stores every `seg`-th state and the backward sweep re-runs the same recurrence from that
 * checkpoint over one segment at a time: the same operations in the same order, so the states
 * are bit-identical to a forward sweep that kept them all.
 *
 * Outputs for this (b, h): dx (b, L, H, P), ddt (b, L, H), dB_h and dC_h (b, L, H, N) -- the
 * head's contribution, summed over the group's heads by the caller -- dA_bh and dD_bh (b, H) --
 * the head's sum over t, summed over the batch by the caller -- and dinit (b, H, P, N).
 */
static int bwd_one(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                   const double *x, const double *dt, const double *A, const double *B,
                   const double *C, const double *D, const double *h0, const double *dy,
                   const double *dfinal, double *dx, double *ddt, double *dB_h, double *dC_h,
                   double *dA_bh, double *dD_bh, double *dinit)
{
    const int64_t g = h / (H / G);
    const int64_t PN = P * N;
    const int64_t seg = 64;
    const int64_t nseg = (L + seg - 1) / seg;
    /* ck[k] = state before token k * seg; run[j] = state after token k * seg + j */
    double *ck = (double *)malloc((size_t)((nseg > 0 ? nseg : 1) * PN) * sizeof(double));
    double *run = (double *)malloc((size_t)(seg * PN) * sizeof(double));
    double *S = (double *)malloc((size_t)PN * sizeof(double));
    double *Gt = (double *)malloc((size_t)PN * sizeof(double));
    if (!ck || !run || !S || !Gt) {
        free(ck); free(run); free(S); free(Gt);
        return -1;
    }

    /* forward sweep: checkpoints and dC_t = S_t^T dy_t */
    if (h0)
        memcpy(S, h0 + (b * H + h) * PN, (size_t)PN * sizeof(double));
    else
        memset(S, 0, (size_t)PN * sizeof(double));
    for (int64_t t = 0; t < L; ++t) {
        if (t % seg == 0)
            memcpy(ck + (t / seg) * PN, S, (size_t)PN * sizeof(double));
        const double dtt = dt[(b * L + t) * H + h];
        const double a = exp(dtt * A[h]);
        const double *xt = x + ((b * L + t) * H + h) * P;
        const double *Bt = B + ((b * L + t) * G + g) * N;
        const double *dyt = dy + ((b * L + t) * H + h) * P;
        double *dCt = dC_h + ((b * L + t) * H + h) * N;
        for (int64_t p = 0; p < P; ++p) {
            const double u = dtt * xt[p];
            for (int64_t n = 0; n < N; ++n)
                S[p * N + n] = a * S[p * N + n] + u * Bt[n];
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t p = 0; p < P; ++p)
                acc += S[p * N + n] * dyt[p];
            dCt[n] = acc;
        }
    }

    /* backward sweep, one segment at a time from the last */
    if (dfinal)
        memcpy(Gt, dfinal + (b * H + h) * PN, (size_t)PN * sizeof(double));
    else
        memset(Gt, 0, (size_t)PN * sizeof(double));
    double anext = 1.0;   /* a_{t+1}; G_{L-1} takes dfinal with factor 1 */
    double dA_acc = 0.0, dD_acc = 0.0;
    for (int64_t k = nseg - 1; k >= 0; --k) {
        const int64_t t0 = k * seg;
        const int64_t t1 = (t0 + seg < L) ? t0 + seg : L;
        /* re-run the segment: run[j] = S_{t0 + j} */
        memcpy(S, ck + k * PN, (size_t)PN * sizeof(double));
        for (int64_t t = t0; t < t1; ++t) {
            const double dtt = dt[(b * L + t) * H + h];
            const double a = exp(dtt * A[h]);
            const double *xt = x + ((b * L + t) * H + h) * P;
            const double *Bt = B + ((b * L + t) * G + g) * N;
            for (int64_t p = 0; p < P; ++p) {
                const double u = dtt * xt[p];
                for (int64_t n = 0; n < N; ++n)
                    S[p * N + n] = a * S[p * N + n] + u * Bt[n];
            }
            memcpy(run + (t - t0) * PN, S, (size_t)PN * sizeof(double));
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const double dtt = dt[(b * L + t) * H + h];
            const double a = exp(dtt * A[h]);
            const double *xt = x + ((b * L + t) * H + h) * P;
            const double *Bt = B + ((b * L + t) * G + g) * N;
            const double *Ct = C + ((b * L + t) * G + g) * N;
            const double *dyt = dy + ((b * L + t) * H + h) * P;
            const double *Sprev = (t > t0) ? run + (t - 1 - t0) * PN
                                           : (t == 0 ? NULL : ck + k * PN);
            /* G_t = dy_t (outer) C_t + a_{t+1} G_{t+1} */
            for (int64_t p = 0; p < P; ++p)
                for (int64_t n = 0; n < N; ++n)
                    Gt[p * N + n] = dyt[p] * Ct[n] + anext * Gt[p * N + n];
            double *dxt = dx + ((b * L + t) * H + h) * P;
            double gbx = 0.0;
            for (int64_t p = 0; p < P; ++p) {
                double gb = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    gb += Gt[p * N + n] * Bt[n];
                dxt[p] = D[h] * dyt[p] + dtt * gb;
                gbx += gb * xt[p];
            }
            double *dBt = dB_h + ((b * L + t) * H + h) * N;
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t p = 0; p < P; ++p)
                    acc += Gt[p * N + n] * xt[p];
                dBt[n] = dtt * acc;
            }
            double gs = 0.0;   /* <G_t, S_{t-1}>, with S_{-1} = h0 or 0 */
            const double *Sp = Sprev ? Sprev : (h0 ? h0 + (b * H + h) * PN : NULL);
            if (Sp)
                for (int64_t i = 0; i < PN; ++i)
                    gs += Gt[i] * Sp[i];
            const double dl = a * gs;
            ddt[(b * L + t) * H + h] = gbx + A[h] * dl;
            dA_acc += dtt * dl;
            double xdy = 0.0;
            for (int64_t p = 0; p < P; ++p)
                xdy += dyt[p] * xt[p];
            dD_acc += xdy;
            anext = a;
        }
    }
    for (int64_t i = 0; i < PN; ++i)
        dinit[(b * H + h) * PN + i] = anext * Gt[i];
    dA_bh[b * H + h] = dA_acc;
    dD_bh[b * H + h] = dD_acc;
    free(ck); free(run); free(S); free(Gt);
    return 0;
}

/*
 * Backward of the full scan (see bwd_one), every (b, h) independently.  h0 and dfinal are
 * nullable (zero).  Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int oracle_ssd_scan_bwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                        int64_t dstate, int64_t ngroups, const double *x, const double *dt,
                        const double *A, const double *B, const double *C, const double *D,
                        const double *h0, const double *dy, const double *dfinal, double *dx,
                        double *ddt, double *dB_h, double *dC_h, double *dA_bh, double *dD_bh,
                        double *dinit)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 ||
        ngroups <= 0 || nheads % ngroups != 0)
        return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int64_t i = 0; i < batch * nheads; ++i)
        failed |= bwd_one(i / nheads, i % nheads, seqlen, nheads, headdim, dstate, ngroups, x,
                          dt, A, B, C, D, h0, dy, dfinal, dx, ddt, dB_h, dC_h, dA_bh, dD_bh,
                          dinit) != 0;
    return failed ? -1 : 0;
}

/* Number of OpenMP threads a parallel region of this library will use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
