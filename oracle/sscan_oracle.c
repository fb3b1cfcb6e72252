/*
 * sscan_oracle.c -- fp64 CPU oracle for the selective-scan (S6) forward.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark load this library.  It
 * shares no code, header, table or helper with the CUDA path, and the CUDA
 * path never calls it.
 *
 * What it computes is the plain definition of the forward pass, one
 * sequential loop over time per (batch b, channel d) row, in double
 * precision:
 *
 *   Abar[t,n] = exp(delta[b,t,d] * A[d,n])                      (ZOH of A)
 *   Euler:  bu[t,n] = delta[b,t,d] * B[b,t,n] * u[b,t,d]
 *   ZOH:    bu[t,n] = (exp(delta*A[d,n]) - 1) / A[d,n] * B[b,t,n] * u[b,t,d]
 *   h[n]    = Abar[t,n] * h[n] + bu[t,n]          h before t=0 is h0 (or 0)
 *   y[b,t,d] = sum_n C[b,t,n] * h[n]              (state AFTER token t)
 *   h_final[b,d,n] = h[n] after the last token
 *
 * Optional fused prologue / epilogue (the _ex entry points):
 *
 *   delta  <- delta + delta_bias[d]                 (when a bias is given)
 *   delta  <- softplus(delta) = log(1 + exp(delta)) (when softplus is set)
 *   y[b,t,d] <- y[b,t,d] * silu(z[b,t,d]),  silu(z) = z / (1 + exp(-z))
 *                                                   (when a gate z is given)
 *
 * Sources (page title, section):
 *  - "tm_ssm_selective" (Transformer Math page on selective SSMs), section
 *    "Discretization becomes a per-token operation": per-token ZOH
 *    Abar = exp(Delta_t A) elementwise for diagonal A, the exact ZOH input
 *    term (Delta A)^-1 (exp(Delta A) - I) Delta B, its Euler limit Delta B
 *    ("what implementations actually use"), the diagonal recurrence and the
 *    readout y_t = sum_n C_t[n] x_t[:, n]; shapes from section
 *    "The mechanism: parameters as functions of the input".
 *  - "12. Selective State Space", the selective_scan reference loop: the
 *    tensors u, delta:(batch, seq, d_inner), A:(d_inner, d_state),
 *    B, C:(batch, seq, d_state), the state update followed by the readout
 *    of the updated state at the same step.
 *  - "Mamba & Mamba-2 Architecture", section 1 (shapes B,C:[B,L,N],
 *    Delta:[B,L,D], A:[D,N]) and the numpy listing in section "Code"
 *    (update, then y_t = c_t . h).
 *  - Prologue: "tm_ssm_selective", section "The mechanism: parameters as
 *    functions of the input": Delta_t = softplus(d_bias + Linear_D(u_t)); the
 *    scan is given Linear_D(u_t) as delta and d_bias per channel.
 *  - Epilogue: "Selective State-Space Models (Mamba) and Hardware-Aware
 *    Scans", section 4: the block's second branch gates the SSM output
 *    multiplicatively, as in gated feed-forward layers.
 *
 * Readings where the pages leave a step open:
 *  - y at step t reads the state after token t's update (all listings agree).
 *  - h0 is an optional input (the pages start from zero); NULL means zero.
 *  - ZOH with A[d,n] == 0 takes the limit (exp(Delta*A)-1)/A -> Delta.
 *  - Without the prologue, delta arrives already positive (softplus done by
 *    the projection layer that produces it).
 *  - The gate branch goes through SiLU (the gated feed-forward form the page
 *    compares it to); the pages give no skip term D*u, so none is added.
 *  - softplus is evaluated as max(s, 0) + log1p(exp(-|s|)), the same value
 *    as log(1 + exp(s)) without overflow.
 *
 * Rows are independent (each (b,d) row has its own state), so rows are
 * spread over POSIX threads; the per-row arithmetic is the same sequential
 * loop whatever the thread count, so results do not depend on it.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared -pthread ... -lm
 * (-ffp-contract=off keeps every multiply and add separately rounded).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

/* softplus(s) = log(1 + exp(s)), written so that exp never overflows. */
static double softplus(double s)
{
    return (s > 0.0 ? s : 0.0) + log1p(exp(-fabs(s)));
}

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* One (b,d) row: the sequential recurrence over L tokens.
 *   u[t*su], dl[t*sd]   input and step size of this channel at token t
 *   bias, sp            delta <- delta + bias, then softplus when sp != 0
 *   z[t*sz]             gate of this channel at token t, or NULL
 *   a[n]                the channel's diagonal A row
 *   Bm[t*N+n], Cm[t*N+n] the batch's input / output projections
 *   h0[n]               initial state, or NULL for zero
 *   y[t*sy]             output of this channel at token t
 *   hfin[n]             final state, or NULL
 *   h                   scratch of N doubles */
static void scan_row(int64_t L, int64_t N,
                     const double *u, int64_t su,
                     const double *dl, int64_t sd,
                     const double *a,
                     const double *Bm, const double *Cm,
                     const double *h0, int zoh,
                     double bias, int sp, const double *z, int64_t sz,
                     double *y, int64_t sy, double *hfin, double *h)
{
    for (int64_t n = 0; n < N; ++n)
        h[n] = h0 ? h0[n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
        double delta = dl[t * sd] + bias;
        if (sp)
            delta = softplus(delta);
        const double x = u[t * su];
        const double *Bt = Bm + t * N;
        const double *Ct = Cm + t * N;
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double abar = exp(delta * a[n]);
            double bbar;
            if (zoh)
                bbar = (a[n] != 0.0) ? expm1(delta * a[n]) / a[n] * Bt[n] : delta * Bt[n];
            else
                bbar = delta * Bt[n];
            h[n] = abar * h[n] + bbar * x;
            acc += Ct[n] * h[n];
        }
        y[t * sy] = z ? acc * silu(z[t * sz]) : acc;
    }
    if (hfin)
        for (int64_t n = 0; n < N; ++n)
            hfin[n] = h[n];
}

/* How a row index maps onto the caller's arrays. */
typedef struct {
    int64_t B, L, D, N;
    int rows_mode;            /* 0: all B*D rows of full tensors; 1: an explicit row list */
    const double *u, *dl, *A, *Bm, *Cm, *h0;
    double *y, *hfin;
    const int64_t *row_b;     /* rows_mode 1: batch index of each row */
    int64_t nrows;
    int zoh;
    const double *bias;       /* [D] (rows_mode 1: [R]) or NULL */
    int softplus;
    const double *z;          /* like u, or NULL */
} job_t;

typedef struct {
    const job_t *job;
    int64_t r0, r1;
    int status;
} slice_t;

static void run_row(const job_t *j, int64_t r, double *h)
{
    const int64_t L = j->L, N = j->N, D = j->D;
    if (j->rows_mode == 0) {
        /* full tensors: u,delta,y [B][L][D]; A [D][N]; B,C [B][L][N]; h0,h_final [B][D][N] */
        const int64_t b = r / D, d = r % D;
        scan_row(L, N,
                 j->u + b * L * D + d, D,
                 j->dl + b * L * D + d, D,
                 j->A + d * N,
                 j->Bm + b * L * N, j->Cm + b * L * N,
                 j->h0 ? j->h0 + (b * D + d) * N : NULL, j->zoh,
                 j->bias ? j->bias[d] : 0.0, j->softplus,
                 j->z ? j->z + b * L * D + d : NULL, D,
                 j->y + b * L * D + d, D,
                 j->hfin ? j->hfin + (b * D + d) * N : NULL, h);
    } else {
        /* row list: u,delta,y [R][L]; A,h0,h_final [R][N]; B,C [B][L][N] indexed by row_b[r] */
        const int64_t b = j->row_b[r];
        scan_row(L, N,
                 j->u + r * L, 1,
                 j->dl + r * L, 1,
                 j->A + r * N,
                 j->Bm + b * L * N, j->Cm + b * L * N,
                 j->h0 ? j->h0 + r * N : NULL, j->zoh,
                 j->bias ? j->bias[r] : 0.0, j->softplus,
                 j->z ? j->z + r * L : NULL, 1,
                 j->y + r * L, 1,
                 j->hfin ? j->hfin + r * N : NULL, h);
    }
}

static void *run_slice(void *arg)
{
    slice_t *s = (slice_t *)arg;
    double *h = (double *)malloc(sizeof(double) * (size_t)(s->job->N > 0 ? s->job->N : 1));
    if (!h) { s->status = 2; return NULL; }
    for (int64_t r = s->r0; r < s->r1; ++r)
        run_row(s->job, r, h);
    free(h);
    s->status = 0;
    return NULL;
}

static int run_job(const job_t *j, int64_t nrows, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    if ((int64_t)nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);
    slice_t *sl = (slice_t *)calloc((size_t)nthreads, sizeof(slice_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!sl || !th) { free(sl); free(th); return 2; }
    int rc = 0, started = 0;
    for (int i = 0; i < nthreads; ++i) {
        sl[i].job = j;
        sl[i].r0 = nrows * i / nthreads;
        sl[i].r1 = nrows * (i + 1) / nthreads;
        sl[i].status = 1;
        if (i == nthreads - 1) break;          /* the calling thread takes the last slice */
        if (pthread_create(&th[i], NULL, run_slice, &sl[i]) != 0) { rc = 3; break; }
        ++started;
    }
    if (rc == 0) run_slice(&sl[nthreads - 1]);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    for (int i = 0; rc == 0 && i < nthreads; ++i)
        if (sl[i].status != 0) rc = sl[i].status;
    free(sl);
    free(th);
    return rc;
}

/* Full forward over contiguous row-major tensors, with the optional
 * prologue / epilogue.
 *   u, delta, y : [B][L][D]     A : [D][N]     Bm, Cm : [B][L][N]
 *   h0, h_final : [B][D][N]     (either may be NULL)
 *   delta_bias  : [D] or NULL   softplus: 0 or 1     z : [B][L][D] or NULL
 * Returns 0 on success, 1 for bad sizes or pointers, 2/3 on allocation or
 * thread-creation failure. */
int sscan_oracle_forward_ex(int64_t B, int64_t L, int64_t D, int64_t N,
                            const double *u, const double *delta, const double *A,
                            const double *Bm, const double *Cm, const double *h0,
                            int zoh, const double *delta_bias, int softplus, const double *z,
                            double *y, double *h_final, int nthreads)
{
    if (B < 0 || L < 0 || D < 0 || N < 0) return 1;
    if (B == 0 || D == 0) return 0;
    if (N > 0 && (!A || ((L > 0) && (!Bm || !Cm)))) return 1;
    if (L > 0 && (!u || !delta || !y)) return 1;
    job_t j = {B, L, D, N, 0, u, delta, A, Bm, Cm, h0, y, h_final, NULL, B * D, zoh,
               delta_bias, softplus != 0, z};
    return run_job(&j, B * D, nthreads);
}

/* The plain forward: no bias, no softplus, no gate. */
int sscan_oracle_forward(int64_t B, int64_t L, int64_t D, int64_t N,
                         const double *u, const double *delta, const double *A,
                         const double *Bm, const double *Cm, const double *h0,
                         int zoh, double *y, double *h_final, int nthreads)
{
    return sscan_oracle_forward_ex(B, L, D, N, u, delta, A, Bm, Cm, h0, zoh, NULL, 0, NULL,
                                   y, h_final, nthreads);
}

/* The same recurrence on an explicit list of R rows (for sampling large
 * problems row by row; rows are independent, so a sampled row is exact).
 *   row_b      : [R]     batch index of each row (indexes Bm/Cm)
 *   u_rows, delta_rows, y_rows : [R][L]   the row's channel, gathered
 *   A_rows, h0_rows, hfin_rows : [R][N]   (h0_rows / hfin_rows may be NULL)
 *   Bm, Cm     : [Bn][L][N]
 *   bias_rows  : [R] delta bias of each row's channel, or NULL
 *   z_rows     : [R][L] gate of each row, or NULL */
int sscan_oracle_rows_ex(int64_t R, int64_t L, int64_t N, int64_t Bn,
                         const int64_t *row_b,
                         const double *u_rows, const double *delta_rows, const double *A_rows,
                         const double *Bm, const double *Cm, const double *h0_rows,
                         int zoh, const double *bias_rows, int softplus, const double *z_rows,
                         double *y_rows, double *hfin_rows, int nthreads)
{
    if (R < 0 || L < 0 || N < 0 || Bn < 0) return 1;
    if (R == 0) return 0;
    if (!row_b) return 1;
    for (int64_t r = 0; r < R; ++r)
        if (row_b[r] < 0 || row_b[r] >= Bn) return 1;
    job_t j = {Bn, L, 0, N, 1, u_rows, delta_rows, A_rows, Bm, Cm, h0_rows,
               y_rows, hfin_rows, row_b, R, zoh, bias_rows, softplus != 0, z_rows};
    return run_job(&j, R, nthreads);
}

/* Row list without prologue / epilogue. */
int sscan_oracle_rows(int64_t R, int64_t L, int64_t N, int64_t Bn,
                      const int64_t *row_b,
                      const double *u_rows, const double *delta_rows, const double *A_rows,
                      const double *Bm, const double *Cm, const double *h0_rows,
                      int zoh, double *y_rows, double *hfin_rows, int nthreads)
{
    return sscan_oracle_rows_ex(R, L, N, Bn, row_b, u_rows, delta_rows, A_rows, Bm, Cm, h0_rows,
                                zoh, NULL, 0, NULL, y_rows, hfin_rows, nthreads);
}

/* ------------------------------------------------------------------ backward
 *
 * Gradients of a scalar loss through the forward above (plain forward, no
 * prologue / epilogue), given dy = dLoss/dy [B][L][D] and optionally
 * dh_final = dLoss/dh_final [B][D][N].  Written out from the recurrence by the
 * chain rule, in the order the forward computes it ("Selective State-Space
 * Models (Mamba) and Hardware-Aware Scans", section 3: the backward pass
 * recomputes the states instead of storing them; here every state of a row is
 * kept, the plain way):
 *
 *   a_t = exp(delta_t A_n),  beta_t = delta_t B_t[n]        (Euler)
 *                            beta_t = (a_t - 1)/A_n B_t[n]   (ZOH; delta_t B_t[n] at A_n = 0)
 *   h_t = a_t h_{t-1} + beta_t u_t,   y_t = sum_n C_t[n] h_t
 *
 *   g_t = dLoss/dh_t = C_t[n] dy_t + a_{t+1} g_{t+1},  g_{L-1} = C dy + dh_final
 *   du_t      = sum_n g_t beta_t
 *   ddelta_t  = sum_n g_t (h_{t-1} A_n a_t + u_t dbeta/ddelta)
 *               dbeta/ddelta = B_t[n] (Euler), a_t B_t[n] (ZOH)
 *   dA[d,n]   = sum_{b,t} g_t (h_{t-1} delta_t a_t + u_t dbeta/dA)
 *               dbeta/dA = 0 (Euler), B_t[n] (delta_t a_t A_n - (a_t - 1)) / A_n^2
 *               (ZOH; delta_t^2 B_t[n] / 2 at A_n = 0)
 *   dB_t[n]   = sum_d g_t u_t dbeta/dB,  dbeta/dB = delta_t (Euler), (a_t - 1)/A_n (ZOH)
 *   dC_t[n]   = sum_d dy_t h_t
 *   dh0       = a_0 g_0
 *
 * Outputs are overwritten (not accumulated into).  One thread per batch row b
 * (dB, dC of row b are its own); each thread sums its dA into a private
 * buffer that is added up in b order at the end, so the result does not
 * depend on the thread count. */

typedef struct {
    int64_t B, L, D, N;
    const double *u, *dl, *A, *Bm, *Cm, *h0, *dy, *dhf;
    int zoh;
    double *du, *ddl, *dA_part, *dB, *dC, *dh0;
    int64_t b0, b1;
    int status;
} bwd_t;

static void bwd_row(const bwd_t *j, int64_t b, int64_t d, double *hs, double *g, double *dA)
{
    const int64_t L = j->L, D = j->D, N = j->N;
    const double *u = j->u + b * L * D + d, *dl = j->dl + b * L * D + d, *dy = j->dy + b * L * D + d;
    const double *a_row = j->A + d * N;
    const double *Bm = j->Bm + b * L * N, *Cm = j->Cm + b * L * N;
    /* forward: hs[(t+1)*N + n] = h_t, hs[n] = h_{-1} = h0 */
    for (int64_t n = 0; n < N; ++n)
        hs[n] = j->h0 ? j->h0[(b * D + d) * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t)
        for (int64_t n = 0; n < N; ++n) {
            const double delta = dl[t * D], an = a_row[n];
            const double abar = exp(delta * an);
            const double beta = j->zoh ? (an != 0.0 ? expm1(delta * an) / an * Bm[t * N + n] : delta * Bm[t * N + n])
                                       : delta * Bm[t * N + n];
            hs[(t + 1) * N + n] = abar * hs[t * N + n] + beta * u[t * D];
        }
    /* backward */
    for (int64_t n = 0; n < N; ++n)
        g[n] = j->dhf ? j->dhf[(b * D + d) * N + n] : 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
        const double delta = dl[t * D], x = u[t * D], dyt = dy[t * D];
        double du = 0.0, ddl = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double an = a_row[n], Bn = Bm[t * N + n], Cn = Cm[t * N + n];
            const double abar = exp(delta * an);
            const double hprev = hs[t * N + n], ht = hs[(t + 1) * N + n];
            g[n] += Cn * dyt;                                   /* g_t = C dy + (carried a_{t+1} g_{t+1}) */
            j->dC[(b * L + t) * N + n] += dyt * ht;
            double beta, dbeta_ddl, dbeta_dA, dbeta_dB;
            if (!j->zoh) {
                beta = delta * Bn; dbeta_ddl = Bn; dbeta_dA = 0.0; dbeta_dB = delta;
            } else if (an != 0.0) {
                const double em1 = expm1(delta * an);
                beta = em1 / an * Bn; dbeta_ddl = abar * Bn;
                dbeta_dA = Bn * (delta * abar * an - em1) / (an * an); dbeta_dB = em1 / an;
            } else {
                beta = delta * Bn; dbeta_ddl = Bn; dbeta_dA = 0.5 * delta * delta * Bn; dbeta_dB = delta;
            }
            du += g[n] * beta;
            ddl += g[n] * (hprev * an * abar + x * dbeta_ddl);
            dA[d * N + n] += g[n] * (hprev * delta * abar + x * dbeta_dA);
            j->dB[(b * L + t) * N + n] += g[n] * x * dbeta_dB;
            g[n] *= abar;                                       /* now a_t g_t: carried to t-1 */
        }
        j->du[(b * L + t) * D + d] = du;
        j->ddl[(b * L + t) * D + d] = ddl;
    }
    if (j->dh0)
        for (int64_t n = 0; n < N; ++n)
            j->dh0[(b * D + d) * N + n] = g[n];               /* a_0 g_0 */
}

static void *bwd_slice(void *arg)
{
    bwd_t *j = (bwd_t *)arg;
    const int64_t L = j->L, N = j->N;
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N + 1));
    double *g = (double *)malloc(sizeof(double) * (size_t)(N + 1));
    if (!hs || !g) { free(hs); free(g); j->status = 2; return NULL; }
    for (int64_t b = j->b0; b < j->b1; ++b) {
        for (int64_t i = 0; i < L * N; ++i) { j->dB[b * L * N + i] = 0.0; j->dC[b * L * N + i] = 0.0; }
        for (int64_t d = 0; d < j->D; ++d)
            bwd_row(j, b, d, hs, g, j->dA_part + b * j->D * N);
    }
    free(hs);
    free(g);
    j->status = 0;
    return NULL;
}

/* Backward over full tensors.  Inputs as for sscan_oracle_forward plus
 *   dy       : [B][L][D]      dh_final : [B][D][N] or NULL (zero)
 * Outputs (all overwritten):
 *   du, ddelta : [B][L][D]    dA : [D][N]    dB, dC : [B][L][N]    dh0 : [B][D][N] or NULL
 * Returns 0 on success, 1 for bad arguments, 2/3 on allocation or thread failure. */
int sscan_oracle_backward(int64_t B, int64_t L, int64_t D, int64_t N,
                          const double *u, const double *delta, const double *A,
                          const double *Bm, const double *Cm, const double *h0, int zoh,
                          const double *dy, const double *dh_final,
                          double *du, double *ddelta, double *dA, double *dB, double *dC,
                          double *dh0, int nthreads)
{
    if (B < 1 || L < 0 || D < 1 || N < 1) return 1;
    if (!A || !dA || (L > 0 && (!u || !delta || !Bm || !Cm || !dy || !du || !ddelta || !dB || !dC))) return 1;
    double *part = (double *)calloc((size_t)(B * D * N), sizeof(double));
    if (!part) return 2;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B) nthreads = (int)B;
    bwd_t *jobs = (bwd_t *)calloc((size_t)nthreads, sizeof(bwd_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(part); free(jobs); free(th); return 2; }
    int rc = 0, started = 0;
    for (int i = 0; i < nthreads; ++i) {
        bwd_t j = {B, L, D, N, u, delta, A, Bm, Cm, h0, dy, dh_final, zoh,
                   du, ddelta, part, dB, dC, dh0, B * i / nthreads, B * (i + 1) / nthreads, 1};
        jobs[i] = j;
        if (i == nthreads - 1) break;
        if (pthread_create(&th[i], NULL, bwd_slice, &jobs[i]) != 0) { rc = 3; break; }
        ++started;
    }
    if (rc == 0) bwd_slice(&jobs[nthreads - 1]);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    for (int i = 0; rc == 0 && i < nthreads; ++i)
        if (jobs[i].status != 0) rc = jobs[i].status;
    if (rc == 0)
        for (int64_t k = 0; k < D * N; ++k) {
            double s = 0.0;
            for (int64_t b = 0; b < B; ++b) s += part[b * D * N + k];
            dA[k] = s;
        }
    free(part);
    free(jobs);
    free(th);
    return rc;
}
