/*
 * oracle.c -- the f64 CPU oracle of the selective state-space scans.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, sequential, obviously
 * correct definition that the CUDA library is checked against.  Only the
 * tests, the package's smoke() check and the benchmark's CPU-baseline leg
 * load it.  It shares no code, header, table or helper with the CUDA path.
 *
 * Everything is computed in double precision with plain loops in the order
 * the recurrences are written.  Inputs arrive as doubles that already hold
 * the io-rounded values.  Independent rows (one (batch, channel) sequence for
 * Mamba-1, one (batch, head) sequence for Mamba-3) run on host threads;
 * reductions that cross rows are kept per thread and added up in thread
 * order afterwards, which changes nothing but the last bits of an f64 sum.
 *
 * What is computed, and where it comes from:
 *
 *   Mamba-1 selective scan ("Selective SSM", state-spaces/mamba README, the
 *   selective SSM layer of the Mamba paper's Section 3 / Algorithm 2; named as
 *   "Mamba SSM (Gu and Dao, 2023)" in the mamba-rs 0.7.0 README, "Features"):
 *       delta_t = softplus(delta_raw_t + bias)        (or delta_raw_t + bias)
 *       h_t[n]  = exp(delta_t * A[n]) * h_{t-1}[n] + delta_t * B_t[n] * x_t
 *       y_t     = sum_n C_t[n] h_t[n] + D * x_t
 *       out_t   = y_t * silu(z_t)
 *   and its backward pass through the recurrent state (backpropagation
 *   through time over the SSM state, mamba-rs 0.7.0 README, "Features").
 *
 *   Mamba-3 SISO scan (mamba-rs 0.7.0 README, "Features"; backward stages
 *   B2 output gating, B3 BPTT and B4 RoPE of Mamba3Scratch in mamba-rs 0.4.2
 *   src/mamba3_siso/cpu/scratch.rs):
 *       phi_t[k] = sum_{s<=t} theta_s[k]                 (cumulative angles)
 *       Bt_t = R(phi_t) B_t,  Ct_t = R(phi_t) C_t        (pairs (2k, 2k+1))
 *       K_t  = x_t (outer) Bt_t                          (headdim x d_state)
 *       S_t  = alpha_t S_{t-1} + beta_t K_{t-1} + gamma_t K_t,   K_{-1} = 0
 *       y_t  = S_t Ct_t + D x_t,   out_t = y_t * silu(z_t)
 *   The per-head d_alpha/d_beta/d_gamma [T*nheads] and d_k_carry buffers of
 *   stage B3 fix this three-term (trapezoidal) form; d_angle_cumsum and
 *   cum_angles [T*nheads*n_angles] of stage B4 fix per-head cumulative angles.
 *
 *   Single-token state update: one step of the Mamba-1 recurrence applied to
 *   a stored state (mamba_step / GpuMambaBackbone::step, mamba-rs 0.7.0
 *   README, "Quick start"), and one step of the Mamba-3 SISO recurrence
 *   applied to a stored state with its last key and cumulative angles
 *   (mamba3_step on a Mamba3State, the same README, "Quick start (CPU)").
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_MAX_N 256

/* ------------------------------------------------------------------ */
/* scalar functions                                                    */
/* ------------------------------------------------------------------ */
static double softplus(double v) { return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v))); }
static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }
static double silu(double v) { return v * sigmoid(v); }
/* d/dv [v * sigmoid(v)] */
static double dsilu(double v) {
    double s = sigmoid(v);
    return s * (1.0 + v * (1.0 - s));
}

/* ------------------------------------------------------------------ */
/* a tiny parallel-for over independent rows                           */
/* ------------------------------------------------------------------ */
typedef void (*row_fn)(void *ctx, int64_t row, int tid);

typedef struct {
    row_fn fn;
    void *ctx;
    int64_t nrows;
    int nthreads;
    int tid;
} worker_arg;

static void *worker_main(void *p) {
    worker_arg *w = (worker_arg *)p;
    for (int64_t r = w->tid; r < w->nrows; r += w->nthreads) w->fn(w->ctx, r, w->tid);
    return NULL;
}

static int resolve_threads(int nthreads, int64_t nrows) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nrows < nthreads) nthreads = (int)(nrows > 0 ? nrows : 1);
    return nthreads;
}

static void parallel_rows(int64_t nrows, int nthreads, row_fn fn, void *ctx) {
    worker_arg *args = (worker_arg *)calloc((size_t)nthreads, sizeof(worker_arg));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int i = 0; i < nthreads; ++i) {
        args[i].fn = fn;
        args[i].ctx = ctx;
        args[i].nrows = nrows;
        args[i].nthreads = nthreads;
        args[i].tid = i;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, worker_main, &args[i]);
    worker_main(&args[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(args);
    free(th);
}

int oracle_default_threads(void) { return resolve_threads(0, 1 << 30); }

/* ------------------------------------------------------------------ */
/* Mamba-1: forward                                                    */
/* ------------------------------------------------------------------ */
typedef struct {
    int64_t Bsz, D, N, L, G;
    int softplus_on;
    const double *u, *delta, *A, *Bm, *Cm, *Dp, *bias, *z, *h0;
    double *out, *final_state, *y_pre;
} m1_fwd_ctx;

/* index helpers: u/delta/z/out are [B, D, L]; B/C are [B, G, N, L] */
#define IDX_BDL(b, c, t) (((b) * D + (c)) * L + (t))
#define IDX_BGNL(b, g, n, t) ((((b) * G + (g)) * N + (n)) * L + (t))

static void m1_fwd_row(void *vctx, int64_t row, int tid) {
    (void)tid;
    const m1_fwd_ctx *c = (const m1_fwd_ctx *)vctx;
    const int64_t D = c->D, N = c->N, L = c->L, G = c->G;
    const int64_t b = row / D, ch = row % D, g = ch / (D / G);
    double h[ORACLE_MAX_N];
    for (int64_t n = 0; n < N; ++n) h[n] = c->h0 ? c->h0[(b * D + ch) * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
        double v = c->delta[IDX_BDL(b, ch, t)] + (c->bias ? c->bias[ch] : 0.0);
        double dt = c->softplus_on ? softplus(v) : v;
        double x = c->u[IDX_BDL(b, ch, t)];
        double y = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double a = exp(dt * c->A[ch * N + n]);
            h[n] = a * h[n] + dt * c->Bm[IDX_BGNL(b, g, n, t)] * x;
            y += c->Cm[IDX_BGNL(b, g, n, t)] * h[n];
        }
        if (c->Dp) y += c->Dp[ch] * x;
        if (c->y_pre) c->y_pre[IDX_BDL(b, ch, t)] = y;
        c->out[IDX_BDL(b, ch, t)] = c->z ? y * silu(c->z[IDX_BDL(b, ch, t)]) : y;
    }
    if (c->final_state)
        for (int64_t n = 0; n < N; ++n) c->final_state[(b * D + ch) * N + n] = h[n];
}

int oracle_m1_fwd(int64_t Bsz, int64_t D, int64_t N, int64_t L, int64_t G, int softplus_on,
                  const double *u, const double *delta, const double *A, const double *Bm,
                  const double *Cm, const double *Dp, const double *bias, const double *z,
                  const double *h0, double *out, double *final_state, double *y_pre,
                  int nthreads) {
    if (N > ORACLE_MAX_N || G < 1 || D % G) return -1;
    m1_fwd_ctx c = {Bsz, D, N, L, G, softplus_on, u, delta, A, Bm, Cm, Dp, bias, z, h0,
                    out, final_state, y_pre};
    int64_t rows = Bsz * D;
    parallel_rows(rows, resolve_threads(nthreads, rows), m1_fwd_row, &c);
    return 0;
}

/*
 * The same forward, with the time recurrence evaluated as a Hillis-Steele
 * inclusive scan of (a_t, b_t) pairs under the combine
 *     (a, b) o (a', b') = (a * a', a' * b + b')
 * instead of the step-by-step loop.  The recurrence h_t = a_t h_{t-1} + b_t is
 * associative under this combine, so the two orders agree up to rounding;
 * the tests use this to pin the combine operator and its carry semantics,
 * which the parallel GPU scan relies on ("sequential and parallel scan
 * regimes", mamba-rs docs/gemm-modes.md, "What is guaranteed").
 */
static void m1_fwd_tree_row(void *vctx, int64_t row, int tid) {
    (void)tid;
    const m1_fwd_ctx *c = (const m1_fwd_ctx *)vctx;
    const int64_t D = c->D, N = c->N, L = c->L, G = c->G;
    const int64_t b = row / D, ch = row % D, g = ch / (D / G);
    double *pa = (double *)malloc(sizeof(double) * (size_t)L);
    double *pb = (double *)malloc(sizeof(double) * (size_t)L);
    double *na = (double *)malloc(sizeof(double) * (size_t)L);
    double *nb = (double *)malloc(sizeof(double) * (size_t)L);
    double *y = (double *)calloc((size_t)L, sizeof(double));
    double *dts = (double *)malloc(sizeof(double) * (size_t)L);
    for (int64_t t = 0; t < L; ++t) {
        double v = c->delta[IDX_BDL(b, ch, t)] + (c->bias ? c->bias[ch] : 0.0);
        dts[t] = c->softplus_on ? softplus(v) : v;
    }
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t t = 0; t < L; ++t) {
            pa[t] = exp(dts[t] * c->A[ch * N + n]);
            pb[t] = dts[t] * c->Bm[IDX_BGNL(b, g, n, t)] * c->u[IDX_BDL(b, ch, t)];
        }
        for (int64_t off = 1; off < L; off *= 2) {
            for (int64_t t = 0; t < L; ++t) {
                if (t >= off) {
                    /* element t-off precedes element t */
                    na[t] = pa[t - off] * pa[t];
                    nb[t] = pa[t] * pb[t - off] + pb[t];
                } else {
                    na[t] = pa[t];
                    nb[t] = pb[t];
                }
            }
            memcpy(pa, na, sizeof(double) * (size_t)L);
            memcpy(pb, nb, sizeof(double) * (size_t)L);
        }
        double hinit = c->h0 ? c->h0[(b * D + ch) * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double h = pa[t] * hinit + pb[t];
            y[t] += c->Cm[IDX_BGNL(b, g, n, t)] * h;
            if (t == L - 1 && c->final_state) c->final_state[(b * D + ch) * N + n] = h;
        }
    }
    for (int64_t t = 0; t < L; ++t) {
        double x = c->u[IDX_BDL(b, ch, t)];
        double yy = y[t] + (c->Dp ? c->Dp[ch] * x : 0.0);
        c->out[IDX_BDL(b, ch, t)] = c->z ? yy * silu(c->z[IDX_BDL(b, ch, t)]) : yy;
    }
    free(pa); free(pb); free(na); free(nb); free(y); free(dts);
}

int oracle_m1_fwd_tree(int64_t Bsz, int64_t D, int64_t N, int64_t L, int64_t G, int softplus_on,
                       const double *u, const double *delta, const double *A, const double *Bm,
                       const double *Cm, const double *Dp, const double *bias, const double *z,
                       const double *h0, double *out, double *final_state, int nthreads) {
    if (N > ORACLE_MAX_N || G < 1 || D % G) return -1;
    m1_fwd_ctx c = {Bsz, D, N, L, G, softplus_on, u, delta, A, Bm, Cm, Dp, bias, z, h0,
                    out, final_state, NULL};
    int64_t rows = Bsz * D;
    parallel_rows(rows, resolve_threads(nthreads, rows), m1_fwd_tree_row, &c);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Mamba-1: backward through the recurrent state                       */
/* ------------------------------------------------------------------ */
/*
 * With g_t = dout_t * silu(z_t) the gradient of the loss w.r.t. y_t, the
 * adjoint of the state obeys the reverse recurrence
 *     lambda_t[n] = g_t C_t[n] + a_{t+1}[n] lambda_{t+1}[n],   lambda after the
 *                                                              last step = 0
 * (the final state is an output, not differentiated), and
 *     dC_t[n]  += g_t h_t[n]                 (summed over the group's channels)
 *     dB_t[n]  += lambda_t[n] delta_t x_t    (summed over the group's channels)
 *     dx_t      = g_t D + delta_t sum_n lambda_t[n] B_t[n]
 *     ddelta_t  = sum_n lambda_t[n] (A[n] a_t[n] h_{t-1}[n] + B_t[n] x_t)
 *     dA[n]    += lambda_t[n] delta_t a_t[n] h_{t-1}[n]
 *     dD       += g_t x_t
 *     dz_t      = dout_t y_t silu'(z_t)
 *     ddelta_raw_t = ddelta_t * sigmoid(delta_raw_t + bias)   (softplus on)
 *     dbias    += ddelta_raw_t
 *     dh0[n]    = a_0[n] lambda_0[n]
 */
typedef struct {
    int64_t Bsz, D, N, L, G;
    int softplus_on;
    const double *u, *delta, *A, *Bm, *Cm, *Dp, *bias, *z, *h0, *dout;
    double *du, *ddelta, *dz, *dh0;
    /* per-thread partial sums for the reductions that cross rows */
    double **dA_part, **dB_part, **dC_part, **dD_part, **dbias_part;
} m1_bwd_ctx;

static void m1_bwd_row(void *vctx, int64_t row, int tid) {
    const m1_bwd_ctx *c = (const m1_bwd_ctx *)vctx;
    const int64_t D = c->D, N = c->N, L = c->L, G = c->G;
    const int64_t b = row / D, ch = row % D, g = ch / (D / G);
    double *hs = (double *)malloc(sizeof(double) * (size_t)(L * N));
    double *as = (double *)malloc(sizeof(double) * (size_t)(L * N));
    double *dts = (double *)malloc(sizeof(double) * (size_t)L);
    double *ys = (double *)malloc(sizeof(double) * (size_t)L);
    double h[ORACLE_MAX_N], mu[ORACLE_MAX_N], hinit[ORACLE_MAX_N];
    double *dA = c->dA_part[tid], *dB = c->dB_part[tid], *dC = c->dC_part[tid];
    double *dD = c->dD_part[tid], *dbias = c->dbias_part[tid];

    /* forward pass, keeping every state */
    for (int64_t n = 0; n < N; ++n) {
        hinit[n] = c->h0 ? c->h0[(b * D + ch) * N + n] : 0.0;
        h[n] = hinit[n];
    }
    for (int64_t t = 0; t < L; ++t) {
        double v = c->delta[IDX_BDL(b, ch, t)] + (c->bias ? c->bias[ch] : 0.0);
        double dt = c->softplus_on ? softplus(v) : v;
        double x = c->u[IDX_BDL(b, ch, t)];
        double y = 0.0;
        dts[t] = dt;
        for (int64_t n = 0; n < N; ++n) {
            double a = exp(dt * c->A[ch * N + n]);
            h[n] = a * h[n] + dt * c->Bm[IDX_BGNL(b, g, n, t)] * x;
            as[t * N + n] = a;
            hs[t * N + n] = h[n];
            y += c->Cm[IDX_BGNL(b, g, n, t)] * h[n];
        }
        if (c->Dp) y += c->Dp[ch] * x;
        ys[t] = y;
    }

    /* reverse pass */
    for (int64_t n = 0; n < N; ++n) mu[n] = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
        const double x = c->u[IDX_BDL(b, ch, t)];
        const double dt = dts[t];
        const double dout = c->dout[IDX_BDL(b, ch, t)];
        double gt = dout;
        if (c->z) {
            double zt = c->z[IDX_BDL(b, ch, t)];
            gt = dout * silu(zt);
            if (c->dz) c->dz[IDX_BDL(b, ch, t)] = dout * ys[t] * dsilu(zt);
        }
        dD[ch] += gt * x;
        double sumB = 0.0, ddt = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double Bv = c->Bm[IDX_BGNL(b, g, n, t)];
            const double Cv = c->Cm[IDX_BGNL(b, g, n, t)];
            const double a = as[t * N + n];
            const double hprev = t > 0 ? hs[(t - 1) * N + n] : hinit[n];
            const double lam = gt * Cv + mu[n];
            dC[IDX_BGNL(b, g, n, t)] += gt * hs[t * N + n];
            dB[IDX_BGNL(b, g, n, t)] += lam * dt * x;
            sumB += lam * Bv;
            ddt += lam * (c->A[ch * N + n] * a * hprev + Bv * x);
            dA[ch * N + n] += lam * dt * a * hprev;
            mu[n] = a * lam;
        }
        c->du[IDX_BDL(b, ch, t)] = gt * (c->Dp ? c->Dp[ch] : 0.0) + dt * sumB;
        double v = c->delta[IDX_BDL(b, ch, t)] + (c->bias ? c->bias[ch] : 0.0);
        double draw = c->softplus_on ? ddt * sigmoid(v) : ddt;
        c->ddelta[IDX_BDL(b, ch, t)] = draw;
        dbias[ch] += draw;
    }
    if (c->dh0)
        for (int64_t n = 0; n < N; ++n) c->dh0[(b * D + ch) * N + n] = mu[n];
    free(hs); free(as); free(dts); free(ys);
}

static double **alloc_parts(int nthreads, int64_t count) {
    double **p = (double **)calloc((size_t)nthreads, sizeof(double *));
    for (int i = 0; i < nthreads; ++i) p[i] = (double *)calloc((size_t)count, sizeof(double));
    return p;
}

/* out[i] = sum over threads, in thread order */
static void fold_parts(double **p, int nthreads, int64_t count, double *out) {
    for (int64_t i = 0; i < count; ++i) {
        double s = 0.0;
        for (int k = 0; k < nthreads; ++k) s += p[k][i];
        if (out) out[i] = s;
    }
    for (int k = 0; k < nthreads; ++k) free(p[k]);
    free(p);
}

int oracle_m1_bwd(int64_t Bsz, int64_t D, int64_t N, int64_t L, int64_t G, int softplus_on,
                  const double *u, const double *delta, const double *A, const double *Bm,
                  const double *Cm, const double *Dp, const double *bias, const double *z,
                  const double *h0, const double *dout, double *du, double *ddelta, double *dA,
                  double *dB, double *dC, double *dD, double *dbias, double *dz, double *dh0,
                  int nthreads) {
    if (N > ORACLE_MAX_N || G < 1 || D % G) return -1;
    int64_t rows = Bsz * D;
    int nt = resolve_threads(nthreads, rows);
    m1_bwd_ctx c = {Bsz, D, N, L, G, softplus_on, u, delta, A, Bm, Cm, Dp, bias, z, h0, dout,
                    du, ddelta, dz, dh0, NULL, NULL, NULL, NULL, NULL};
    c.dA_part = alloc_parts(nt, D * N);
    c.dB_part = alloc_parts(nt, Bsz * G * N * L);
    c.dC_part = alloc_parts(nt, Bsz * G * N * L);
    c.dD_part = alloc_parts(nt, D);
    c.dbias_part = alloc_parts(nt, D);
    parallel_rows(rows, nt, m1_bwd_row, &c);
    fold_parts(c.dA_part, nt, D * N, dA);
    fold_parts(c.dB_part, nt, Bsz * G * N * L, dB);
    fold_parts(c.dC_part, nt, Bsz * G * N * L, dC);
    fold_parts(c.dD_part, nt, D, dD);
    fold_parts(c.dbias_part, nt, D, dbias);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Single-token state update                                           */
/* ------------------------------------------------------------------ */
/*
 * One step of the Mamba-1 recurrence on a stored state, written out on its
 * own (not by calling the scan) so that the tests can check the two against
 * each other.  state [B, D, N] is updated in place; x, delta, z, out are
 * [B, D]; B, C are [B, G, N].
 */
int oracle_ssm_state_update(int64_t Bsz, int64_t D, int64_t N, int64_t G, int softplus_on,
                            double *state, const double *x, const double *delta,
                            const double *A, const double *Bm, const double *Cm,
                            const double *Dp, const double *bias, const double *z,
                            double *out) {
    if (N > ORACLE_MAX_N || G < 1 || D % G) return -1;
    for (int64_t b = 0; b < Bsz; ++b) {
        for (int64_t ch = 0; ch < D; ++ch) {
            const int64_t g = ch / (D / G);
            const int64_t i = b * D + ch;
            double v = delta[i] + (bias ? bias[ch] : 0.0);
            double dt = softplus_on ? softplus(v) : v;
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double *s = &state[i * N + n];
                *s = exp(dt * A[ch * N + n]) * *s + dt * Bm[(b * G + g) * N + n] * x[i];
                y += Cm[(b * G + g) * N + n] * *s;
            }
            if (Dp) y += Dp[ch] * x[i];
            out[i] = z ? y * silu(z[i]) : y;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Mamba-3 SISO                                                        */
/* ------------------------------------------------------------------ */
/* layouts: x, z, out [B, L, H, P]; B, C [B, L, G, N]; alpha, beta, gamma
 * [B, L, H]; theta [B, L, H, K]; D [H]; h0, final state [B, H, P, N]       */
#define IDX_X(b, t, h, p) ((((b) * L + (t)) * H + (h)) * P + (p))
#define IDX_BC(b, t, g, n) ((((b) * L + (t)) * G + (g)) * N + (n))
#define IDX_T(b, t, h) (((b) * L + (t)) * H + (h))
#define IDX_TH(b, t, h, k) ((((b) * L + (t)) * H + (h)) * K + (k))

/* out = R(phi) v : pairs (2k, 2k+1) for k < K rotated counter-clockwise by
 * phi[k]; components from 2K on pass through unrotated. */
static void rope_apply(const double *v, const double *phi, int64_t N, int64_t K, double *out) {
    for (int64_t k = 0; k < K; ++k) {
        double cs = cos(phi[k]), sn = sin(phi[k]);
        out[2 * k] = cs * v[2 * k] - sn * v[2 * k + 1];
        out[2 * k + 1] = sn * v[2 * k] + cs * v[2 * k + 1];
    }
    for (int64_t n = 2 * K; n < N; ++n) out[n] = v[n];
}

typedef struct {
    int64_t Bsz, L, H, P, N, G, K;
    const double *x, *z, *Bm, *Cm, *alpha, *beta, *gamma, *theta, *Dp, *h0, *dout;
    double *out, *final_state;
    /* backward outputs */
    double *dx, *dz, *dalpha, *dbeta, *dgamma, *dtheta, *dh0;
    double **dB_part, **dC_part, **dD_part;
} m3_ctx;

/* One (batch, head) row, forward.  If Ss is non-NULL every state S_t
 * (P x N) is stored there, and Bts/Cts/phis receive the rotated B, C and the
 * cumulative angles of every step. */
static void m3_forward_row(const m3_ctx *c, int64_t b, int64_t h, double *Ss, double *Bts,
                           double *Cts, double *phis, double *ys) {
    const int64_t L = c->L, H = c->H, P = c->P, N = c->N, G = c->G, K = c->K;
    const int64_t g = h / (H / G);
    double *S = (double *)malloc(sizeof(double) * (size_t)(P * N));
    double *Kp = (double *)calloc((size_t)(P * N), sizeof(double));
    double phi[ORACLE_MAX_N], Bt[ORACLE_MAX_N], Ct[ORACLE_MAX_N];
    for (int64_t k = 0; k < K; ++k) phi[k] = 0.0;
    for (int64_t i = 0; i < P * N; ++i) S[i] = c->h0 ? c->h0[(b * H + h) * P * N + i] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
        for (int64_t k = 0; k < K; ++k) phi[k] += c->theta[IDX_TH(b, t, h, k)];
        rope_apply(&c->Bm[IDX_BC(b, t, g, 0)], phi, N, K, Bt);
        rope_apply(&c->Cm[IDX_BC(b, t, g, 0)], phi, N, K, Ct);
        const double al = c->alpha[IDX_T(b, t, h)];
        const double be = c->beta[IDX_T(b, t, h)];
        const double ga = c->gamma[IDX_T(b, t, h)];
        for (int64_t p = 0; p < P; ++p) {
            const double xp = c->x[IDX_X(b, t, h, p)];
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double knew = xp * Bt[n];
                S[p * N + n] = al * S[p * N + n] + be * Kp[p * N + n] + ga * knew;
                Kp[p * N + n] = knew;
                y += Ct[n] * S[p * N + n];
            }
            if (c->Dp) y += c->Dp[h] * xp;
            if (ys) ys[t * P + p] = y;
            if (c->out)
                c->out[IDX_X(b, t, h, p)] = c->z ? y * silu(c->z[IDX_X(b, t, h, p)]) : y;
        }
        if (Ss) memcpy(&Ss[t * P * N], S, sizeof(double) * (size_t)(P * N));
        if (Bts) memcpy(&Bts[t * N], Bt, sizeof(double) * (size_t)N);
        if (Cts) memcpy(&Cts[t * N], Ct, sizeof(double) * (size_t)N);
        if (phis) memcpy(&phis[t * K], phi, sizeof(double) * (size_t)K);
    }
    if (c->final_state) memcpy(&c->final_state[(b * H + h) * P * N], S,
                               sizeof(double) * (size_t)(P * N));
    free(S);
    free(Kp);
}

static void m3_fwd_row(void *vctx, int64_t row, int tid) {
    (void)tid;
    const m3_ctx *c = (const m3_ctx *)vctx;
    m3_forward_row(c, row / c->H, row % c->H, NULL, NULL, NULL, NULL, NULL);
}

int oracle_m3_fwd(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t K,
                  const double *x, const double *z, const double *Bm, const double *Cm,
                  const double *alpha, const double *beta, const double *gamma,
                  const double *theta, const double *Dp, const double *h0, double *out,
                  double *final_state, int nthreads) {
    if (N > ORACLE_MAX_N || 2 * K > N || G < 1 || H % G) return -1;
    m3_ctx c;
    memset(&c, 0, sizeof(c));
    c.Bsz = Bsz; c.L = L; c.H = H; c.P = P; c.N = N; c.G = G; c.K = K;
    c.x = x; c.z = z; c.Bm = Bm; c.Cm = Cm; c.alpha = alpha; c.beta = beta; c.gamma = gamma;
    c.theta = theta; c.Dp = Dp; c.h0 = h0; c.out = out; c.final_state = final_state;
    int64_t rows = Bsz * H;
    parallel_rows(rows, resolve_threads(nthreads, rows), m3_fwd_row, &c);
    return 0;
}

/*
 * Backward of one (batch, head) row.  With g_t = dout_t * silu(z_t):
 *   Lambda_t = g_t (outer) Ct_t + alpha_{t+1} Lambda_{t+1}      (dL/dS_t)
 *   dK_t     = gamma_t Lambda_t + beta_{t+1} Lambda_{t+1}       (dL/dK_t; the
 *              second term is the d_k_carry of stage B3)
 *   dalpha_t = <Lambda_t, S_{t-1}>, dbeta_t = <Lambda_t, K_{t-1}>,
 *   dgamma_t = <Lambda_t, K_t>
 *   dx_t[p]  = sum_n dK_t[p,n] Bt_t[n] + D g_t[p]
 *   dBt_t[n] = sum_p dK_t[p,n] x_t[p],   dCt_t[n] = sum_p g_t[p] S_t[p,n]
 *   RoPE backward: dB = R(phi)^T dBt (summed over the heads of the group),
 *   dphi_t[k] = dBt[2k+1] Bt[2k] - dBt[2k] Bt[2k+1] + (same with C),
 *   dtheta_t[k] = sum_{s >= t} dphi_s[k]        (reverse cumulative sum)
 *   dD += sum_p g_t[p] x_t[p],  dz_t = dout_t y_t silu'(z_t),
 *   dh0 = alpha_0 Lambda_0.
 */
static void m3_bwd_row(void *vctx, int64_t row, int tid) {
    const m3_ctx *c = (const m3_ctx *)vctx;
    const int64_t L = c->L, H = c->H, P = c->P, N = c->N, G = c->G, K = c->K;
    const int64_t b = row / H, h = row % H, g = h / (H / G);
    double *Ss = (double *)malloc(sizeof(double) * (size_t)(L * P * N));
    double *Bts = (double *)malloc(sizeof(double) * (size_t)(L * N));
    double *Cts = (double *)malloc(sizeof(double) * (size_t)(L * N));
    double *phis = (double *)malloc(sizeof(double) * (size_t)(L * (K > 0 ? K : 1)));
    double *ys = (double *)malloc(sizeof(double) * (size_t)(L * P));
    double *Lam = (double *)calloc((size_t)(P * N), sizeof(double));
    double *LamNext = (double *)calloc((size_t)(P * N), sizeof(double));
    double *dK = (double *)malloc(sizeof(double) * (size_t)(P * N));
    double gv[ORACLE_MAX_N * 4];
    double dBt[ORACLE_MAX_N], dCt[ORACLE_MAX_N], dphi[ORACLE_MAX_N], acc[ORACLE_MAX_N];
    double *dB = c->dB_part[tid], *dC = c->dC_part[tid], *dD = c->dD_part[tid];
    double alNext = 0.0, beNext = 0.0;

    m3_forward_row(c, b, h, Ss, Bts, Cts, phis, ys);
    for (int64_t k = 0; k < K; ++k) acc[k] = 0.0;

    for (int64_t t = L - 1; t >= 0; --t) {
        const double al = c->alpha[IDX_T(b, t, h)];
        const double be = c->beta[IDX_T(b, t, h)];
        const double ga = c->gamma[IDX_T(b, t, h)];
        const double *St = &Ss[t * P * N];
        const double *Bt = &Bts[t * N], *Ct = &Cts[t * N];
        for (int64_t p = 0; p < P; ++p) {
            const double dout = c->dout[IDX_X(b, t, h, p)];
            gv[p] = dout;
            if (c->z) {
                const double zt = c->z[IDX_X(b, t, h, p)];
                gv[p] = dout * silu(zt);
                if (c->dz) c->dz[IDX_X(b, t, h, p)] = dout * ys[t * P + p] * dsilu(zt);
            }
        }
        double dal = 0.0, dbe = 0.0, dga = 0.0;
        for (int64_t n = 0; n < N; ++n) { dBt[n] = 0.0; dCt[n] = 0.0; }
        for (int64_t p = 0; p < P; ++p) {
            const double xp = c->x[IDX_X(b, t, h, p)];
            const double xprev = t > 0 ? c->x[IDX_X(b, t - 1, h, p)] : 0.0;
            double dxp = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const int64_t i = p * N + n;
                Lam[i] = gv[p] * Ct[n] + alNext * LamNext[i];
                dK[i] = ga * Lam[i] + beNext * LamNext[i];
                const double Sprev = t > 0 ? Ss[(t - 1) * P * N + i]
                                           : (c->h0 ? c->h0[(b * H + h) * P * N + i] : 0.0);
                const double Kprev = t > 0 ? xprev * Bts[(t - 1) * N + n] : 0.0;
                const double Kt = xp * Bt[n];
                dal += Lam[i] * Sprev;
                dbe += Lam[i] * Kprev;
                dga += Lam[i] * Kt;
                dCt[n] += gv[p] * St[i];
                dBt[n] += dK[i] * xp;
                dxp += dK[i] * Bt[n];
            }
            if (c->Dp) dxp += c->Dp[h] * gv[p];
            c->dx[IDX_X(b, t, h, p)] = dxp;
            dD[h] += gv[p] * xp;
        }
        c->dalpha[IDX_T(b, t, h)] = dal;
        c->dbeta[IDX_T(b, t, h)] = dbe;
        c->dgamma[IDX_T(b, t, h)] = dga;

        /* RoPE backward */
        const double *phi = &phis[t * K];
        for (int64_t k = 0; k < K; ++k) {
            const double cs = cos(phi[k]), sn = sin(phi[k]);
            dB[IDX_BC(b, t, g, 2 * k)] += cs * dBt[2 * k] + sn * dBt[2 * k + 1];
            dB[IDX_BC(b, t, g, 2 * k + 1)] += -sn * dBt[2 * k] + cs * dBt[2 * k + 1];
            dC[IDX_BC(b, t, g, 2 * k)] += cs * dCt[2 * k] + sn * dCt[2 * k + 1];
            dC[IDX_BC(b, t, g, 2 * k + 1)] += -sn * dCt[2 * k] + cs * dCt[2 * k + 1];
            dphi[k] = dBt[2 * k + 1] * Bt[2 * k] - dBt[2 * k] * Bt[2 * k + 1]
                    + dCt[2 * k + 1] * Ct[2 * k] - dCt[2 * k] * Ct[2 * k + 1];
        }
        for (int64_t n = 2 * K; n < N; ++n) {
            dB[IDX_BC(b, t, g, n)] += dBt[n];
            dC[IDX_BC(b, t, g, n)] += dCt[n];
        }
        for (int64_t k = 0; k < K; ++k) {
            acc[k] += dphi[k];
            c->dtheta[IDX_TH(b, t, h, k)] = acc[k];
        }
        double *tmp = LamNext; LamNext = Lam; Lam = tmp;
        alNext = al;
        beNext = be;
    }
    if (c->dh0)
        for (int64_t i = 0; i < P * N; ++i) c->dh0[(b * H + h) * P * N + i] = alNext * LamNext[i];
    free(Ss); free(Bts); free(Cts); free(phis); free(ys); free(Lam); free(LamNext); free(dK);
}

int oracle_m3_bwd(int64_t Bsz, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t K,
                  const double *x, const double *z, const double *Bm, const double *Cm,
                  const double *alpha, const double *beta, const double *gamma,
                  const double *theta, const double *Dp, const double *h0, const double *dout,
                  double *dx, double *dz, double *dB, double *dC, double *dalpha, double *dbeta,
                  double *dgamma, double *dtheta, double *dD, double *dh0, int nthreads) {
    if (N > ORACLE_MAX_N || 2 * K > N || G < 1 || H % G || P > 4 * ORACLE_MAX_N) return -1;
    m3_ctx c;
    memset(&c, 0, sizeof(c));
    c.Bsz = Bsz; c.L = L; c.H = H; c.P = P; c.N = N; c.G = G; c.K = K;
    c.x = x; c.z = z; c.Bm = Bm; c.Cm = Cm; c.alpha = alpha; c.beta = beta; c.gamma = gamma;
    c.theta = theta; c.Dp = Dp; c.h0 = h0; c.dout = dout;
    c.dx = dx; c.dz = dz; c.dalpha = dalpha; c.dbeta = dbeta; c.dgamma = dgamma;
    c.dtheta = dtheta; c.dh0 = dh0;
    int64_t rows = Bsz * H;
    int nt = resolve_threads(nthreads, rows);
    c.dB_part = alloc_parts(nt, Bsz * L * G * N);
    c.dC_part = alloc_parts(nt, Bsz * L * G * N);
    c.dD_part = alloc_parts(nt, H);
    parallel_rows(rows, nt, m3_bwd_row, &c);
    fold_parts(c.dB_part, nt, Bsz * L * G * N, dB);
    fold_parts(c.dC_part, nt, Bsz * L * G * N, dC);
    fold_parts(c.dD_part, nt, H, dD);
    return 0;
}

/*
 * Mamba-3 SISO single-token state update (the step mamba3_step applies to a
 * Mamba3State, mamba-rs 0.7.0 README, "Quick start (CPU)", Mamba-3): one step
 * of the recurrence above for every (batch, head), written out on its own.
 * The carried state is S [B, H, P, N], the last step's input x_prev [B, H, P],
 * its rotated B bt_prev [B, H, N] (so that K_{t-1} = x_prev (outer) bt_prev)
 * and the cumulative angles phi [B, H, K]; all are updated in place.
 * Inputs: x, z, out [B, H, P]; B, C [B, G, N]; alpha, beta, gamma [B, H];
 * theta [B, H, K]; D [H].
 *   phi += theta;  Bt = R(phi) B;  Ct = R(phi) C
 *   S    = alpha S + beta x_prev (outer) bt_prev + gamma x (outer) Bt
 *   out  = (S Ct + D x) silu(z);   x_prev = x;  bt_prev = Bt
 */
int oracle_m3_state_update(int64_t Bsz, int64_t H, int64_t P, int64_t N, int64_t G, int64_t K,
                           double *S, double *x_prev, double *bt_prev, double *phi,
                           const double *x, const double *z, const double *Bm,
                           const double *Cm, const double *alpha, const double *beta,
                           const double *gamma, const double *theta, const double *Dp,
                           double *out) {
    if (N > ORACLE_MAX_N || 2 * K > N || G < 1 || H % G) return -1;
    double Bt[ORACLE_MAX_N], Ct[ORACLE_MAX_N];
    for (int64_t b = 0; b < Bsz; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const int64_t bh = b * H + h, g = h / (H / G);
            double *ph = &phi[bh * K];
            for (int64_t k = 0; k < K; ++k) ph[k] += theta[bh * K + k];
            rope_apply(&Bm[(b * G + g) * N], ph, N, K, Bt);
            rope_apply(&Cm[(b * G + g) * N], ph, N, K, Ct);
            const double al = alpha[bh], be = beta[bh], ga = gamma[bh];
            for (int64_t p = 0; p < P; ++p) {
                const double xp = x[bh * P + p], xq = x_prev[bh * P + p];
                double y = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double *s = &S[(bh * P + p) * N + n];
                    *s = al * *s + be * xq * bt_prev[bh * N + n] + ga * xp * Bt[n];
                    y += Ct[n] * *s;
                }
                if (Dp) y += Dp[h] * xp;
                out[bh * P + p] = z ? y * silu(z[bh * P + p]) : y;
            }
            for (int64_t p = 0; p < P; ++p) x_prev[bh * P + p] = x[bh * P + p];
            for (int64_t n = 0; n < N; ++n) bt_prev[bh * N + n] = Bt[n];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Causal depthwise conv1d ahead of the Mamba-1 scan                   */
/* ------------------------------------------------------------------ */
/*
 * The Mamba block's local convolution (the Mamba README, "Usage / Mamba
 * Block": d_conv, "Local convolution width"; the causal-conv1d extra of its
 * installation table; MambaState carries d_conv per layer, mamba-rs 0.7.0
 * README, "Quick start (CPU)"): per channel c, a causal convolution of width
 * W over time followed by SiLU, giving the scan's input u:
 *   v[b,c,t] = bias[c] + sum_{k<W} w[c,k] x[b,c,t-(W-1)+k]
 *   u[b,c,t] = silu(v[b,c,t])
 * with x at t < 0 taken from the initial conv state xs0[b,c,0..W-2] (the W-1
 * inputs before the sequence, oldest first) or 0.  The final conv state is
 * the last W-1 inputs.  Layouts: x, u [B, D, L]; w [D, W]; bias [D];
 * xs0, xs_final [B, D, W-1].
 */
static double conv_x(const double *x, const double *xs0, int64_t row, int64_t L, int64_t W,
                     int64_t t) {
    if (t >= 0) return x[row * L + t];
    return xs0 ? xs0[row * (W - 1) + (W - 1) + t] : 0.0;  /* t in [-(W-1), -1] */
}

int oracle_conv1d_fwd(int64_t Bsz, int64_t D, int64_t L, int64_t W, const double *x,
                      const double *w, const double *bias, const double *xs0, double *u,
                      double *xs_final) {
    if (W < 1) return -1;
    for (int64_t row = 0; row < Bsz * D; ++row) {
        const int64_t c = row % D;
        for (int64_t t = 0; t < L; ++t) {
            double v = bias ? bias[c] : 0.0;
            for (int64_t k = 0; k < W; ++k)
                v += w[c * W + k] * conv_x(x, xs0, row, L, W, t - (W - 1) + k);
            u[row * L + t] = silu(v);
        }
        if (xs_final)
            for (int64_t k = 0; k < W - 1; ++k)
                xs_final[row * (W - 1) + k] = conv_x(x, xs0, row, L, W, L - (W - 1) + k);
    }
    return 0;
}

/*
 * Backward of the above for an upstream gradient du [B, D, L]:
 *   dv[t]     = du[t] silu'(v[t])
 *   dx[t]     = sum_{k<W, t+(W-1)-k < L} w[c,k] dv[t+(W-1)-k]
 *   dw[c,k]   = sum_{b,t} dv[t] x[t-(W-1)+k]      (x at t < 0 from xs0 or 0)
 *   dbias[c]  = sum_{b,t} dv[t]
 *   dxs0[b,c,j] = sum_{k, 0 <= tau+(W-1)-k < L} w[c,k] dv[tau+(W-1)-k]
 *                 with tau = j-(W-1), the time of initial-state entry j
 */
int oracle_conv1d_bwd(int64_t Bsz, int64_t D, int64_t L, int64_t W, const double *x,
                      const double *w, const double *bias, const double *xs0, const double *du,
                      double *dx, double *dw, double *dbias, double *dxs0) {
    if (W < 1) return -1;
    double *dv = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int64_t i = 0; i < D * W; ++i) dw[i] = 0.0;
    if (dbias) for (int64_t c = 0; c < D; ++c) dbias[c] = 0.0;
    for (int64_t row = 0; row < Bsz * D; ++row) {
        const int64_t c = row % D;
        for (int64_t t = 0; t < L; ++t) {
            double v = bias ? bias[c] : 0.0;
            for (int64_t k = 0; k < W; ++k)
                v += w[c * W + k] * conv_x(x, xs0, row, L, W, t - (W - 1) + k);
            dv[t] = du[row * L + t] * dsilu(v);
        }
        for (int64_t t = 0; t < L; ++t) {
            double s = 0.0;
            for (int64_t k = 0; k < W; ++k) {
                const int64_t tt = t + (W - 1) - k;
                if (tt < L) s += w[c * W + k] * dv[tt];
            }
            dx[row * L + t] = s;
        }
        for (int64_t k = 0; k < W; ++k) {
            double s = 0.0;
            for (int64_t t = 0; t < L; ++t) s += dv[t] * conv_x(x, xs0, row, L, W, t - (W - 1) + k);
            dw[c * W + k] += s;
        }
        if (dbias) {
            double s = 0.0;
            for (int64_t t = 0; t < L; ++t) s += dv[t];
            dbias[c] += s;
        }
        if (dxs0)
            for (int64_t j = 0; j < W - 1; ++j) {  /* x at time tau = j - (W-1) */
                const int64_t tau = j - (W - 1);
                double s = 0.0;
                for (int64_t k = 0; k < W; ++k) {
                    const int64_t tt = tau + (W - 1) - k;
                    if (tt >= 0 && tt < L) s += w[c * W + k] * dv[tt];
                }
                dxs0[row * (W - 1) + j] = s;
            }
    }
    free(dv);
    return 0;
}
