/*
 * mss_oracle.c -- plain, slow, fp64 CPU oracle for the selective scan (S6)
 * forward pass and its single-token decode update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file or the library built from it: only the tests, the smoke
 * check of __graft_entry__ and the CPU-baseline leg of bench.py use it.  It
 * shares no source, header, table or helper with the CUDA library.
 *
 * What it computes, and where each step comes from:
 *
 *   - Continuous diagonal SSM h'(t) = A h(t) + B x(t), y = C h(t), one
 *     real SISO system per channel with diagonal A
 *     ["Mamba" paper review, section "SSM": the ODE and the diagonal/SISO
 *      shapes A in R^{NxN} diag, B in R^{Nx1}, C in R^{1xN}].
 *   - Step size Delta = softplus(Delta_raw + bias), softplus(x) = ln(1+e^x)
 *     ["Exercises -- State-space models (Mamba, S4)", the softplus exercise:
 *      Delta must be strictly positive, softplus maps R onto (0, inf)].
 *     softplus can be switched off (then Delta = Delta_raw + bias).
 *   - Zero-order hold for the transition: Abar = exp(Delta*A), per state for
 *     a diagonal A ["Mamba" paper review, section "SSM", discretisation
 *     formula; "Paper: Mamba" course page, Objectives, zero-order hold].
 *   - Input matrix by the Euler rule Bbar = Delta*B (the course page lists
 *     Euler as the alternative to the exact ZOH input matrix); so the input
 *     term is Bbar x = Delta * B_t * u_t.  On request (zoh_input), the exact
 *     zero-order-hold input matrix instead:
 *     Bbar = (Delta A)^{-1} (e^{Delta A} - I) Delta B = (e^{Delta A} - 1)/A * B
 *     per state ("Mamba" paper review, section "SSM"; "Paper: Mamba",
 *     Objectives), written with expm1 and with its limit Delta*B at A = 0.
 *   - Selective recurrence, state zero before the first token, update then
 *     read out:  h_t = Abar_t (.) h_{t-1} + Bbar_t x_t ,  y_t = C_t . h_t
 *     ["Mamba" paper review, section "SSM", discrete recurrence; "Exercises",
 *      recurrent view h_k = Abar h_{k-1} + Bbar x_k, then y_k = C h_k, worked
 *      impulse response starting from h = 0].  B_t and C_t depend on the
 *     token ("Mamba" paper review, section "Selection Mechanism").
 *   - Skip term and gate: y_t = (C_t . h_t + D u_t) * silu(z_t), with
 *     silu(z) = z / (1 + e^{-z}); z absent means no gate, D absent means 0.
 *     The pages name a gating mechanism that mixes in the residual
 *     ("Mamba" paper review, section "SSM", block description) but print no
 *     formula for it: this part has no printed value to pin against
 *     (parity unpinned beyond its closed-form definition).
 *   - Optional causal convolution in front of the scan: the input branch is
 *     "expanded via a linear layer, followed by a convolution and
 *     non-linearity" before the bank of SISO systems ("Mamba" paper review,
 *     section "SSM", block description), and the fused kernel of "NN Lab:
 *     Mamba" includes the causal 1D convolution.  Read as a depthwise
 *     (per-channel) causal convolution of width K followed by SiLU:
 *       u_t = silu(cb + sum_{k=0}^{K-1} w[k] x_{t-(K-1)+k}),
 *     with the K-1 values before the first token taken from a conv state
 *     (zero by default), and the conv state after the last token returned.
 *   - Final state: the state after the last token.  Decode: one step of the
 *     same recurrence starting from a caller-supplied state, which the
 *     "Exercises" page describes as the generation-time view (constant-size
 *     state, O(1) work per token).
 *
 * The sequential loop below is the plain definition.  A parallel scan
 * reaches the same numbers up to rounding order because the composition of
 * affine steps is associative ("NN Lab: Mamba", section "The Associative
 * Property of Linear Recurrence").
 *
 * Precision: every operation is fp64.  Inputs arrive as fp32 arrays: bf16
 * inputs are widened exactly by the caller, so no information is lost.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

/* softplus(s) = ln(1 + e^s).  For s > 0 the identity
 * ln(1 + e^s) = s + ln(1 + e^{-s}) keeps exp from overflowing; it is exact
 * algebra, not an approximation. */
double mss_oracle_softplus(double s)
{
    if (s > 0.0)
        return s + log1p(exp(-s));
    return log1p(exp(s));
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^{-z}). */
double mss_oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* One step of the discrete recurrence of one channel:
 *   h[n] <- abar[n] * h[n] + bx[n]    for every state n,
 * and the read-out sum_n c[n] * h[n] of the updated state. */
static double recurrence_step(double *h, const double *abar, const double *bx,
                              const double *c, int64_t N)
{
    double acc = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        h[n] = abar[n] * h[n] + bx[n];
        acc += c[n] * h[n];
    }
    return acc;
}

/* The discrete recurrence fed with already-discretised coefficients, for one
 * channel:  abar, bbar_x, c are [L][N] (row t holds Abar_t, Bbar_t x_t, C_t);
 * h starts at zero.  Writes y_out[L] and, if h_out is not NULL, the state
 * after every token into h_out[L][N].  Used to check the recurrence on the
 * worked example of the "Exercises" page, where Abar and Bbar are given. */
int mss_oracle_recurrence(const double *abar, const double *bbar_x, const double *c,
                          int64_t L, int64_t N, double *h_out, double *y_out)
{
    if (!abar || !bbar_x || !c || !y_out || L < 0 || N <= 0)
        return ORACLE_EINVAL;
    double *h = (double *)calloc((size_t)N, sizeof(double));
    if (!h)
        return ORACLE_ENOMEM;
    for (int64_t t = 0; t < L; ++t) {
        y_out[t] = recurrence_step(h, abar + t * N, bbar_x + t * N, c + t * N, N);
        if (h_out)
            for (int64_t n = 0; n < N; ++n)
                h_out[t * N + n] = h[n];
    }
    free(h);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Selective scan forward pass.                                              */

typedef struct {
    /* inputs, layouts as documented at mss_oracle_scan_fwd */
    const float *u, *delta, *A, *B, *C, *D, *z, *bias;
    const double *initial_state;
    int softplus_flag, zoh_input;
    double *y, *last_state;
    int64_t batch, dim, N, L;
    /* causal convolution in front of the scan (conv_width > 0: u holds x) */
    const float *conv_w, *conv_b;
    const double *conv_state_in;
    double *conv_state_out;
    int conv_width;
    /* rows [row_begin, row_end) of the flattened (batch, dim) index */
    int64_t row_begin, row_end;
    int status;
} scan_job;

/* Causal depthwise convolution of one channel.  ext holds the K-1 values
 * before the first token followed by the L inputs; out[t] is the
 * pre-activation cb + sum_k w[k] * ext[t + k] (ext[t + k] = x_{t-(K-1)+k}). */
static void causal_conv_row(const double *ext, int64_t L, const float *w, int K, double cb,
                            double *out)
{
    for (int64_t t = 0; t < L; ++t) {
        double acc = cb;
        for (int k = 0; k < K; ++k)
            acc += (double)w[k] * ext[t + k];
        out[t] = acc;
    }
}

/* The extended input of one channel: history (conv state, or zeros) then x. */
static void conv_extend(const double *state_in, const float *x, int64_t L, int K, double *ext)
{
    for (int k = 0; k < K - 1; ++k)
        ext[k] = state_in ? state_in[k] : 0.0;
    for (int64_t t = 0; t < L; ++t)
        ext[K - 1 + t] = (double)x[t];
}

/* Discretise one token of one channel: Delta from the raw value, then
 * Abar[n] = exp(Delta*A[n]) and Bbar x[n] = Delta * B[n] * u (Euler input
 * rule) or ((e^{Delta A[n]} - 1)/A[n]) * B[n] * u (zero-order hold). */
static double discretise(double delta_raw, double bias, int softplus_flag, int zoh_input,
                         const float *A_row, const float *B_bt, const float *C_bt,
                         int64_t L, int64_t N, double u,
                         double *abar, double *bx, double *c)
{
    double s = delta_raw + bias;
    double dt = softplus_flag ? mss_oracle_softplus(s) : s;
    for (int64_t n = 0; n < N; ++n) {
        const double a = (double)A_row[n];
        abar[n] = exp(dt * a);
        const double w = (zoh_input && a != 0.0) ? expm1(dt * a) / a : dt;
        bx[n] = w * (double)B_bt[n * L] * u;
        c[n] = (double)C_bt[n * L];
    }
    return dt;
}

static void *scan_rows(void *arg)
{
    scan_job *j = (scan_job *)arg;
    const int64_t N = j->N, L = j->L;
    const int K = j->conv_width;
    /* conv: the extended input (K-1+L) and the activations u (L) of a row */
    const int64_t conv_len = K > 0 ? (K - 1 + 2 * L) : 0;
    double *work = (double *)malloc((size_t)(4 * N + conv_len) * sizeof(double));
    if (!work) {
        j->status = ORACLE_ENOMEM;
        return NULL;
    }
    double *h = work, *abar = work + N, *bx = work + 2 * N, *c = work + 3 * N;
    double *ext = work + 4 * N, *uc = ext + (K > 0 ? K - 1 + L : 0);
    for (int64_t row = j->row_begin; row < j->row_end; ++row) {
        const int64_t b = row / j->dim, d = row % j->dim;
        const float *u = j->u + row * L;
        if (K > 0) {
            conv_extend(j->conv_state_in ? j->conv_state_in + row * (K - 1) : NULL, u, L, K, ext);
            causal_conv_row(ext, L, j->conv_w + d * K, K, j->conv_b ? (double)j->conv_b[d] : 0.0, uc);
            for (int64_t t = 0; t < L; ++t)
                uc[t] = mss_oracle_silu(uc[t]);
            if (j->conv_state_out)
                for (int k = 0; k < K - 1; ++k)
                    j->conv_state_out[row * (K - 1) + k] = ext[L + k];
        }
        const float *dr = j->delta + row * L;
        const float *z = j->z ? j->z + row * L : NULL;
        const float *A_row = j->A + d * N;
        const float *B_b = j->B + b * N * L; /* B[b][n][t] = B_b[n*L + t] */
        const float *C_b = j->C + b * N * L;
        const double Dd = j->D ? (double)j->D[d] : 0.0;
        const double bias = j->bias ? (double)j->bias[d] : 0.0;
        double *y = j->y + row * L;
        for (int64_t n = 0; n < N; ++n)
            h[n] = j->initial_state ? j->initial_state[row * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const double ut = K > 0 ? uc[t] : (double)u[t];
            discretise((double)dr[t], bias, j->softplus_flag, j->zoh_input, A_row, B_b + t, C_b + t,
                       L, N, ut, abar, bx, c);
            double out = recurrence_step(h, abar, bx, c, N) + Dd * ut;
            if (z)
                out *= mss_oracle_silu((double)z[t]);
            y[t] = out;
        }
        if (j->last_state)
            for (int64_t n = 0; n < N; ++n)
                j->last_state[row * N + n] = h[n];
    }
    free(work);
    j->status = ORACLE_OK;
    return NULL;
}

/* Run `fn` over rows [0, rows) split into `nthreads` contiguous ranges. */
static int run_threaded(scan_job *proto, int64_t rows, int nthreads, void *(*fn)(void *))
{
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > rows)
        nthreads = rows > 0 ? (int)rows : 1;
    scan_job *jobs = (scan_job *)calloc((size_t)nthreads, sizeof(scan_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = *proto;
        jobs[i].row_begin = rows * i / nthreads;
        jobs[i].row_end = rows * (i + 1) / nthreads;
        jobs[i].status = ORACLE_EINVAL;
        /* one range runs here; so does a range whose thread could not start */
        if (nthreads == 1 || pthread_create(&tids[i], NULL, fn, &jobs[i]) != 0) {
            fn(&jobs[i]);
            tids[i] = 0;
        }
    }
    int rc = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) {
        if (tids[i])
            pthread_join(tids[i], NULL);
        if (jobs[i].status != ORACLE_OK)
            rc = jobs[i].status;
    }
    free(jobs);
    free(tids);
    return rc;
}

/*
 * Forward pass.  Layouts (all contiguous, C order):
 *   u, delta, z : [batch][dim][L]   (token index fastest)
 *   A           : [dim][N]          (negative reals for a stable system)
 *   B, C        : [batch][N][L]     (shared by all channels of a batch row)
 *   D, bias     : [dim]             (D, z, bias may be NULL)
 *   zoh_input   : nonzero -> exact zero-order-hold input matrix, else Euler
 *   initial_state: [batch][dim][N]  fp64 state before the first token, or
 *                                   NULL for the zero state of the pages
 *   y           : [batch][dim][L]   fp64 output
 *   last_state  : [batch][dim][N]   fp64 output, may be NULL
 * Returns 0, or a negative code for bad arguments / no memory.
 */
int mss_oracle_scan_fwd(const float *u, const float *delta, const float *A,
                        const float *B, const float *C, const float *D,
                        const float *z, const float *delta_bias, int softplus_flag,
                        int zoh_input, const double *initial_state, double *y,
                        double *last_state, int64_t batch, int64_t dim, int64_t dstate,
                        int64_t seqlen, int nthreads)
{
    if (!u || !delta || !A || !B || !C || !y)
        return ORACLE_EINVAL;
    if (batch < 0 || dim < 0 || dstate <= 0 || seqlen < 0)
        return ORACLE_EINVAL;
    scan_job proto = {u, delta, A, B, C, D, z, delta_bias, initial_state, softplus_flag,
                      zoh_input, y, last_state, batch, dim, dstate, seqlen,
                      NULL, NULL, NULL, NULL, 0, 0, 0, ORACLE_OK};
    if (batch * dim == 0)
        return ORACLE_OK;
    return run_threaded(&proto, batch * dim, nthreads, scan_rows);
}

/*
 * Forward pass with the causal convolution in front: x takes the place of
 * u, and u = silu(conv(x)) feeds both the input term and the skip term.
 *   x            : [batch][dim][L]
 *   conv_w       : [dim][K], tap k multiplies x_{t-(K-1)+k}
 *   conv_b       : [dim] (may be NULL)
 *   conv_state_in: [batch][dim][K-1] fp64, x before the first token, oldest
 *                  first (NULL: zeros)
 *   conv_state_out: [batch][dim][K-1] fp64, the last K-1 values of the
 *                  history followed by x (may be NULL)
 * The other arguments are those of mss_oracle_scan_fwd.  K >= 1.
 */
int mss_oracle_scan_fwd_conv(const float *x, const float *conv_w, const float *conv_b,
                             int conv_width, const double *conv_state_in, double *conv_state_out,
                             const float *delta, const float *A, const float *B, const float *C,
                             const float *D, const float *z, const float *delta_bias,
                             int softplus_flag, int zoh_input, const double *initial_state,
                             double *y, double *last_state, int64_t batch, int64_t dim,
                             int64_t dstate, int64_t seqlen, int nthreads)
{
    if (!x || !conv_w || conv_width < 1 || !delta || !A || !B || !C || !y)
        return ORACLE_EINVAL;
    if (batch < 0 || dim < 0 || dstate <= 0 || seqlen < 0)
        return ORACLE_EINVAL;
    scan_job proto = {x, delta, A, B, C, D, z, delta_bias, initial_state, softplus_flag,
                      zoh_input, y, last_state, batch, dim, dstate, seqlen,
                      conv_w, conv_b, conv_state_in, conv_state_out, conv_width, 0, 0, ORACLE_OK};
    if (batch * dim == 0)
        return ORACLE_OK;
    return run_threaded(&proto, batch * dim, nthreads, scan_rows);
}

/*
 * The causal convolution alone (pre-activation, no SiLU), with the layouts of
 * mss_oracle_scan_fwd_conv; xc: [batch][dim][L] fp64.
 */
int mss_oracle_causal_conv(const float *x, const float *conv_w, const float *conv_b,
                           int conv_width, const double *conv_state_in, double *xc,
                           double *conv_state_out, int64_t batch, int64_t dim, int64_t seqlen)
{
    if (!x || !conv_w || conv_width < 1 || !xc || batch < 0 || dim < 0 || seqlen < 0)
        return ORACLE_EINVAL;
    const int K = conv_width;
    const int64_t L = seqlen;
    double *ext = (double *)malloc((size_t)(K - 1 + L + 1) * sizeof(double));
    if (!ext)
        return ORACLE_ENOMEM;
    for (int64_t row = 0; row < batch * dim; ++row) {
        const int64_t d = row % dim;
        conv_extend(conv_state_in ? conv_state_in + row * (K - 1) : NULL, x + row * L, L, K, ext);
        causal_conv_row(ext, L, conv_w + d * K, K, conv_b ? (double)conv_b[d] : 0.0, xc + row * L);
        if (conv_state_out)
            for (int k = 0; k < K - 1; ++k)
                conv_state_out[row * (K - 1) + k] = ext[L + k];
    }
    free(ext);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Single-token decode update.                                               */

typedef struct {
    double *state;
    const float *u, *delta, *A, *B, *C, *D, *z, *bias;
    int softplus_flag, zoh_input;
    double *y;
    int64_t dim, N;
    /* causal convolution in front (conv_width > 0: u holds x, conv_state is
     * read and shifted in place) */
    const float *conv_w, *conv_b;
    double *conv_state;
    int conv_width;
    int64_t row_begin, row_end;
    int status;
} step_job;

static void *step_rows(void *arg)
{
    step_job *j = (step_job *)arg;
    const int64_t N = j->N;
    double *work = (double *)malloc((size_t)(3 * N) * sizeof(double));
    if (!work) {
        j->status = ORACLE_ENOMEM;
        return NULL;
    }
    double *abar = work, *bx = work + N, *c = work + 2 * N;
    for (int64_t row = j->row_begin; row < j->row_end; ++row) {
        const int64_t b = row / j->dim, d = row % j->dim;
        double ut = (double)j->u[row];
        if (j->conv_width > 0) {
            /* the window: the K-1 stored values then this token's x */
            const int K = j->conv_width;
            double *cs = j->conv_state + row * (K - 1);
            double acc = j->conv_b ? (double)j->conv_b[d] : 0.0;
            for (int k = 0; k < K - 1; ++k)
                acc += (double)j->conv_w[d * K + k] * cs[k];
            acc += (double)j->conv_w[d * K + K - 1] * ut;
            for (int k = 0; k + 1 < K - 1; ++k)
                cs[k] = cs[k + 1];
            if (K > 1)
                cs[K - 2] = ut;
            ut = mss_oracle_silu(acc);
        }
        const double bias = j->bias ? (double)j->bias[d] : 0.0;
        /* B, C of a decode step are [batch][N]: stride 1 between states. */
        discretise((double)j->delta[row], bias, j->softplus_flag, j->zoh_input, j->A + d * N,
                   j->B + b * N, j->C + b * N, 1, N, ut, abar, bx, c);
        double out = recurrence_step(j->state + row * N, abar, bx, c, N);
        out += (j->D ? (double)j->D[d] : 0.0) * ut;
        if (j->z)
            out *= mss_oracle_silu((double)j->z[row]);
        j->y[row] = out;
    }
    free(work);
    j->status = ORACLE_OK;
    return NULL;
}

static int run_steps(step_job *proto, int64_t rows, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > rows)
        nthreads = rows > 0 ? (int)rows : 1;
    step_job *jobs = (step_job *)calloc((size_t)nthreads, sizeof(step_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = *proto;
        jobs[i].row_begin = rows * i / nthreads;
        jobs[i].row_end = rows * (i + 1) / nthreads;
        jobs[i].status = ORACLE_EINVAL;
        if (nthreads == 1 || pthread_create(&tids[i], NULL, step_rows, &jobs[i]) != 0) {
            step_rows(&jobs[i]);
            tids[i] = 0;
        }
    }
    int rc = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) {
        if (tids[i])
            pthread_join(tids[i], NULL);
        if (jobs[i].status != ORACLE_OK)
            rc = jobs[i].status;
    }
    free(jobs);
    free(tids);
    return rc;
}

/*
 * One decode step for every (batch, channel):
 *   state      : [batch][dim][N] fp64, read and overwritten in place
 *   u, delta, z: [batch][dim]
 *   A          : [dim][N]
 *   B, C       : [batch][N]
 *   D, bias    : [dim]  (D, z, bias may be NULL)
 *   zoh_input  : nonzero -> exact zero-order-hold input matrix, else Euler
 *   y          : [batch][dim] fp64 output
 */
int mss_oracle_state_update(double *state, const float *u, const float *delta,
                            const float *A, const float *B, const float *C,
                            const float *D, const float *z, const float *delta_bias,
                            int softplus_flag, int zoh_input, double *y,
                            int64_t batch, int64_t dim, int64_t dstate, int nthreads)
{
    if (!state || !u || !delta || !A || !B || !C || !y)
        return ORACLE_EINVAL;
    if (batch < 0 || dim < 0 || dstate <= 0)
        return ORACLE_EINVAL;
    step_job proto = {state, u, delta, A, B, C, D, z, delta_bias, softplus_flag, zoh_input, y,
                      dim, dstate, NULL, NULL, NULL, 0, 0, 0, ORACLE_OK};
    if (batch * dim == 0)
        return ORACLE_OK;
    return run_steps(&proto, batch * dim, nthreads);
}

/*
 * One decode step with the causal convolution in front: x takes the place of
 * u; conv_state [batch][dim][K-1] fp64 (oldest first) is read, shifted by one
 * and ends with this token's x.  Other arguments as mss_oracle_state_update.
 */
int mss_oracle_state_update_conv(double *state, double *conv_state, const float *x,
                                 const float *conv_w, const float *conv_b, int conv_width,
                                 const float *delta, const float *A, const float *B,
                                 const float *C, const float *D, const float *z,
                                 const float *delta_bias, int softplus_flag, int zoh_input,
                                 double *y, int64_t batch, int64_t dim, int64_t dstate,
                                 int nthreads)
{
    if (!state || !x || !conv_w || conv_width < 1 || (conv_width > 1 && !conv_state) ||
        !delta || !A || !B || !C || !y)
        return ORACLE_EINVAL;
    if (batch < 0 || dim < 0 || dstate <= 0)
        return ORACLE_EINVAL;
    step_job proto = {state, x, delta, A, B, C, D, z, delta_bias, softplus_flag, zoh_input, y,
                      dim, dstate, conv_w, conv_b, conv_state, conv_width, 0, 0, ORACLE_OK};
    if (batch * dim == 0)
        return ORACLE_OK;
    return run_steps(&proto, batch * dim, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Backward pass (reverse mode) of the forward pass above.                   */
/*
 * The pages train the model end to end ("Mamba" paper review, section
 * "Selection Mechanism": the kernel recomputes intermediate states in the
 * backward pass instead of storing them).  They print no gradient formula,
 * so this is the chain rule applied by hand to the definition above, one
 * step at a time, with the states of each row recomputed in fp64:
 *
 *   y_t = r_t * g_t,  g_t = silu(z_t) (1 without a gate),
 *   r_t = sum_n C_tn h_tn + D u_t,   h_tn = a_tn h_{t-1,n} + w_tn B_tn u_t,
 *   a_tn = exp(Delta_t A_n),  w_tn = Delta_t (Euler) or expm1(Delta_t A_n)/A_n,
 *   Delta_t = softplus(s_t) (or s_t),  s_t = delta_raw_t + bias.
 *
 * Walking t from L-1 down to 0 with gh = dLoss/dh_t (starting from the
 * gradient of last_state), each step adds dr_t C_t to gh, takes the
 * gradients of a_tn and of the input term, and leaves gh * a_t as
 * dLoss/dh_{t-1}.  B and C are shared by the channels of a batch row, A, D
 * and the bias by the rows of a channel: their gradients are summed.
 */

typedef struct {
    const float *u, *delta, *A, *B, *C, *D, *z, *bias, *dy;
    const double *initial_state, *dlast;
    int softplus_flag, zoh_input;
    int64_t batch, dim, N, L;
    /* per-row outputs */
    double *du, *ddelta, *dz, *dinit;
    /* summed outputs, private to this job: dA [dim][N], dD [dim], dbias [dim],
     * dB, dC [batch][N][L] */
    double *dA, *dD, *dbias, *dB, *dC;
    int64_t row_begin, row_end;
    int status;
} bwd_job;

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static void *bwd_rows(void *arg)
{
    bwd_job *j = (bwd_job *)arg;
    const int64_t N = j->N, L = j->L;
    /* per row: states h_t (L+1 rows, row 0 = the starting state), a_t, w_t,
     * Delta_t, s_t, r_t, and the adjoint gh */
    double *h = (double *)malloc((size_t)((L + 1) * N) * sizeof(double));
    double *a = (double *)malloc((size_t)(L * N + 1) * sizeof(double));
    double *w = (double *)malloc((size_t)(L * N + 1) * sizeof(double));
    double *sc = (double *)malloc((size_t)(3 * L + 1) * sizeof(double));
    double *gh = (double *)malloc((size_t)N * sizeof(double));
    if (!h || !a || !w || !sc || !gh) {
        free(h); free(a); free(w); free(sc); free(gh);
        j->status = ORACLE_ENOMEM;
        return NULL;
    }
    double *dts = sc, *ss = sc + L, *rs = sc + 2 * L;
    for (int64_t row = j->row_begin; row < j->row_end; ++row) {
        const int64_t b = row / j->dim, d = row % j->dim;
        const float *u = j->u + row * L, *dr_raw = j->delta + row * L;
        const float *z = j->z ? j->z + row * L : NULL;
        const float *dy = j->dy + row * L;
        const float *A_row = j->A + d * N;
        const float *B_b = j->B + b * N * L, *C_b = j->C + b * N * L;
        const double Dd = j->D ? (double)j->D[d] : 0.0;
        const double bias = j->bias ? (double)j->bias[d] : 0.0;
        /* forward, keeping every intermediate */
        for (int64_t n = 0; n < N; ++n)
            h[n] = j->initial_state ? j->initial_state[row * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const double s = (double)dr_raw[t] + bias;
            const double dt = j->softplus_flag ? mss_oracle_softplus(s) : s;
            const double ut = (double)u[t];
            double acc = 0.0;
            ss[t] = s;
            dts[t] = dt;
            for (int64_t n = 0; n < N; ++n) {
                const double An = (double)A_row[n];
                a[t * N + n] = exp(dt * An);
                w[t * N + n] = (j->zoh_input && An != 0.0) ? expm1(dt * An) / An : dt;
                h[(t + 1) * N + n] = a[t * N + n] * h[t * N + n] + w[t * N + n] * (double)B_b[n * L + t] * ut;
                acc += (double)C_b[n * L + t] * h[(t + 1) * N + n];
            }
            rs[t] = acc + Dd * ut;
        }
        /* reverse */
        for (int64_t n = 0; n < N; ++n)
            gh[n] = j->dlast ? j->dlast[row * N + n] : 0.0;
        for (int64_t t = L - 1; t >= 0; --t) {
            const double ut = (double)u[t], dt = dts[t];
            double dr = (double)dy[t];
            if (z) {
                const double zt = (double)z[t], sg = sigmoid(zt);
                j->dz[row * L + t] = (double)dy[t] * rs[t] * (sg + zt * sg * (1.0 - sg));
                dr *= mss_oracle_silu(zt);
            }
            j->dD[d] += dr * ut;
            double du = dr * Dd, ddt = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double An = (double)A_row[n], Bn = (double)B_b[n * L + t], Cn = (double)C_b[n * L + t];
                const double atn = a[t * N + n], wtn = w[t * N + n];
                gh[n] += dr * Cn; /* now dLoss/dh_t */
                j->dC[(b * N + n) * L + t] += dr * h[(t + 1) * N + n];
                /* input term w B u */
                j->dB[(b * N + n) * L + t] += gh[n] * wtn * ut;
                du += gh[n] * wtn * Bn;
                const double dw = gh[n] * Bn * ut;
                /* transition a = exp(Delta A) */
                const double da = gh[n] * h[t * N + n];
                ddt += da * atn * An;
                j->dA[d * N + n] += da * atn * dt;
                /* weight: Euler dw/dDelta = 1; zero-order hold dw/dDelta = a,
                 * dw/dA = (Delta a - w)/A (Delta^2/2 at A = 0) */
                if (j->zoh_input) {
                    ddt += dw * atn;
                    j->dA[d * N + n] += dw * (An != 0.0 ? (dt * atn - wtn) / An : 0.5 * dt * dt);
                } else {
                    ddt += dw;
                }
                gh[n] *= atn; /* dLoss/dh_{t-1} */
            }
            const double ds = ddt * (j->softplus_flag ? sigmoid(ss[t]) : 1.0);
            j->du[row * L + t] = du;
            j->ddelta[row * L + t] = ds;
            j->dbias[d] += ds;
        }
        if (j->dinit)
            for (int64_t n = 0; n < N; ++n)
                j->dinit[row * N + n] = gh[n];
    }
    free(h); free(a); free(w); free(sc); free(gh);
    j->status = ORACLE_OK;
    return NULL;
}

/*
 * Backward pass.  Inputs as mss_oracle_scan_fwd, plus
 *   dy      : [batch][dim][L]  gradient of the loss with respect to y
 *   dlast   : [batch][dim][N]  fp64 gradient with respect to last_state (NULL: 0)
 * Outputs (fp64, all written):
 *   du, ddelta   : [batch][dim][L]  (ddelta is with respect to delta_raw)
 *   dz           : [batch][dim][L]  (NULL allowed; required when z is given)
 *   dA           : [dim][N];  dD, dbias: [dim]
 *   dB, dC       : [batch][N][L]
 *   dinit        : [batch][dim][N] gradient with respect to initial_state (may be NULL)
 */
int mss_oracle_scan_bwd(const float *u, const float *delta, const float *A, const float *B,
                        const float *C, const float *D, const float *z, const float *delta_bias,
                        int softplus_flag, int zoh_input, const double *initial_state,
                        const float *dy, const double *dlast,
                        double *du, double *ddelta, double *dz, double *dA, double *dB, double *dC,
                        double *dD, double *dbias, double *dinit,
                        int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int nthreads)
{
    if (!u || !delta || !A || !B || !C || !dy || !du || !ddelta || !dA || !dB || !dC || !dD || !dbias ||
        (z && !dz))
        return ORACLE_EINVAL;
    if (batch < 0 || dim < 0 || dstate <= 0 || seqlen < 0)
        return ORACLE_EINVAL;
    const int64_t N = dstate, L = seqlen, rows = batch * dim;
    const size_t nA = (size_t)(dim * N), nBC = (size_t)(batch * N * L);
    for (size_t i = 0; i < nA; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < dim; ++i) dD[i] = dbias[i] = 0.0;
    for (size_t i = 0; i < nBC; ++i) dB[i] = dC[i] = 0.0;
    if (rows == 0)
        return ORACLE_OK;
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > rows)
        nthreads = (int)rows;
    bwd_job *jobs = (bwd_job *)calloc((size_t)nthreads, sizeof(bwd_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    /* each job sums into private buffers, added up at the end */
    const size_t priv = nA + 2 * (size_t)dim + 2 * nBC;
    double *sums = (double *)calloc((size_t)nthreads * priv, sizeof(double));
    if (!jobs || !tids || !sums) {
        free(jobs); free(tids); free(sums);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; ++i) {
        bwd_job *jb = &jobs[i];
        double *p = sums + (size_t)i * priv;
        *jb = (bwd_job){u, delta, A, B, C, D, z, delta_bias, dy, initial_state, dlast,
                        softplus_flag, zoh_input, batch, dim, N, L, du, ddelta, dz, dinit,
                        p, p + nA, p + nA + dim, p + nA + 2 * dim, p + nA + 2 * dim + nBC,
                        rows * i / nthreads, rows * (i + 1) / nthreads, ORACLE_EINVAL};
        if (nthreads == 1 || pthread_create(&tids[i], NULL, bwd_rows, jb) != 0) {
            bwd_rows(jb);
            tids[i] = 0;
        }
    }
    int rc = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) {
        if (tids[i])
            pthread_join(tids[i], NULL);
        if (jobs[i].status != ORACLE_OK)
            rc = jobs[i].status;
    }
    for (int i = 0; rc == ORACLE_OK && i < nthreads; ++i) {
        const bwd_job *jb = &jobs[i];
        for (size_t k = 0; k < nA; ++k) dA[k] += jb->dA[k];
        for (int64_t k = 0; k < dim; ++k) {
            dD[k] += jb->dD[k];
            dbias[k] += jb->dbias[k];
        }
        for (size_t k = 0; k < nBC; ++k) {
            dB[k] += jb->dB[k];
            dC[k] += jb->dC[k];
        }
    }
    free(jobs); free(tids); free(sums);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Structured state space duality (Mamba-2): scalar-times-identity A.        */
/*
 * "NN Lab: Mamba" (Structured State Space Duality) and the "Mamba" paper
 * review (section "Mamba 2"): A is restricted to a scalar times the identity
 * per head, which makes the sequence map a 1-semiseparable matrix
 * M_ji = a_{j:i} (C_j . B_i) and lets heads of P channels share B and C.
 * The oracle is the recurrence itself, per (batch, head), with an N x P state:
 *
 *   Delta_t = softplus(dt_t + bias_h),  a_t = exp(Delta_t A_h),
 *   S_t[n][p] = a_t S_{t-1}[n][p] + Delta_t B_t[n] x_t[p],
 *   y_t[p] = sum_n C_t[n] S_t[n][p] + D_h x_t[p],  times silu(z_t[p]).
 *
 * Layouts (token-major, as the heads of a token are contiguous):
 *   x, z, y : [batch][L][H][P];  dt: [batch][L][H];  A, D, bias: [H];
 *   B, C    : [batch][L][G][N], head h reads group h / (H / G);
 *   initial_state, last_state: [batch][H][N][P] (fp64).
 */

typedef struct {
    const float *x, *dt, *A, *B, *C, *D, *z, *bias;
    const double *initial_state;
    int softplus_flag;
    double *y, *last_state;
    int64_t batch, L, H, P, G, N;
    int64_t row_begin, row_end; /* rows = (batch, head) pairs */
    int status;
} ssd_job;

static void *ssd_rows(void *arg)
{
    ssd_job *j = (ssd_job *)arg;
    const int64_t L = j->L, H = j->H, P = j->P, G = j->G, N = j->N;
    double *S = (double *)malloc((size_t)(N * P) * sizeof(double));
    if (!S) {
        j->status = ORACLE_ENOMEM;
        return NULL;
    }
    for (int64_t row = j->row_begin; row < j->row_end; ++row) {
        const int64_t b = row / H, h = row % H, g = h / (H / G);
        const double Ah = (double)j->A[h];
        const double bias = j->bias ? (double)j->bias[h] : 0.0;
        const double Dh = j->D ? (double)j->D[h] : 0.0;
        for (int64_t k = 0; k < N * P; ++k)
            S[k] = j->initial_state ? j->initial_state[row * N * P + k] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const double s = (double)j->dt[(b * L + t) * H + h] + bias;
            const double delta = j->softplus_flag ? mss_oracle_softplus(s) : s;
            const double a = exp(delta * Ah);
            const float *Bt = j->B + ((b * L + t) * G + g) * N;
            const float *Ct = j->C + ((b * L + t) * G + g) * N;
            const float *xt = j->x + ((b * L + t) * H + h) * P;
            for (int64_t p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    S[n * P + p] = a * S[n * P + p] + delta * (double)Bt[n] * (double)xt[p];
                    acc += (double)Ct[n] * S[n * P + p];
                }
                double out = acc + Dh * (double)xt[p];
                if (j->z)
                    out *= mss_oracle_silu((double)j->z[((b * L + t) * H + h) * P + p]);
                j->y[((b * L + t) * H + h) * P + p] = out;
            }
        }
        if (j->last_state)
            for (int64_t k = 0; k < N * P; ++k)
                j->last_state[row * N * P + k] = S[k];
    }
    free(S);
    j->status = ORACLE_OK;
    return NULL;
}

int mss_oracle_ssd_fwd(const float *x, const float *dt, const float *A, const float *B, const float *C,
                       const float *D, const float *z, const float *dt_bias, int softplus_flag,
                       const double *initial_state, double *y, double *last_state,
                       int64_t batch, int64_t L, int64_t H, int64_t P, int64_t G, int64_t N, int nthreads)
{
    if (!x || !dt || !A || !B || !C || !y || batch < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 ||
        H % G != 0)
        return ORACLE_EINVAL;
    const int64_t rows = batch * H;
    if (rows == 0)
        return ORACLE_OK;
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > rows)
        nthreads = (int)rows;
    ssd_job *jobs = (ssd_job *)calloc((size_t)nthreads, sizeof(ssd_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (ssd_job){x, dt, A, B, C, D, z, dt_bias, initial_state, softplus_flag, y, last_state,
                            batch, L, H, P, G, N, rows * i / nthreads, rows * (i + 1) / nthreads, ORACLE_EINVAL};
        if (nthreads == 1 || pthread_create(&tids[i], NULL, ssd_rows, &jobs[i]) != 0) {
            ssd_rows(&jobs[i]);
            tids[i] = 0;
        }
    }
    int rc = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) {
        if (tids[i])
            pthread_join(tids[i], NULL);
        if (jobs[i].status != ORACLE_OK)
            rc = jobs[i].status;
    }
    free(jobs);
    free(tids);
    return rc;
}
