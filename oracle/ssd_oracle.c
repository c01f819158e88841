/*
 * ssd_oracle.c -- plain, slow, sequential fp64 reference of the Mamba-2 / SSD
 * selective-state-space mixer scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; its one input is plain arrays of numbers.
 *
 * What it computes, per (batch row b, head h), one token at a time:
 *
 *   1. causal depthwise conv (kernel K, usually 4) over the x|B|C channels,
 *      then SiLU  -- "Mini-K3-1H-mamba2-n64-g8" model card, Architecture
 *      ("causal depthwise-convolution kernel 4"); channel order x|B|C and
 *      conv_dim = d_inner + 2*n_groups*d_state from the codestral_mamba.ts
 *      weight-port header (tensor list).  K = 1 means "no conv" (the
 *      mojolearn Mamba3Block description: v is the raw x split, no conv), and
 *      then no SiLU either.
 *      Tap order is upstream PyTorch Conv1d order: w[c, K-1] multiplies the
 *      current token, w[c, 0] the token K-1 steps back (codestral_mamba.ts,
 *      "conv1d ... taps reversed" is the other engine's order, not ours).
 *   2. optional B/C RMSNorm (eps 1e-5) times a weight, plus a per-head bias
 *      -- mojolearn Mamba3Block, class description and Parameters
 *      (B_norm/C_norm weight (N,), B_bias/C_bias (H, N)).
 *   3. dt = softplus(dt_raw + dt_bias[h]) with no clamp -- falcon_mamba.ts
 *      header ("softplus(dt + bias)"), Mamba3Block ("no dt clamp").
 *   4. a = A[h] (per-head A, given already negative: A = -exp(A_log) per the
 *      codestral_mamba.ts reconciliation 2), or the per-token per-head
 *      A[b,t,h] clamped so that |a| >= 1e-4 (Mamba3Block, "A floor 1e-4").
 *   5. packed-document reset: when seq_idx[t] != seq_idx[t-1] the recurrent
 *      state restarts from zero and the conv sees no tap from another
 *      document (model card, "Checkpoint and training": document IDs reset
 *      convolution history and recurrent state at every boundary).  The
 *      caller's initial state belongs to the first document of the row.
 *   6. h[p,n] <- exp(dt*a) * h[p,n] + dt * x[p] * B[n]
 *   7. y[p] = sum_n C[n] * h[p,n] + D[h] * x[p];  out = y * silu(z[p])
 *      (the gate is applied in the core: Mamba3Block class description; D is
 *      the "structural D (skip connection)" of the transplant article).
 *   8. after the last token: final SSM state h, and the last K-1 raw conv
 *      inputs, zeroed where they belong to another document than the last
 *      token's.
 *   9. ragged batches: with per-row lengths, row b holds lengths[b] tokens and
 *      the rest of the row is padding -- no token of the recurrence at all.
 *      Padding outputs are +0.0, and the final state and conv history are
 *      those after the row's last real token (a zero-length row hands its
 *      initial state and history through unchanged).
 *
 * A decode step is this same computation at L = 1 with the state carried
 * (Mamba3Block.step: "the same computation as forward at L = 1").
 *
 * Everything is double precision.  Inputs arrive as float32 arrays holding
 * exactly the values the GPU receives (bf16 values widen to fp32 exactly).
 * Work is spread over (b, h) pairs with POSIX threads; each pair is computed
 * by one thread, in token order, with no blocking or reordering.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Shapes and switches of one call.  Layouts (row-major, contiguous):
 *   x, z      (batch, seqlen, nheads*headdim)        float32
 *   Bm, Cm    (batch, seqlen, ngroups*dstate)        float32
 *   dt_raw    (batch, seqlen, nheads)                float32
 *   dt_bias, D (nheads)                              float32
 *   A         (nheads) or (batch, seqlen, nheads)    float32, already negative
 *   conv_w    (conv_dim, dconv), conv_b (conv_dim)   float32, x|B|C channel order
 *   seq_idx   (batch, seqlen) int32 or NULL (one document per row)
 *   init_ssm  (batch, nheads, headdim, dstate) float32 or NULL (zeros)
 *   init_conv (batch, dconv-1, conv_dim) float32 or NULL (zeros); index 0 is
 *             the oldest token
 *   bn_w, cn_w (dstate) or NULL (ones); bn_bias, cn_bias (nheads, dstate) or
 *             NULL (zeros) -- only read when bc_norm != 0
 *   lengths   (batch) int32 real tokens per row, clamped to [0, seqlen], or
 *             NULL (every row is seqlen long)
 * Outputs (double):
 *   out       (batch, seqlen, nheads*headdim)
 *   fin_ssm   (batch, nheads, headdim, dstate) or NULL
 *   fin_conv  (batch, dconv-1, conv_dim) or NULL
 */
typedef struct {
    int batch, seqlen, nheads, headdim, dstate, ngroups, dconv;
    int a_per_token, bc_norm;
} oracle_dims;

typedef struct {
    const float *x, *z, *Bm, *Cm, *dt_raw, *dt_bias, *A, *D, *conv_w, *conv_b;
    const int32_t *seq_idx;
    const float *init_ssm, *init_conv;
    const float *bn_w, *cn_w, *bn_bias, *cn_bias;
    const int32_t *lengths;
} oracle_inputs;

/* Real tokens of row b. */
static int row_len(const oracle_dims *d, const oracle_inputs *in, int b)
{
    if (!in->lengths) return d->seqlen;
    const int v = in->lengths[b];
    return v < 0 ? 0 : (v > d->seqlen ? d->seqlen : v);
}

static double softplus_exact(double v)
{
    /* log(1 + e^v), written so that neither branch overflows. */
    if (v > 20.0) return v + log1p(exp(-v));
    return log1p(exp(v));
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

static int conv_dim_of(const oracle_dims *d)
{
    return d->nheads * d->headdim + 2 * d->ngroups * d->dstate;
}

/* Raw (pre-conv) value of channel ch of the x|B|C stream at (b, t). */
static double xbc_raw(const oracle_dims *d, const oracle_inputs *in, int b, int t, int ch)
{
    const int dx = d->nheads * d->headdim, gn = d->ngroups * d->dstate;
    const size_t row = (size_t)b * d->seqlen + t;
    if (ch < dx) return in->x[row * dx + ch];
    if (ch < dx + gn) return in->Bm[row * gn + (ch - dx)];
    return in->Cm[row * gn + (ch - dx - gn)];
}

/* 1 when no document boundary lies in (t0, t1], t0 <= t1: a boundary is a
 * position r > 0 whose id differs from its left neighbour's, so ids are only
 * ever compared between neighbours (an id may recur later in the row and
 * still start a new document). */
static int same_doc(const oracle_inputs *in, const oracle_dims *d, int b, int t0, int t1)
{
    if (!in->seq_idx) return 1;
    const int32_t *s = in->seq_idx + (size_t)b * d->seqlen;
    for (int r = t0 + 1; r <= t1; r++)
        if (s[r] != s[r - 1]) return 0;
    return 1;
}

/* Channel ch of the conv+SiLU output at (b, t); with dconv == 1 the raw value. */
static double conv_silu(const oracle_dims *d, const oracle_inputs *in, int b, int t, int ch)
{
    const int K = d->dconv, cd = conv_dim_of(d);
    if (K == 1) return xbc_raw(d, in, b, t, ch);
    double acc = in->conv_b[ch];
    for (int k = 0; k < K; k++) {
        const int tau = t - (K - 1) + k;
        double v = 0.0;
        if (tau >= 0) {
            if (same_doc(in, d, b, tau, t)) v = xbc_raw(d, in, b, tau, ch);
        } else if (in->init_conv && same_doc(in, d, b, 0, t)) {
            v = in->init_conv[((size_t)b * (K - 1) + (tau + K - 1)) * cd + ch];
        }
        acc += (double)in->conv_w[(size_t)ch * K + k] * v;
    }
    return silu(acc);
}

typedef struct {
    const oracle_dims *d;
    const oracle_inputs *in;
    double *out, *fin_ssm;
    const int32_t *pairs; /* (b, h) pairs, or NULL for all */
    int npairs;
    int next;             /* next pair index, taken under the lock */
    pthread_mutex_t lock;
} pair_job;

static void run_pair(const oracle_dims *d, const oracle_inputs *in, int b, int h,
                     double *out, double *fin_ssm)
{
    const int L = d->seqlen, P = d->headdim, N = d->dstate, H = d->nheads;
    const int g = h / (H / d->ngroups);
    const int dx = H * P, gn = d->ngroups * N;
    double *hs = calloc((size_t)P * N, sizeof(double));
    double *ux = malloc(sizeof(double) * P);
    double *ub = malloc(sizeof(double) * N);
    double *uc = malloc(sizeof(double) * N);
    if (!hs || !ux || !ub || !uc) abort();

    if (in->init_ssm) {
        const float *s0 = in->init_ssm + ((size_t)b * H + h) * P * N;
        for (int i = 0; i < P * N; i++) hs[i] = s0[i];
    }
    const int Lb = row_len(d, in, b);
    for (int t = Lb; t < L; t++)   /* padding */
        for (int p = 0; p < P; p++) out[((size_t)b * L + t) * dx + h * P + p] = 0.0;
    for (int t = 0; t < Lb; t++) {
        if (t > 0 && !same_doc(in, d, b, t - 1, t)) memset(hs, 0, sizeof(double) * P * N);

        for (int p = 0; p < P; p++) ux[p] = conv_silu(d, in, b, t, h * P + p);
        for (int n = 0; n < N; n++) {
            ub[n] = conv_silu(d, in, b, t, dx + g * N + n);
            uc[n] = conv_silu(d, in, b, t, dx + gn + g * N + n);
        }
        if (d->bc_norm) {
            double sb = 0.0, sc = 0.0;
            for (int n = 0; n < N; n++) { sb += ub[n] * ub[n]; sc += uc[n] * uc[n]; }
            const double rb = 1.0 / sqrt(sb / N + 1e-5), rc = 1.0 / sqrt(sc / N + 1e-5);
            for (int n = 0; n < N; n++) {
                const double wb = in->bn_w ? in->bn_w[n] : 1.0, wc = in->cn_w ? in->cn_w[n] : 1.0;
                const double bb = in->bn_bias ? in->bn_bias[(size_t)h * N + n] : 0.0;
                const double bc = in->cn_bias ? in->cn_bias[(size_t)h * N + n] : 0.0;
                ub[n] = ub[n] * rb * wb + bb;
                uc[n] = uc[n] * rc * wc + bc;
            }
        }

        const size_t tok = (size_t)b * L + t;
        const double dt = softplus_exact((double)in->dt_raw[tok * H + h] + in->dt_bias[h]);
        double a;
        if (d->a_per_token) {
            a = in->A[tok * H + h];
            if (a > -1e-4) a = -1e-4;
        } else {
            a = in->A[h];
        }
        const double decay = exp(dt * a);

        for (int p = 0; p < P; p++) {
            double *hp = hs + (size_t)p * N;
            const double dxp = dt * ux[p];
            double y = 0.0;
            for (int n = 0; n < N; n++) {
                hp[n] = decay * hp[n] + dxp * ub[n];
                y += uc[n] * hp[n];
            }
            y += in->D[h] * ux[p];
            const double zv = in->z[tok * dx + h * P + p];
            out[tok * dx + h * P + p] = y * silu(zv);
        }
    }
    if (fin_ssm) memcpy(fin_ssm + ((size_t)b * H + h) * P * N, hs, sizeof(double) * P * N);
    free(hs); free(ux); free(ub); free(uc);
}

static void *pair_worker(void *arg)
{
    pair_job *j = arg;
    const int total = j->pairs ? j->npairs : j->d->batch * j->d->nheads;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        const int i = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (i >= total) break;
        int b, h;
        if (j->pairs) { b = j->pairs[2 * i]; h = j->pairs[2 * i + 1]; }
        else { b = i / j->d->nheads; h = i % j->d->nheads; }
        run_pair(j->d, j->in, b, h, j->out, j->fin_ssm);
    }
    return NULL;
}

/* Number of worker threads the oracle uses when asked for 0 (all online cores). */
int oracle_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/*
 * Full forward.  pairs: npairs (b, h) pairs to compute, or NULL for all;
 * outputs of pairs not computed are left untouched.  fin_conv, when given, is
 * filled for every batch row.  Returns the number of threads used, or -1 on a
 * bad argument.
 */
int oracle_forward(const oracle_dims *d, const oracle_inputs *in,
                   const int32_t *pairs, int npairs, int nthreads,
                   double *out, double *fin_ssm, double *fin_conv)
{
    if (!d || !in || !out) return -1;
    if (d->batch < 0 || d->seqlen < 1 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 ||
        d->ngroups < 1 || d->nheads % d->ngroups || d->dconv < 1)
        return -1;
    if (d->dconv > 1 && (!in->conv_w || !in->conv_b)) return -1;

    pair_job j;
    j.d = d; j.in = in; j.out = out; j.fin_ssm = fin_ssm;
    j.pairs = pairs; j.npairs = npairs; j.next = 0;
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads <= 0) nthreads = oracle_default_threads();
    const int total = pairs ? npairs : d->batch * d->nheads;
    if (nthreads > total) nthreads = total > 0 ? total : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; i++) pthread_create(&th[i], NULL, pair_worker, &j);
    pair_worker(&j);
    for (int i = 1; i < nthreads; i++) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j.lock);

    if (fin_conv && d->dconv > 1) {
        const int K = d->dconv, cd = conv_dim_of(d);
        for (int b = 0; b < d->batch; b++)
            for (int i = 0; i < K - 1; i++) {
                const int L = row_len(d, in, b);   /* the row's last real token is L - 1 */
                const int tau = L - (K - 1) + i;
                for (int ch = 0; ch < cd; ch++) {
                    double v = 0.0;
                    if (tau >= 0) {
                        if (same_doc(in, d, b, tau, L - 1)) v = xbc_raw(d, in, b, tau, ch);
                    } else if (in->init_conv && same_doc(in, d, b, 0, L - 1)) {
                        v = in->init_conv[((size_t)b * (K - 1) + (tau + K - 1)) * cd + ch];
                    }
                    fin_conv[((size_t)b * (K - 1) + i) * cd + ch] = v;
                }
            }
    }
    return nthreads;
}

/* Stage: conv+SiLU output of every x|B|C channel, (batch, seqlen, conv_dim). */
int oracle_conv(const oracle_dims *d, const oracle_inputs *in, double *u)
{
    if (!d || !in || !u || d->dconv < 1) return -1;
    const int cd = conv_dim_of(d);
    for (int b = 0; b < d->batch; b++)
        for (int t = 0; t < d->seqlen; t++)
            for (int ch = 0; ch < cd; ch++)
                u[((size_t)b * d->seqlen + t) * cd + ch] = conv_silu(d, in, b, t, ch);
    return 0;
}

/* Stage: dt = softplus(dt_raw + dt_bias) and a (floored when per token), (batch, seqlen, nheads). */
int oracle_dt(const oracle_dims *d, const oracle_inputs *in, double *dt, double *a)
{
    if (!d || !in || !dt) return -1;
    const int H = d->nheads;
    for (int b = 0; b < d->batch; b++)
        for (int t = 0; t < d->seqlen; t++)
            for (int h = 0; h < H; h++) {
                const size_t i = ((size_t)b * d->seqlen + t) * H + h;
                dt[i] = softplus_exact((double)in->dt_raw[i] + in->dt_bias[h]);
                if (a) {
                    double av = d->a_per_token ? in->A[i] : in->A[h];
                    if (d->a_per_token && av > -1e-4) av = -1e-4;
                    a[i] = av;
                }
            }
    return 0;
}

/* Stage: normalised, biased B and C per head, (batch, seqlen, nheads, dstate) each,
 * taken from the raw B and C (the configurations with a B/C norm have no conv). */
int oracle_bcnorm(const oracle_dims *d, const oracle_inputs *in, double *bh, double *ch_out)
{
    if (!d || !in || !bh || !ch_out) return -1;
    const int H = d->nheads, N = d->dstate, gn = d->ngroups * N;
    for (int b = 0; b < d->batch; b++)
        for (int t = 0; t < d->seqlen; t++) {
            const size_t row = (size_t)b * d->seqlen + t;
            for (int h = 0; h < H; h++) {
                const int g = h / (H / d->ngroups);
                const float *bv = in->Bm + row * gn + (size_t)g * N;
                const float *cv = in->Cm + row * gn + (size_t)g * N;
                double sb = 0.0, sc = 0.0;
                for (int n = 0; n < N; n++) { sb += (double)bv[n] * bv[n]; sc += (double)cv[n] * cv[n]; }
                const double rb = 1.0 / sqrt(sb / N + 1e-5), rc = 1.0 / sqrt(sc / N + 1e-5);
                for (int n = 0; n < N; n++) {
                    const size_t o = (row * H + h) * N + n;
                    bh[o] = bv[n] * rb * (in->bn_w ? in->bn_w[n] : 1.0) +
                            (in->bn_bias ? in->bn_bias[(size_t)h * N + n] : 0.0);
                    ch_out[o] = cv[n] * rc * (in->cn_w ? in->cn_w[n] : 1.0) +
                                (in->cn_bias ? in->cn_bias[(size_t)h * N + n] : 0.0);
                }
            }
        }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Mamba-1 selective scan (S6) -- the second scan the pages describe, for the
 * Falcon-Mamba port (falcon_mamba.ts header, "Mamba-1 / S6"):
 *
 *   per batch row b and channel d (d_inner of them), state size N:
 *     A[d,n] = -exp(clamp(A_log[d,n], -10, 5))       (selective_scan.ts, quoted
 *                                                      by the falcon_mamba.ts header)
 *     dt_t   = softplus(delta_t[d] + delta_bias[d])   ("softplus(dt + bias)", no clamp)
 *     h[n]  <- exp(dt_t A[d,n]) h[n] + dt_t u_t[d] B_t[n]
 *     y_t    = sum_n C_t[n] h[n] + D[d] u_t[d];   out = y_t * silu(z_t[d]) (no z: y_t)
 *
 * A is diagonal (one decay per channel and state), B and C are shared by all
 * channels of a token, u is the already convolved input (the conv sits before
 * the x_proj projection that produces delta, B and C).  Same fp64, one-token-
 * at-a-time evaluation as oracle_forward; rows run in parallel threads.
 *
 * Layouts (row-major, float32 in):
 *   u, delta, z   (batch, seqlen, d_inner)   (z may be NULL)
 *   Bm, Cm        (batch, seqlen, dstate)
 *   A_log         (d_inner, dstate);  delta_bias, D (d_inner)
 *   init          (batch, d_inner, dstate) or NULL (zeros)
 * Out (double): out (batch, seqlen, d_inner); fin (batch, d_inner, dstate) or NULL.
 */
typedef struct {
    int batch, seqlen, d_inner, dstate;
} oracle_s6_dims;

typedef struct {
    const float *u, *delta, *delta_bias, *A_log, *Bm, *Cm, *D, *z, *init;
} oracle_s6_inputs;

typedef struct {
    const oracle_s6_dims *d;
    const oracle_s6_inputs *in;
    double *out, *fin;
    int next;
    pthread_mutex_t lock;
} s6_job;

static void s6_row(const oracle_s6_dims *d, const oracle_s6_inputs *in, int b, double *out, double *fin)
{
    const int L = d->seqlen, DI = d->d_inner, N = d->dstate;
    double *h = malloc(sizeof(double) * (size_t)DI * N);
    double *a = malloc(sizeof(double) * (size_t)DI * N);
    if (!h || !a) abort();
    for (int c = 0; c < DI; c++)
        for (int n = 0; n < N; n++) {
            double al = in->A_log[(size_t)c * N + n];
            if (al < -10.0) al = -10.0;
            if (al > 5.0) al = 5.0;
            a[(size_t)c * N + n] = -exp(al);
            h[(size_t)c * N + n] = in->init ? in->init[((size_t)b * DI + c) * N + n] : 0.0;
        }
    for (int t = 0; t < L; t++) {
        const size_t tok = (size_t)b * L + t;
        const float *Bt = in->Bm + tok * N, *Ct = in->Cm + tok * N;
        for (int c = 0; c < DI; c++) {
            const double dt = softplus_exact((double)in->delta[tok * DI + c] + in->delta_bias[c]);
            const double uv = in->u[tok * DI + c];
            double *hc = h + (size_t)c * N;
            double y = 0.0;
            for (int n = 0; n < N; n++) {
                hc[n] = exp(dt * a[(size_t)c * N + n]) * hc[n] + dt * uv * Bt[n];
                y += Ct[n] * hc[n];
            }
            y += in->D[c] * uv;
            out[tok * DI + c] = in->z ? y * silu(in->z[tok * DI + c]) : y;
        }
    }
    if (fin) memcpy(fin + (size_t)b * DI * N, h, sizeof(double) * (size_t)DI * N);
    free(h); free(a);
}

static void *s6_worker(void *arg)
{
    s6_job *j = arg;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        const int b = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (b >= j->d->batch) break;
        s6_row(j->d, j->in, b, j->out, j->fin);
    }
    return NULL;
}

/* Returns the number of threads used, or -1 on a bad argument. */
int oracle_s6_forward(const oracle_s6_dims *d, const oracle_s6_inputs *in, int nthreads,
                      double *out, double *fin)
{
    if (!d || !in || !out || d->batch < 0 || d->seqlen < 1 || d->d_inner < 1 || d->dstate < 1)
        return -1;
    if (!in->u || !in->delta || !in->delta_bias || !in->A_log || !in->Bm || !in->Cm || !in->D)
        return -1;
    s6_job j;
    j.d = d; j.in = in; j.out = out; j.fin = fin; j.next = 0;
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads <= 0) nthreads = oracle_default_threads();
    if (nthreads > d->batch) nthreads = d->batch > 0 ? d->batch : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; i++) pthread_create(&th[i], NULL, s6_worker, &j);
    s6_worker(&j);
    for (int i = 1; i < nthreads; i++) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j.lock);
    return nthreads;
}

/* ------------------------------------------------------------------------------------
 * Backward of a zero-state prefill: the vector-Jacobian product of
 * oracle_forward (mojolearn Mamba3Block, method "backward": the gradients of
 * the loss with respect to the forward input and every weight, given the
 * gradient of the output; nothing with respect to a carried state, and no
 * final-state cotangent -- so init_ssm and init_conv must be NULL).
 *
 * Plain reverse-mode differentiation of the same per-token steps 1-9, in
 * double precision, done per batch row:
 *
 *   forward sweep   per head, token by token, keeping every state h_t;
 *   reverse sweep   per head, from the row's last real token to the first:
 *     out = y silu(z)          gy = gout silu(z),  gz = gout y silu'(z)
 *     y = C.h_t + D u_x        gC += gy h_t, gh_t += gy C, gD += gy u_x, gu_x += gy D
 *     h_t = e h_{t-1} + dt u_x B
 *                              ge = <gh_t, h_{t-1}>, gdt += <gh_t, u_x B>,
 *                              gu_x += dt gh_t B, gB += dt gh_t^T u_x,
 *                              gh_{t-1} = e gh_t, or 0 when t starts a document
 *     e = exp(dt a)            gdt += ge e a,  ga = ge e dt
 *     dt = softplus(v)         gv = gdt sigmoid(v) -> dt_raw[t], dt_bias
 *     a = min(A, -1e-4)        ga passes where A <= -1e-4, else 0 (per-token A)
 *     B^ = B r w + bias, r = (mean(B^2) + 1e-5)^(-1/2)
 *                              gw += gB^ B r, gbias += gB^,
 *                              gB = r w gB^ - (r^3 / N) B <gB^, w B>
 *   then the conv of the row:  u = silu(pre), pre = b + sum_k w_k x[t-3+k] (same document)
 *                              gpre = gu silu'(pre), gb += gpre, gw_k += gpre x[.],
 *                              gx[.] += gpre w_k
 *
 * B and C (and their conv channels) are shared by the heads of a group, so
 * their gradients are sums over those heads.  Weight gradients are summed
 * per row, and then over rows in row order.  Padding tokens of a ragged row
 * (t >= lengths[b]) take no part: every gradient there is 0 and the output
 * gradient there is ignored.
 *
 * gout has the layout of out (float32).  Gradients (double) have the layout
 * of the input they belong to; the conv ones (conv_w, conv_b) are only
 * written when dconv > 1 and the norm ones (bn_w .. cn_bias) only when
 * bc_norm != 0.
 */
typedef struct {
    double *x, *z, *Bm, *Cm, *dt_raw, *dt_bias, *A, *D, *conv_w, *conv_b;
    double *bn_w, *cn_w, *bn_bias, *cn_bias;
} oracle_grads;

/* Weight gradients of one batch row (summed over rows afterwards). */
typedef struct {
    double *dt_bias, *A, *D, *conv_w, *conv_b, *bn_w, *cn_w, *bn_bias, *cn_bias;
} row_wgrads;

/* What token t of head h sees: u_x (P), the raw group B/C after the conv (N),
 * the per-head B^/C^ (N), the norms' 1/rms, dt, its softplus argument, the
 * decay rate and whether the per-token floor replaced it. */
typedef struct {
    double *ux, *ub, *uc, *bh, *ch;
    double rb, rc, dt, v, a, decay;
    int floored;
} tok_terms;

static void token_terms(const oracle_dims *d, const oracle_inputs *in, int b, int h, int t,
                        tok_terms *k)
{
    const int P = d->headdim, N = d->dstate, H = d->nheads;
    const int g = h / (H / d->ngroups);
    const int dx = H * P, gn = d->ngroups * N;
    for (int p = 0; p < P; p++) k->ux[p] = conv_silu(d, in, b, t, h * P + p);
    for (int n = 0; n < N; n++) {
        k->ub[n] = conv_silu(d, in, b, t, dx + g * N + n);
        k->uc[n] = conv_silu(d, in, b, t, dx + gn + g * N + n);
    }
    k->rb = k->rc = 1.0;
    if (d->bc_norm) {
        double sb = 0.0, sc = 0.0;
        for (int n = 0; n < N; n++) { sb += k->ub[n] * k->ub[n]; sc += k->uc[n] * k->uc[n]; }
        k->rb = 1.0 / sqrt(sb / N + 1e-5);
        k->rc = 1.0 / sqrt(sc / N + 1e-5);
    }
    for (int n = 0; n < N; n++) {
        if (d->bc_norm) {
            const double wb = in->bn_w ? in->bn_w[n] : 1.0, wc = in->cn_w ? in->cn_w[n] : 1.0;
            const double bb = in->bn_bias ? in->bn_bias[(size_t)h * N + n] : 0.0;
            const double bc = in->cn_bias ? in->cn_bias[(size_t)h * N + n] : 0.0;
            k->bh[n] = k->ub[n] * k->rb * wb + bb;
            k->ch[n] = k->uc[n] * k->rc * wc + bc;
        } else {
            k->bh[n] = k->ub[n];
            k->ch[n] = k->uc[n];
        }
    }
    const size_t tok = (size_t)b * d->seqlen + t;
    k->v = (double)in->dt_raw[tok * H + h] + in->dt_bias[h];
    k->dt = softplus_exact(k->v);
    k->floored = 0;
    if (d->a_per_token) {
        k->a = in->A[tok * H + h];
        if (k->a > -1e-4) { k->a = -1e-4; k->floored = 1; }
    } else {
        k->a = in->A[h];
    }
    k->decay = exp(k->dt * k->a);
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* d silu(v) / dv */
static double silu_grad(double v)
{
    const double s = sigmoid(v);
    return s * (1.0 + v * (1.0 - s));
}

/* Pre-activation of conv channel ch at (b, t) (no initial history: zero-state prefill). */
static double conv_pre(const oracle_dims *d, const oracle_inputs *in, int b, int t, int ch)
{
    const int K = d->dconv;
    double acc = in->conv_b[ch];
    for (int k = 0; k < K; k++) {
        const int tau = t - (K - 1) + k;
        if (tau >= 0 && same_doc(in, d, b, tau, t))
            acc += (double)in->conv_w[(size_t)ch * K + k] * xbc_raw(d, in, b, tau, ch);
    }
    return acc;
}

static void backward_row(const oracle_dims *d, const oracle_inputs *in, const float *gout, int b,
                         const oracle_grads *gr, row_wgrads *wg)
{
    const int L = d->seqlen, P = d->headdim, N = d->dstate, H = d->nheads, G = d->ngroups;
    const int dx = H * P, gn = G * N, cd = conv_dim_of(d), K = d->dconv;
    const int Lb = row_len(d, in, b);
    double *gu = calloc((size_t)L * cd, sizeof(double));     /* gradient of the conv output */
    double *hist = malloc(sizeof(double) * ((size_t)(Lb > 0 ? Lb : 1) * P * N));
    double *gh = malloc(sizeof(double) * (size_t)P * N);
    double *buf = malloc(sizeof(double) * (size_t)(P + 4 * N));
    double *gux = malloc(sizeof(double) * (size_t)P);
    double *gbh = malloc(sizeof(double) * (size_t)N), *gch = malloc(sizeof(double) * (size_t)N);
    if (!gu || !hist || !gh || !buf || !gux || !gbh || !gch) abort();
    tok_terms k;
    k.ux = buf; k.ub = buf + P; k.uc = k.ub + N; k.bh = k.uc + N; k.ch = k.bh + N;

    for (int h = 0; h < H; h++) {
        const int g = h / (H / G);
        /* forward sweep: every state h_t after its update */
        for (int t = 0; t < Lb; t++) {
            token_terms(d, in, b, h, t, &k);
            const int carry = t > 0 && same_doc(in, d, b, t - 1, t);
            double *ht = hist + (size_t)t * P * N;
            for (int p = 0; p < P; p++)
                for (int n = 0; n < N; n++) {
                    const double prev = carry ? hist[((size_t)(t - 1) * P + p) * N + n] : 0.0;
                    ht[p * N + n] = k.decay * prev + k.dt * k.ux[p] * k.bh[n];
                }
        }
        /* reverse sweep */
        memset(gh, 0, sizeof(double) * (size_t)P * N);
        for (int t = Lb - 1; t >= 0; t--) {
            token_terms(d, in, b, h, t, &k);
            const size_t tok = (size_t)b * L + t;
            const int carry = t > 0 && same_doc(in, d, b, t - 1, t);
            const double *ht = hist + (size_t)t * P * N;
            const double *hprev = carry ? hist + (size_t)(t - 1) * P * N : NULL;
            for (int n = 0; n < N; n++) { gbh[n] = 0.0; gch[n] = 0.0; }
            for (int p = 0; p < P; p++) {
                double y = 0.0;
                for (int n = 0; n < N; n++) y += k.ch[n] * ht[p * N + n];
                y += in->D[h] * k.ux[p];
                const double zv = in->z[tok * dx + h * P + p];
                const double go = gout[tok * dx + h * P + p];
                const double gy = go * silu(zv);
                gr->z[tok * dx + h * P + p] = go * y * silu_grad(zv);
                wg->D[h] += gy * k.ux[p];
                gux[p] = gy * in->D[h];
                for (int n = 0; n < N; n++) {
                    gch[n] += gy * ht[p * N + n];
                    gh[p * N + n] += gy * k.ch[n];
                }
            }
            double gdecay = 0.0, gdt = 0.0;
            for (int p = 0; p < P; p++)
                for (int n = 0; n < N; n++) {
                    const double ghv = gh[p * N + n];
                    if (hprev) gdecay += ghv * hprev[p * N + n];
                    gdt += ghv * k.ux[p] * k.bh[n];
                    gux[p] += k.dt * ghv * k.bh[n];
                    gbh[n] += k.dt * ghv * k.ux[p];
                }
            gdt += gdecay * k.decay * k.a;
            const double ga = gdecay * k.decay * k.dt;
            const double gv = gdt * sigmoid(k.v);
            gr->dt_raw[tok * H + h] = gv;
            wg->dt_bias[h] += gv;
            if (d->a_per_token) gr->A[tok * H + h] = k.floored ? 0.0 : ga;
            else wg->A[h] += ga;

            /* B^ / C^ back to the group's conv outputs */
            double *gub = gu + (size_t)t * cd + dx + g * N;
            double *guc = gu + (size_t)t * cd + dx + gn + g * N;
            if (d->bc_norm) {
                double sb = 0.0, sc = 0.0;
                for (int n = 0; n < N; n++) {
                    const double wb = in->bn_w ? in->bn_w[n] : 1.0, wc = in->cn_w ? in->cn_w[n] : 1.0;
                    wg->bn_w[n] += gbh[n] * k.ub[n] * k.rb;
                    wg->cn_w[n] += gch[n] * k.uc[n] * k.rc;
                    wg->bn_bias[(size_t)h * N + n] += gbh[n];
                    wg->cn_bias[(size_t)h * N + n] += gch[n];
                    sb += gbh[n] * wb * k.ub[n];
                    sc += gch[n] * wc * k.uc[n];
                }
                for (int n = 0; n < N; n++) {
                    const double wb = in->bn_w ? in->bn_w[n] : 1.0, wc = in->cn_w ? in->cn_w[n] : 1.0;
                    gub[n] += k.rb * wb * gbh[n] - k.rb * k.rb * k.rb / N * k.ub[n] * sb;
                    guc[n] += k.rc * wc * gch[n] - k.rc * k.rc * k.rc / N * k.uc[n] * sc;
                }
            } else {
                for (int n = 0; n < N; n++) { gub[n] += gbh[n]; guc[n] += gch[n]; }
            }
            for (int p = 0; p < P; p++) gu[(size_t)t * cd + h * P + p] += gux[p];

            /* the adjoint state handed to token t-1 */
            if (carry)
                for (int i = 0; i < P * N; i++) gh[i] *= k.decay;
            else
                memset(gh, 0, sizeof(double) * (size_t)P * N);
        }
    }

    /* conv (+ SiLU) of the row, back to the raw x|B|C inputs */
    double *graw = calloc((size_t)L * cd, sizeof(double));
    if (!graw) abort();
    for (int t = 0; t < Lb; t++)
        for (int ch = 0; ch < cd; ch++) {
            const double gv = gu[(size_t)t * cd + ch];
            if (K == 1) { graw[(size_t)t * cd + ch] += gv; continue; }
            const double gpre = gv * silu_grad(conv_pre(d, in, b, t, ch));
            wg->conv_b[ch] += gpre;
            for (int kk = 0; kk < K; kk++) {
                const int tau = t - (K - 1) + kk;
                if (tau < 0 || !same_doc(in, d, b, tau, t)) continue;
                wg->conv_w[(size_t)ch * K + kk] += gpre * xbc_raw(d, in, b, tau, ch);
                graw[(size_t)tau * cd + ch] += gpre * in->conv_w[(size_t)ch * K + kk];
            }
        }
    for (int t = 0; t < L; t++) {
        const size_t row = (size_t)b * L + t;
        for (int c = 0; c < dx; c++) gr->x[row * dx + c] = graw[(size_t)t * cd + c];
        for (int c = 0; c < gn; c++) {
            gr->Bm[row * gn + c] = graw[(size_t)t * cd + dx + c];
            gr->Cm[row * gn + c] = graw[(size_t)t * cd + dx + gn + c];
        }
    }
    /* padding tokens: nothing reaches them */
    for (int t = Lb; t < L; t++) {
        const size_t tok = (size_t)b * L + t;
        for (int c = 0; c < dx; c++) gr->z[tok * dx + c] = 0.0;
        for (int hh = 0; hh < H; hh++) {
            gr->dt_raw[tok * H + hh] = 0.0;
            if (d->a_per_token) gr->A[tok * H + hh] = 0.0;
        }
    }
    free(gu); free(hist); free(gh); free(buf); free(gux); free(gbh); free(gch); free(graw);
}

typedef struct {
    const oracle_dims *d;
    const oracle_inputs *in;
    const float *gout;
    const oracle_grads *gr;
    row_wgrads *rows;
    int next;
    pthread_mutex_t lock;
} bwd_job;

static void *bwd_worker(void *arg)
{
    bwd_job *j = arg;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        const int b = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (b >= j->d->batch) break;
        backward_row(j->d, j->in, j->gout, b, j->gr, &j->rows[b]);
    }
    return NULL;
}

/* Returns the number of threads used, or -1 on a bad argument. */
int oracle_backward(const oracle_dims *d, const oracle_inputs *in, const float *gout,
                    int nthreads, const oracle_grads *gr)
{
    if (!d || !in || !gout || !gr) return -1;
    if (d->batch < 0 || d->seqlen < 1 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 ||
        d->ngroups < 1 || d->nheads % d->ngroups || d->dconv < 1)
        return -1;
    if (in->init_ssm || in->init_conv) return -1;          /* zero-state prefill only */
    if (d->dconv > 1 && (!in->conv_w || !in->conv_b || !gr->conv_w || !gr->conv_b)) return -1;
    if (d->bc_norm && (!gr->bn_w || !gr->cn_w || !gr->bn_bias || !gr->cn_bias)) return -1;
    if (!gr->x || !gr->z || !gr->Bm || !gr->Cm || !gr->dt_raw || !gr->dt_bias || !gr->A || !gr->D)
        return -1;

    const int H = d->nheads, N = d->dstate, K = d->dconv, cd = conv_dim_of(d);
    /* one block of weight gradients per row: dt_bias, A (per head), D, conv_w, conv_b,
     * bn_w, cn_w, bn_bias, cn_bias */
    const size_t per_row = (size_t)3 * H + (size_t)cd * K + cd + 2 * (size_t)N + 2 * (size_t)H * N;
    const int rows = d->batch > 0 ? d->batch : 1;
    double *pool = calloc(per_row * rows, sizeof(double));
    row_wgrads *rw = malloc(sizeof(row_wgrads) * (size_t)rows);
    if (!pool || !rw) abort();
    for (int b = 0; b < rows; b++) {
        double *q = pool + per_row * b;
        rw[b].dt_bias = q; q += H;
        rw[b].A = q; q += H;
        rw[b].D = q; q += H;
        rw[b].conv_w = q; q += (size_t)cd * K;
        rw[b].conv_b = q; q += cd;
        rw[b].bn_w = q; q += N;
        rw[b].cn_w = q; q += N;
        rw[b].bn_bias = q; q += (size_t)H * N;
        rw[b].cn_bias = q;
    }

    bwd_job j;
    j.d = d; j.in = in; j.gout = gout; j.gr = gr; j.rows = rw; j.next = 0;
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads <= 0) nthreads = oracle_default_threads();
    if (nthreads > d->batch) nthreads = d->batch > 0 ? d->batch : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; i++) pthread_create(&th[i], NULL, bwd_worker, &j);
    bwd_worker(&j);
    for (int i = 1; i < nthreads; i++) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&j.lock);

    /* sum the rows' weight gradients in row order */
    for (int i = 0; i < H; i++) {
        double sbias = 0.0, sa = 0.0, sd = 0.0;
        for (int b = 0; b < d->batch; b++) { sbias += rw[b].dt_bias[i]; sa += rw[b].A[i]; sd += rw[b].D[i]; }
        gr->dt_bias[i] = sbias;
        gr->D[i] = sd;
        if (!d->a_per_token) gr->A[i] = sa;
    }
    if (K > 1) {
        for (size_t i = 0; i < (size_t)cd * K; i++) {
            double s = 0.0;
            for (int b = 0; b < d->batch; b++) s += rw[b].conv_w[i];
            gr->conv_w[i] = s;
        }
        for (int i = 0; i < cd; i++) {
            double s = 0.0;
            for (int b = 0; b < d->batch; b++) s += rw[b].conv_b[i];
            gr->conv_b[i] = s;
        }
    }
    if (d->bc_norm) {
        for (int i = 0; i < N; i++) {
            double sb = 0.0, sc = 0.0;
            for (int b = 0; b < d->batch; b++) { sb += rw[b].bn_w[i]; sc += rw[b].cn_w[i]; }
            gr->bn_w[i] = sb;
            gr->cn_w[i] = sc;
        }
        for (size_t i = 0; i < (size_t)H * N; i++) {
            double sb = 0.0, sc = 0.0;
            for (int b = 0; b < d->batch; b++) { sb += rw[b].bn_bias[i]; sc += rw[b].cn_bias[i]; }
            gr->bn_bias[i] = sb;
            gr->cn_bias[i] = sc;
        }
    }
    free(pool); free(rw);
    return nthreads;
}

/* ------------------------------------------------------------------------------------
 * Gated RMSNorm after the scan: upstream Mamba-2's norm(y * silu(z)) with the
 * weight mixer.norm.weight of shape (d_inner) -- codestral_mamba.ts weight-port
 * header (tensor list, and reconciliation 3: upstream computes
 * "norm(y * silu(z))").  The gated product y * silu(z) is exactly what
 * oracle_forward returns as out, so this step takes that output:
 *
 *   for each token row and each group of `group` consecutive channels
 *   (group == d_inner: one norm over the whole row):
 *     r = 1 / sqrt(mean over the group of g^2 + eps);   out[c] = g[c] * r * w[c]
 *
 * g, out: (rows, d_inner) double (may alias); w: (d_inner) float32 or NULL
 * (ones).  Returns 0, or -1 on a bad argument.
 */
int oracle_gated_norm(int rows, int d_inner, int group, double eps, const double *g,
                      const float *w, double *out)
{
    if (rows < 0 || d_inner < 1 || group < 1 || d_inner % group || !(eps >= 0.0) || !g || !out)
        return -1;
    for (int r = 0; r < rows; r++)
        for (int c0 = 0; c0 < d_inner; c0 += group) {
            const double *gv = g + (size_t)r * d_inner + c0;
            double ss = 0.0;
            for (int c = 0; c < group; c++) ss += gv[c] * gv[c];
            const double rs = 1.0 / sqrt(ss / group + eps);
            for (int c = 0; c < group; c++)
                out[(size_t)r * d_inner + c0 + c] = gv[c] * rs * (w ? w[c0 + c] : 1.0);
        }
    return 0;
}
