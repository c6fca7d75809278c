/*
 * gdn_oracle.c -- plain, slow, sequential fp64 CPU statement of the Gated
 * DeltaNet (GDN) forward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg use it; the CUDA library never
 * links, calls or includes it, and it includes nothing of the CUDA library.
 *
 * What it computes.  The LinMorph project page (Abstract; "Why learn the
 * initialization?") replaces softmax self-attention in a video DiT with a
 * Gated DeltaNet module whose parameters are "update gates, decay terms, short
 * convolutions, and normalization parameters".  The recurrence itself is the
 * gated delta rule of Yang, Kautz and Hatamizadeh, "Gated Delta Networks:
 * Improving Mamba2 with Delta Rule" (reference [57] on the VMonarch page,
 * References).  Written out, per batch item b and head h, over the
 * frame-major token sequence t = 0..T-1:
 *
 *   1. short conv:  u_t[i] = sum_{j=0..3} w[h*d+i][j] * x_{t-3+j}[i]
 *                   (x_{<0} = 0, restart per batch item), then SiLU,
 *                   separately for q, k and v;
 *   2. q^ = q'/sqrt(|q'|^2 + eps_l2), k^ likewise; v^ = v' (not normalised);
 *   3. alpha_t = exp(-exp(A_log[h]) * softplus(g_t + dt_bias[h])),
 *      beta_t  = sigmoid(b_t);
 *   4. S_t = alpha_t * S_{t-1} (I - beta_t k^_t k^_t^T) + beta_t v^_t k^_t^T,
 *      S_{-1} = 0 (d_v x d_k), and o_t = S_t q^_t / sqrt(d_k);
 *   5. y_t = o_t / sqrt(mean(o_t^2) + eps_rms) * w_norm * SiLU(z_t).
 *
 * Every step is the literal definition, in fp64, in the order above: no
 * chunking, no blocking, no reordering.  Where the definition is silent the
 * readings are: conv tap 3 multiplies the current token (cross-correlation
 * with left zero padding 3, no bias); SiLU before the L2 norm; the scale
 * 1/sqrt(d_k) on the output; o_t uses the state after token t's update;
 * softplus(x) = max(x,0) + log1p(exp(-|x|)).
 *
 * Layouts: activations [B][T][H][d] (token-major, heads interleaved), gates
 * [B][T][H], conv weights [H*d][4], A_log and dt_bias [H], norm weight [d_v].
 * Inputs arrive as fp32 (bf16 inputs widened exactly by the caller); every
 * intermediate and output is fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

static double silu(double u) { return u / (1.0 + exp(-u)); }

static double softplus(double x) { return (x > 0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* Step 1: causal depthwise short convolution (kernel 4) followed by SiLU.
 * LinMorph project page, "Why learn the initialization?" ("short
 * convolutions"). */
void oracle_conv_silu(int B, int T, int H, int d, const float *x, const float *w, double *out)
{
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h)
                for (int i = 0; i < d; ++i) {
                    const int c = h * d + i;
                    double u = 0.0;
                    for (int j = 0; j < 4; ++j) {
                        const int s = t - 3 + j;
                        if (s < 0) continue;
                        u += (double)w[(size_t)c * 4 + j] *
                             (double)x[(((size_t)b * T + s) * H + h) * d + i];
                    }
                    out[(((size_t)b * T + t) * H + h) * d + i] = silu(u);
                }
}

/* Step 2: L2 normalisation of each d-vector, in place (the q and k
 * "normalization" of the GDN module; LinMorph page, same section). */
void oracle_l2norm(long long n_vec, int d, double eps, double *x)
{
    for (long long n = 0; n < n_vec; ++n) {
        double *v = x + (size_t)n * d;
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += v[i] * v[i];
        const double inv = 1.0 / sqrt(ss + eps);
        for (int i = 0; i < d; ++i) v[i] *= inv;
    }
}

/* Step 3: decay term alpha and update gate beta per (b, t, h) (the "decay
 * terms" and "update gates" of the LinMorph page, same section). */
void oracle_gates(int B, int T, int H, const float *g, const float *bgate,
                  const float *A_log, const float *dt_bias, double *alpha, double *beta)
{
    for (size_t n = 0; n < (size_t)B * T; ++n)
        for (int h = 0; h < H; ++h) {
            const size_t idx = n * H + h;
            const double a = exp((double)A_log[h]);
            alpha[idx] = exp(-a * softplus((double)g[idx] + (double)dt_bias[h]));
            beta[idx] = 1.0 / (1.0 + exp(-(double)bgate[idx]));
        }
}

/* Step 4 for one (b, h): the gated delta-rule recurrence, token by token
 * (Gated Delta Networks, reference [57] on the VMonarch page).  S is kept
 * d_v x d_k, row-major.  s0 (may be NULL = zero) is the state before token 0;
 * s_end (may be NULL) receives the state after the last token. */
static void core_one(int T, int H, int h, int dk, int dv, size_t bT,
                     const double *qh, const double *kh, const double *vh,
                     const double *alpha, const double *beta, double *o,
                     const double *s0, double *s_end)
{
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *Sk = (double *)malloc((size_t)dv * sizeof(double));
    if (s0) memcpy(S, s0, (size_t)dv * dk * sizeof(double));
    const double scale = 1.0 / sqrt((double)dk);
    for (int t = 0; t < T; ++t) {
        const size_t row = (bT + t) * H + h;
        const double *k = kh + row * dk, *q = qh + row * dk, *v = vh + row * dv;
        const double a = alpha[row], be = beta[row];
        /* S k */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * k[j];
            Sk[i] = acc;
        }
        /* S <- a * S (I - be k k^T) + be v k^T = a * (S - be (S k) k^T) + be v k^T */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) {
                double *s = &S[(size_t)i * dk + j];
                *s = a * (*s - be * Sk[i] * k[j]) + be * v[i] * k[j];
            }
        /* o_t = S_t q_t / sqrt(d_k) */
        double *ot = o + row * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * q[j];
            ot[i] = acc * scale;
        }
    }
    if (s_end) memcpy(s_end, S, (size_t)dv * dk * sizeof(double));
    free(Sk);
    free(S);
}

typedef struct {
    int B, T, H, dk, dv;
    const double *qh, *kh, *vh, *alpha, *beta;
    double *o;
    const double *s0;
    double *s_end;
    int first, stride;
} core_job;

static void *core_worker(void *arg)
{
    core_job *j = (core_job *)arg;
    const size_t ss = (size_t)j->dv * j->dk;
    for (int bh = j->first; bh < j->B * j->H; bh += j->stride) {
        const int b = bh / j->H, h = bh % j->H;
        core_one(j->T, j->H, h, j->dk, j->dv, (size_t)b * j->T, j->qh, j->kh, j->vh,
                 j->alpha, j->beta, j->o, j->s0 ? j->s0 + (size_t)bh * ss : NULL,
                 j->s_end ? j->s_end + (size_t)bh * ss : NULL);
    }
    return NULL;
}

/* Step 4 for all (b, h), one pthread per (b, h) group.  q^, k^ must already be
 * normalised by the caller if the full method is wanted; the core itself
 * applies only the recurrence and the 1/sqrt(d_k) output scale.  s0/s_end are
 * [B][H][d_v][d_k] or NULL. */
void oracle_core(int B, int T, int H, int dk, int dv, const double *qh, const double *kh,
                 const double *vh, const double *alpha, const double *beta, double *o,
                 const double *s0, double *s_end, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * H) nthreads = B * H;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    core_job *jobs = (core_job *)malloc(sizeof(core_job) * nthreads);
    for (int n = 0; n < nthreads; ++n) {
        core_job j = {B, T, H, dk, dv, qh, kh, vh, alpha, beta, o, s0, s_end, n, nthreads};
        jobs[n] = j;
        pthread_create(&th[n], NULL, core_worker, &jobs[n]);
    }
    for (int n = 0; n < nthreads; ++n) pthread_join(th[n], NULL);
    free(jobs);
    free(th);
}

/* Step 5: RMSNorm over d_v, times the norm weight, times SiLU(z) (the
 * "normalization parameters" of the GDN module; LinMorph page, same
 * section). */
void oracle_output(long long n_vec, int dv, const double *o, const float *z,
                   const float *norm_w, double eps, double *y)
{
    for (long long n = 0; n < n_vec; ++n) {
        const double *ov = o + (size_t)n * dv;
        const float *zv = z + (size_t)n * dv;
        double ms = 0.0;
        for (int i = 0; i < dv; ++i) ms += ov[i] * ov[i];
        const double r = 1.0 / sqrt(ms / dv + eps);
        for (int i = 0; i < dv; ++i)
            y[(size_t)n * dv + i] = ov[i] * r * (double)norm_w[i] * silu((double)zv[i]);
    }
}

/* Steps 1-5 composed.  Optional intermediate outputs (any may be NULL):
 * qh, kh, vh [B][T][H][d] after conv+SiLU(+L2), alpha, beta [B][T][H],
 * o [B][T][H][d_v] before the output norm.  Returns 0, or -1 when out of
 * memory. */
int oracle_forward(int B, int T, int H, int dk, int dv,
                   const float *q, const float *k, const float *v, const float *z,
                   const float *g, const float *bgate,
                   const float *conv_q, const float *conv_k, const float *conv_v,
                   const float *A_log, const float *dt_bias, const float *norm_w,
                   double l2_eps, double norm_eps, int nthreads,
                   double *y, double *qh_out, double *kh_out, double *vh_out,
                   double *alpha_out, double *beta_out, double *o_out)
{
    const size_t nk = (size_t)B * T * H * dk, nv = (size_t)B * T * H * dv, ng = (size_t)B * T * H;
    double *qh = qh_out ? qh_out : (double *)malloc(nk * sizeof(double));
    double *kh = kh_out ? kh_out : (double *)malloc(nk * sizeof(double));
    double *vh = vh_out ? vh_out : (double *)malloc(nv * sizeof(double));
    double *al = alpha_out ? alpha_out : (double *)malloc(ng * sizeof(double));
    double *be = beta_out ? beta_out : (double *)malloc(ng * sizeof(double));
    double *o = o_out ? o_out : (double *)malloc(nv * sizeof(double));
    int rc = 0;
    if (!qh || !kh || !vh || !al || !be || !o) { rc = -1; goto done; }
    oracle_conv_silu(B, T, H, dk, q, conv_q, qh);
    oracle_conv_silu(B, T, H, dk, k, conv_k, kh);
    oracle_conv_silu(B, T, H, dv, v, conv_v, vh);
    oracle_l2norm((long long)B * T * H, dk, l2_eps, qh);
    oracle_l2norm((long long)B * T * H, dk, l2_eps, kh);
    oracle_gates(B, T, H, g, bgate, A_log, dt_bias, al, be);
    oracle_core(B, T, H, dk, dv, qh, kh, vh, al, be, o, NULL, NULL, nthreads);
    oracle_output((long long)B * T * H, dv, o, z, norm_w, norm_eps, y);
done:
    if (!qh_out) free(qh);
    if (!kh_out) free(kh);
    if (!vh_out) free(vh);
    if (!alpha_out) free(al);
    if (!beta_out) free(be);
    if (!o_out) free(o);
    return rc;
}
