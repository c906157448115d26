/*
 * ssd_oracle.c -- plain, slow, fp64 CPU oracle of the Mamba-2 mixer core.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the correctness oracle for the CUDA
 * library in hybrid_mamba_ssm_causal_b200/. Only tests/, the smoke check in
 * __graft_entry__.py and the cpu_baseline / reference leg of bench.py may load
 * it. It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes: everything between in_proj and out_proj of a Nemotron-H
 * Mamba-2 layer: its causal conv, its selective state-space scan and its gated norm
 * that the mixer table of gllm PR #86 "feat(model): Nemotron-H hybrid (Mamba2 +
 * attention + MoE) on the CPU" (section "2. feat(model): Nemotron-H on the CPU",
 * row M) places between the two projections:
 *
 *   1. xBC = [x | B | C] on the channel axis (the fused projection's output row
 *      holds z, then x, B and C, then dt -- same PR, "Supporting changes";
 *      Modalities PR #459, notes on the packed projection layout).
 *   2. Depthwise causal conv of width K over time, per channel c:
 *        s    = [init_conv[c][0..K-2] (oldest first), xBC[0..L-1][c]]
 *        v[t] = conv_b[c] + sum_{k=0}^{K-1} conv_w[c][k] * s[t+k]
 *        xBC'[t][c] = SiLU(v[t]) = v / (1 + exp(-v))
 *      final_conv[c][k] = s[L+k], k = 0..K-2 (the last K-1 raw inputs).
 *   3. delta[t][h] = softplus(dt[t][h] + dt_bias[h]), softplus(u) = log(1+e^u).
 *   4. For each head h, with group g = h / (H/G) sharing B and C:
 *        h_t = exp(delta_t * A_h) * h_{t-1} + delta_t * x'_t (outer) B'_t
 *        y_t = h_t . C'_t + D_h * x'_t
 *      (the sequential Mamba-2 recurrence that the Modalities PR's section
 *      "Testing" validates its chunked scan against, and that gllm's scan is,
 *      per the gllm PR's "Reference quirk" paragraph). final_ssm = h_L.
 *   5. Gated group RMSNorm: gate = y * SiLU(z); for every token and every
 *      contiguous group of H*P/G channels,
 *        out = gate / sqrt(mean(gate^2) + eps) * norm_w.
 *
 * Readings taken where the pages are silent (listed with reasons in the
 * design notes): gate before normalising; norm group = H*P/G contiguous
 * channels; head h uses group h / (H/G); D and A are scalars per head and A
 * arrives already negative; no clamp on delta; conv state holds the last K-1
 * raw inputs, oldest first.
 *
 * Layouts (all fp64, contiguous, row-major):
 *   x, z, y, y_pre [b][L][H*P]     B, C [b][L][G*N]     dt, delta [b][L][H]
 *   xbc_act [b][L][H*P + 2*G*N]    conv_w [Cc][K]       conv_b [Cc]
 *   A, D, dt_bias [H]   norm_w [H*P]   ssm states [b][H][P][N]
 *   conv states [b][Cc][K-1]
 * The problem separates by (batch row, group): every unit owns its group's
 * heads, x channels, B and C channels and norm group. Units run on a few
 * pthreads; the arithmetic inside a unit is the plain definition above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t batch, seqlen;
    int32_t nheads, headdim, ngroups, dstate, dconv;
    double eps;
} ssd_oracle_dims;

typedef struct {
    const ssd_oracle_dims* d;
    const double *x, *z, *Bm, *Cm, *dt;
    const double *A, *D, *conv_w, *conv_b, *dt_bias, *norm_w;
    const double *init_ssm, *init_conv;
    double *y, *final_ssm, *final_conv;
    double *xbc_act, *delta, *y_pre;
    int64_t nunits;
    int64_t next_unit; /* shared work counter */
    int failed;
} oracle_job;

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* log(1 + e^u) written so that neither branch overflows. */
static double softplus(double u) { return (u > 0.0 ? u : 0.0) + log1p(exp(-fabs(u))); }

/* Causal depthwise conv + SiLU of one channel over the whole sequence.
 * u: input channel, element t at u[t*ustride]. init: K-1 taps or NULL.
 * act: output, element t at act[t*astride]. fin: K-1 final taps (may be NULL). */
static void conv_channel(int64_t L, int K, const double* u, int64_t ustride, const double* init,
                         const double* w, double bias, double* act, int64_t astride, double* fin)
{
    /* s has L + K - 1 entries: K-1 from the initial state, then the inputs. */
    double* s = (double*)malloc(sizeof(double) * (size_t)(L + K - 1));
    for (int k = 0; k < K - 1; ++k) s[k] = init ? init[k] : 0.0;
    for (int64_t t = 0; t < L; ++t) s[K - 1 + t] = u[t * ustride];
    for (int64_t t = 0; t < L; ++t) {
        double v = bias;
        for (int k = 0; k < K; ++k) v += w[k] * s[t + k];
        act[t * astride] = silu(v);
    }
    if (fin)
        for (int k = 0; k < K - 1; ++k) fin[k] = s[L + k];
    free(s);
}

static int run_unit(oracle_job* j, int64_t b, int g)
{
    const ssd_oracle_dims* d = j->d;
    const int64_t L = d->seqlen;
    const int H = d->nheads, P = d->headdim, G = d->ngroups, N = d->dstate, K = d->dconv;
    const int r = H / G;          /* heads per group */
    const int64_t HP = (int64_t)H * P, GN = (int64_t)G * N, Cc = HP + 2 * GN;
    const int64_t gw = (int64_t)r * P; /* channels of this group's heads = norm group size */
    const int64_t xc0 = (int64_t)g * gw;          /* first x channel of the group */
    const int64_t bc0 = HP + (int64_t)g * N;      /* first B channel in xBC */
    const int64_t cc0 = HP + GN + (int64_t)g * N; /* first C channel in xBC */

    double* xa = (double*)malloc(sizeof(double) * (size_t)(L * gw));  /* x' [L][gw] */
    double* Ba = (double*)malloc(sizeof(double) * (size_t)(L * N));   /* B' [L][N] */
    double* Ca = (double*)malloc(sizeof(double) * (size_t)(L * N));   /* C' [L][N] */
    double* dl = (double*)malloc(sizeof(double) * (size_t)(L * r));   /* delta [L][r] */
    double* yp = (double*)malloc(sizeof(double) * (size_t)(L * gw));  /* y before the norm */
    double* hs = (double*)malloc(sizeof(double) * (size_t)P * N);     /* one head's state */
    if (!xa || !Ba || !Ca || !dl || !yp || !hs) {
        free(xa); free(Ba); free(Ca); free(dl); free(yp); free(hs);
        return -1;
    }

    /* 1-2. conv + SiLU over the group's x, B and C channels. */
    const double* xrow = j->x + b * L * HP;
    const double* Brow = j->Bm + b * L * GN;
    const double* Crow = j->Cm + b * L * GN;
    const double* ic = j->init_conv ? j->init_conv + b * Cc * (K - 1) : NULL;
    double* fc = j->final_conv ? j->final_conv + b * Cc * (K - 1) : NULL;
    for (int64_t c = 0; c < gw; ++c) {
        const int64_t ch = xc0 + c;
        conv_channel(L, K, xrow + ch, HP, ic ? ic + ch * (K - 1) : NULL, j->conv_w + ch * K,
                     j->conv_b[ch], xa + c, gw, fc ? fc + ch * (K - 1) : NULL);
    }
    for (int n = 0; n < N; ++n) {
        const int64_t chb = bc0 + n, chc = cc0 + n;
        conv_channel(L, K, Brow + (int64_t)g * N + n, GN, ic ? ic + chb * (K - 1) : NULL,
                     j->conv_w + chb * K, j->conv_b[chb], Ba + n, N, fc ? fc + chb * (K - 1) : NULL);
        conv_channel(L, K, Crow + (int64_t)g * N + n, GN, ic ? ic + chc * (K - 1) : NULL,
                     j->conv_w + chc * K, j->conv_b[chc], Ca + n, N, fc ? fc + chc * (K - 1) : NULL);
    }
    if (j->xbc_act) {
        double* o = j->xbc_act + b * L * Cc;
        for (int64_t t = 0; t < L; ++t) {
            for (int64_t c = 0; c < gw; ++c) o[t * Cc + xc0 + c] = xa[t * gw + c];
            for (int n = 0; n < N; ++n) {
                o[t * Cc + bc0 + n] = Ba[t * N + n];
                o[t * Cc + cc0 + n] = Ca[t * N + n];
            }
        }
    }

    /* 3. delta = softplus(dt + dt_bias) for the group's heads. */
    for (int64_t t = 0; t < L; ++t)
        for (int i = 0; i < r; ++i) {
            const int h = g * r + i;
            dl[t * r + i] = softplus(j->dt[(b * L + t) * H + h] + j->dt_bias[h]);
            if (j->delta) j->delta[(b * L + t) * H + h] = dl[t * r + i];
        }

    /* 4. the sequential recurrence, one head at a time. */
    for (int i = 0; i < r; ++i) {
        const int h = g * r + i;
        const double Ah = j->A[h], Dh = j->D[h];
        const int64_t soff = ((b * H) + h) * (int64_t)P * N;
        if (j->init_ssm) memcpy(hs, j->init_ssm + soff, sizeof(double) * (size_t)P * N);
        else memset(hs, 0, sizeof(double) * (size_t)P * N);
        for (int64_t t = 0; t < L; ++t) {
            const double dlt = dl[t * r + i];
            const double decay = exp(dlt * Ah);
            const double* xt = xa + t * gw + (int64_t)i * P;
            const double* Bt = Ba + t * N;
            const double* Ct = Ca + t * N;
            for (int p = 0; p < P; ++p) {
                double yv = 0.0;
                double* hp = hs + (int64_t)p * N;
                for (int n = 0; n < N; ++n) {
                    hp[n] = decay * hp[n] + dlt * xt[p] * Bt[n];
                    yv += hp[n] * Ct[n];
                }
                yp[t * gw + (int64_t)i * P + p] = yv + Dh * xt[p];
            }
        }
        if (j->final_ssm) memcpy(j->final_ssm + soff, hs, sizeof(double) * (size_t)P * N);
    }

    /* 5. gate, then RMS-normalise over the group's channels. */
    for (int64_t t = 0; t < L; ++t) {
        const double* zt = j->z + (b * L + t) * HP + xc0;
        double* yt = j->y + (b * L + t) * HP + xc0;
        double ss = 0.0;
        for (int64_t c = 0; c < gw; ++c) {
            const double gate = yp[t * gw + c] * silu(zt[c]);
            yt[c] = gate;
            ss += gate * gate;
        }
        const double inv = 1.0 / sqrt(ss / (double)gw + d->eps);
        for (int64_t c = 0; c < gw; ++c) yt[c] = yt[c] * inv * j->norm_w[xc0 + c];
        if (j->y_pre)
            for (int64_t c = 0; c < gw; ++c) j->y_pre[(b * L + t) * HP + xc0 + c] = yp[t * gw + c];
    }

    free(xa); free(Ba); free(Ca); free(dl); free(yp); free(hs);
    return 0;
}

static void* worker(void* arg)
{
    oracle_job* j = (oracle_job*)arg;
    for (;;) {
        const int64_t u = __atomic_fetch_add(&j->next_unit, 1, __ATOMIC_RELAXED);
        if (u >= j->nunits) break;
        if (run_unit(j, u / j->d->ngroups, (int)(u % j->d->ngroups)) != 0)
            __atomic_store_n(&j->failed, 1, __ATOMIC_RELAXED);
    }
    return NULL;
}

/* Returns 0 on success, -1 on bad dims, -2 on allocation failure.
 * init_ssm / init_conv may be NULL (zeros). final_* / xbc_act / delta / y_pre
 * may be NULL (not produced). nthreads <= 0 means 1. */
int ssd_oracle_prefill(const ssd_oracle_dims* d, const double* x, const double* z,
                       const double* Bm, const double* Cm, const double* dt, const double* A,
                       const double* D, const double* conv_w, const double* conv_b,
                       const double* dt_bias, const double* norm_w, const double* init_ssm,
                       const double* init_conv, double* y, double* final_ssm,
                       double* final_conv, double* xbc_act, double* delta, double* y_pre,
                       int nthreads)
{
    if (!d || d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->headdim <= 0 ||
        d->ngroups <= 0 || d->dstate <= 0 || d->dconv < 1 || d->nheads % d->ngroups != 0)
        return -1;
    oracle_job j;
    memset(&j, 0, sizeof(j));
    j.d = d;
    j.x = x; j.z = z; j.Bm = Bm; j.Cm = Cm; j.dt = dt;
    j.A = A; j.D = D; j.conv_w = conv_w; j.conv_b = conv_b; j.dt_bias = dt_bias; j.norm_w = norm_w;
    j.init_ssm = init_ssm; j.init_conv = init_conv;
    j.y = y; j.final_ssm = final_ssm; j.final_conv = final_conv;
    j.xbc_act = xbc_act; j.delta = delta; j.y_pre = y_pre;
    j.nunits = d->batch * d->ngroups;
    if (nthreads <= 0) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads == 1 || j.nunits <= 1) {
        worker(&j);
    } else {
        pthread_t th[256];
        int started = 0;
        for (int i = 0; i < nthreads; ++i)
            if (pthread_create(&th[i], NULL, worker, &j) == 0) ++started;
        if (started == 0) worker(&j);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    }
    return j.failed ? -2 : 0;
}
