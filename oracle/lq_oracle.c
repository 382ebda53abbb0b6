/*
 * lq_oracle.c -- plain, slow CPU oracle for windowed low-bit recurrent-state
 * decode of delta-rule linear attention (Gated DeltaNet and KDA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg load this library.  It shares no code, no
 * header and no constant table with the CUDA library; it reads plain host
 * arrays and writes plain host arrays.
 *
 * Precision: all floating-point arithmetic is double, except the steps that
 * turn a value into an integer code (x = R/m, s = a/qmax, code = rne(x/s)),
 * which are taken in float, the precision the CUDA kernels decide them in.
 * Stored quantities that the method keeps in float (compensator vectors,
 * scales, the residual handed to the quantizer) are rounded to float at the
 * point where they are stored.  Built with -ffp-contract=off so that every
 * expression is evaluated as written.
 *
 * Sources (page title, then the place on that page):
 *  [Table3]  "LinQuant: Functional Invariances for Low-Precision Linear
 *            Recurrences", appendix Table 3 (state-update rules): Gated
 *            DeltaNet S_t = a_t S_{t-1}(I - b_t k k^T) + b_t v k^T and KDA
 *            S_t = S_{t-1} diag(a_t)(I - b_t k k^T) + b_t v k^T, with S in
 *            (d_v x d_k) form.  Here S is kept transposed (d_k x d_v, key rows,
 *            value columns), which gives S_t = (I - b k k^T) D_t S_{t-1} + b k v^T.
 *  [Leap-W]  "LeapQuant: Efficient Linear Attention with Accurate Recurrent
 *            State Quantization" (project page), paragraph on leaping over a
 *            window: low-bit state at the window start, held fixed, buffered
 *            higher-precision token updates, one reconstruct + quantize at the
 *            window end.
 *  [Leap-C]  same page, Compensator Tokens paragraph: a few high-precision
 *            rank-one outer products hold the largest outliers; they take the
 *            real tokens' update path.
 *  [Leap-S]  same page, smoothing paragraph: after the compensators are removed
 *            the residual's key-row magnitudes are balanced before quantizing;
 *            the scales are recomputed at every window boundary.
 *  [STEP]    "How does STEPQuant compress recurrent states without losing
 *            accuracy?", key-row and value-column scales.
 *  [DAMP]    "DAMP: Decay-Aware Mixed-Precision Recurrent-State Quantization",
 *            abstract: high-risk channels chosen offline by quantization-error
 *            energy and decay persistence are stored at higher precision.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - quantizer: symmetric, no zero point, codes in [-qmax, qmax], round half
 *    to even, one scale per value column s_c = amax_c / qmax of the smoothed
 *    residual, one smoothing scale per key row m_i = RMS of row i.  The b-bit
 *    state (b = 8, 6 or 4: the LeapQuant page's 8-, 6- and 4-bit rows of its
 *    results table) takes qmax = 2^(b-1) - 1 = 127, 31 or 7; the most
 *    negative code of each width is left unused, as for INT8.
 *  - compensators: power iteration on the residual, start w = 1/sqrt(d_v),
 *    K steps of z = R w / |R w|, w = R^T z / |R^T z|; then c = R w and
 *    R <- R - c w^T; repeated r times (deflation).  A zero norm gives a zero
 *    compensator.
 *  - output o_t = S_t^T q_t from the updated state, no 1/sqrt(d_k).
 *  - the flush happens after the W-th token's output; none at the run's end
 *    unless asked.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int dk, dv;
    int gate;      /* 0: one decay per head (GDN); 1: one per key channel (KDA) */
    int W;         /* window length */
    int r;         /* compensator tokens */
    int K;         /* power-iteration steps per compensator */
    int smoothing; /* 1: per-row RMS smoothing; 0: m_i = 1 */
    int P;         /* BF16 key rows per head (DAMP); 0 = none */
    int quantize;  /* 0: identity quantizer (FP32-state mode); 1: INT8 */
    int bf16_buffer; /* 1: each token's update is kept in BF16 (see lqo_step_bf16) */
    int bits;      /* code width of the quantized state: 8 (0 reads as 8), 6 or 4 */
    /* smoothing == 2 (static, fitted offline; see lqo_fit_static): the
     * head's key-row scales [dk] and value-column scales [dv] (lqo_run: the
     * arrays of all heads, [nh][dk] and [nh][dv]) */
    const float *static_m;
    const float *static_s;
} lqo_cfg;

/* Largest code magnitude of a b-bit symmetric quantizer. */
static int lqo_qmax(const lqo_cfg *cfg)
{
    const int b = cfg->bits == 0 ? 8 : cfg->bits;
    return (1 << (b - 1)) - 1;
}

/* A quantized view of one head.  codes are [dk][dv] with the BF16 rows' codes
 * left at 0; hp holds the BF16 rows in the order of hp_rows. */
typedef struct {
    int8_t *codes;    /* [dk*dv] */
    float *m;         /* [dk]   smoothing scale per key row (1 on BF16 rows) */
    float *s;         /* [dv]   quantization scale per value column */
    float *c;         /* [r*dk] compensator key-side vectors */
    float *w;         /* [r*dv] compensator value-side vectors */
    uint16_t *hp;     /* [P*dv] BF16 rows (bit patterns) */
} lqo_view;

/* ------------------------------------------------------------------ */
/* Recurrence [Table3].                                                */
/* ------------------------------------------------------------------ */

/* One token: S <- (I - beta k k^T) D S + beta k v^T ;  o = S^T q.
 * Evaluated as S' = D S, y = S'^T k, u = beta (v - y), S = S' + k u^T, which is
 * the same product expanded (the projection applied to D S). */
void lqo_step(const lqo_cfg *cfg, double *S, const float *q, const float *k,
              const float *v, float beta, const float *alpha, double *o)
{
    const int dk = cfg->dk, dv = cfg->dv;
    double *u = (double *)malloc(sizeof(double) * dv);
    for (int i = 0; i < dk; ++i) {
        const double d = cfg->gate ? (double)alpha[i] : (double)alpha[0];
        for (int c = 0; c < dv; ++c) S[i * dv + c] *= d;
    }
    for (int c = 0; c < dv; ++c) {
        double y = 0.0;
        for (int i = 0; i < dk; ++i) y += (double)k[i] * S[i * dv + c];
        u[c] = (double)beta * ((double)v[c] - y);
    }
    for (int i = 0; i < dk; ++i)
        for (int c = 0; c < dv; ++c) S[i * dv + c] += (double)k[i] * u[c];
    for (int c = 0; c < dv; ++c) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[i * dv + c] * (double)q[i];
        o[c] = acc;
    }
    free(u);
}

/* ------------------------------------------------------------------ */
/* Quantizer Q and its inverse [Leap-C], [Leap-S], [STEP], [DAMP].      */
/* ------------------------------------------------------------------ */

uint16_t lqo_bf16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float lqo_bf16_to_float(uint16_t h)
{
    const uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* The window's decay product as the BF16 buffer keys against it: an FP32
 * significand chain G_t = a_t G_{t-1} whose exponent is kept apart -- when the
 * product falls below 2^-64 it is taken as (a_t 2^64) G_{t-1} instead (the
 * same rounding, 64 binades up), and when even that is below 2^-64 (one
 * token's decay under 2^-128) the chain restarts at 1.  Only the rounding
 * of k / G depends on it: the token's contribution is G bf16(k / G), so the
 * exponent kept apart cancels, and the state itself decays exactly (in
 * double).  Reading of the BF16-buffer option for decays whose product leaves
 * the FP32 range (the pages store the buffered updates in higher precision
 * and say nothing of a decay's range). */
static float lqo_gate_chain(float a, float g)
{
    float p = a * g;
    if (p >= 0.0f && p < 0x1p-64f) {
        p = (a * 0x1p64f) * g;
        if (!(p >= 0x1p-64f)) p = 1.0f;
    }
    return p;
}

/* One token with the window's buffered updates kept in BF16 (the
 * traffic-lean buffer): as lqo_step, except that the rank-one update enters
 * the state rounded, the way the windowed kernels store it -- the key side
 * divided by the window's decay so far, ktil = k / G_t, and the value side
 * u, each rounded to BF16 (round to nearest even) from FP32:
 *     S <- S' + (G_t * bf16(ktil)) bf16(u)^T,   o = S^T q.
 * G_t (per key row for KDA, one value for GDN) is the decay chain of
 * lqo_gate_chain carried in FP32 in gam[] (1 at the window start), and ktil
 * and u are formed in FP32 before rounding: BF16 rounding decides the stored
 * bits, so it is taken in the kernels' precision. */
void lqo_step_bf16(const lqo_cfg *cfg, double *S, float *gam, const float *q, const float *k,
                   const float *v, float beta, const float *alpha, double *o)
{
    const int dk = cfg->dk, dv = cfg->dv, ga = cfg->gate ? dk : 1;
    double *u = (double *)malloc(sizeof(double) * dv);
    double *kg = (double *)malloc(sizeof(double) * dk);
    for (int j = 0; j < ga; ++j) gam[j] = lqo_gate_chain(alpha[j], gam[j]);
    for (int i = 0; i < dk; ++i) {
        const double d = cfg->gate ? (double)alpha[i] : (double)alpha[0];
        for (int c = 0; c < dv; ++c) S[i * dv + c] *= d;
    }
    for (int c = 0; c < dv; ++c) {
        double y = 0.0;
        for (int i = 0; i < dk; ++i) y += (double)k[i] * S[i * dv + c];
        const float uf = (float)((double)beta * ((double)v[c] - y));
        u[c] = (double)lqo_bf16_to_float(lqo_bf16_rne(uf));
    }
    for (int i = 0; i < dk; ++i) {
        const float g = cfg->gate ? gam[i] : gam[0];
        const float kt = k[i] / g;
        kg[i] = (double)g * (double)lqo_bf16_to_float(lqo_bf16_rne(kt));
    }
    for (int i = 0; i < dk; ++i)
        for (int c = 0; c < dv; ++c) S[i * dv + c] += kg[i] * u[c];
    for (int c = 0; c < dv; ++c) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[i * dv + c] * (double)q[i];
        o[c] = acc;
    }
    free(u);
    free(kg);
}

static int is_hp_row(const int *hp_rows, int P, int i)
{
    for (int p = 0; p < P; ++p)
        if (hp_rows[p] == i) return 1;
    return 0;
}

/* Q: float state S [dk][dv] -> view.  `ratio` (nullable, [dk*dv]) receives
 * the exact quotient x/s (as double) behind every code, for tie analysis. */
void lqo_quantize(const lqo_cfg *cfg, const int *hp_rows, const float *S,
                  lqo_view *out, double *ratio)
{
    const int dk = cfg->dk, dv = cfg->dv, r = cfg->r, P = cfg->P;
    double *R = (double *)malloc(sizeof(double) * dk * dv);
    double *z = (double *)malloc(sizeof(double) * dk);
    double *w = (double *)malloc(sizeof(double) * dv);
    float *R32 = (float *)malloc(sizeof(float) * dk * dv);
    float *x = (float *)malloc(sizeof(float) * dk * dv);
    for (int e = 0; e < dk * dv; ++e) R[e] = (double)S[e];

    /* Compensator tokens: deflated power iteration on the residual. */
    for (int j = 0; j < r; ++j) {
        int zero = 0;
        for (int c = 0; c < dv; ++c) w[c] = 1.0 / sqrt((double)dv);
        for (int it = 0; it < cfg->K && !zero; ++it) {
            double nz = 0.0;
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int c = 0; c < dv; ++c) acc += R[i * dv + c] * w[c];
                z[i] = acc;
                nz += acc * acc;
            }
            nz = sqrt(nz);
            if (nz == 0.0) { zero = 1; break; }
            for (int i = 0; i < dk; ++i) z[i] /= nz;
            double nw = 0.0;
            for (int c = 0; c < dv; ++c) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += R[i * dv + c] * z[i];
                w[c] = acc;
                nw += acc * acc;
            }
            nw = sqrt(nw);
            if (nw == 0.0) { zero = 1; break; }
            for (int c = 0; c < dv; ++c) w[c] /= nw;
        }
        float *cj = out->c + (size_t)j * dk, *wj = out->w + (size_t)j * dv;
        if (zero) {
            for (int i = 0; i < dk; ++i) cj[i] = 0.0f;
            for (int c = 0; c < dv; ++c) wj[c] = 0.0f;
            continue;
        }
        for (int c = 0; c < dv; ++c) wj[c] = (float)w[c];
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int c = 0; c < dv; ++c) acc += R[i * dv + c] * (double)wj[c];
            cj[i] = (float)acc;
        }
        for (int i = 0; i < dk; ++i)
            for (int c = 0; c < dv; ++c)
                R[i * dv + c] -= (double)cj[i] * (double)wj[c];
    }
    for (int e = 0; e < dk * dv; ++e) R32[e] = (float)R[e];

    /* BF16 rows (DAMP): stored as rounded bf16 of the residual row. */
    for (int p = 0; p < P; ++p) {
        const int i = hp_rows[p];
        for (int c = 0; c < dv; ++c) out->hp[(size_t)p * dv + c] = lqo_bf16_rne(R32[i * dv + c]);
    }

    /* Smoothing: per key row RMS of the residual (static scales: the
     * head's fitted ones). */
    for (int i = 0; i < dk; ++i) {
        float mi = 1.0f;
        if (cfg->smoothing == 2) {
            mi = cfg->static_m[i];
        } else if (cfg->smoothing && !is_hp_row(hp_rows, P, i)) {
            double ss = 0.0;
            for (int c = 0; c < dv; ++c) ss += (double)R32[i * dv + c] * (double)R32[i * dv + c];
            mi = (float)sqrt(ss / (double)dv);
            if (mi == 0.0f) mi = 1.0f;
        }
        out->m[i] = mi;
        for (int c = 0; c < dv; ++c) x[i * dv + c] = R32[i * dv + c] / mi;   /* float division */
    }

    /* Per value column scale and codes. */
    for (int c = 0; c < dv; ++c) {
        float a = 0.0f;
        for (int i = 0; i < dk; ++i) {
            if (is_hp_row(hp_rows, P, i)) continue;
            const float ax = fabsf(x[i * dv + c]);
            if (ax > a) a = ax;
        }
        const float qmax = (float)lqo_qmax(cfg);
        const float sc = cfg->smoothing == 2 ? cfg->static_s[c] : a / qmax;
        out->s[c] = sc;
        for (int i = 0; i < dk; ++i) {
            int8_t code = 0;
            double rt = 0.0;
            if (!is_hp_row(hp_rows, P, i) && sc != 0.0f) {
                const float qf = x[i * dv + c] / sc;   /* float division */
                float rq = rintf(qf);                  /* round half to even */
                if (rq > qmax) rq = qmax;
                if (rq < -qmax) rq = -qmax;
                code = (int8_t)rq;
                rt = (double)x[i * dv + c] / (double)sc;
            }
            out->codes[i * dv + c] = code;
            if (ratio) ratio[i * dv + c] = rt;
        }
    }
    free(R); free(z); free(w); free(R32); free(x);
}

/* Window-start state: S = Deq(C, m, s) + sum_j c_j w_j^T, with
 * Deq_ic = (C_ic * s_c) * m_i evaluated in float in that order, BF16 rows
 * widened exactly. */
void lqo_dequantize(const lqo_cfg *cfg, const int *hp_rows, const lqo_view *in, double *S)
{
    const int dk = cfg->dk, dv = cfg->dv, P = cfg->P;
    for (int i = 0; i < dk; ++i)
        for (int c = 0; c < dv; ++c) {
            const float cs = (float)in->codes[i * dv + c] * in->s[c];
            S[i * dv + c] = (double)(cs * in->m[i]);
        }
    for (int p = 0; p < P; ++p) {
        const int i = hp_rows[p];
        for (int c = 0; c < dv; ++c) S[i * dv + c] = (double)lqo_bf16_to_float(in->hp[(size_t)p * dv + c]);
    }
    for (int j = 0; j < cfg->r; ++j)
        for (int i = 0; i < dk; ++i)
            for (int c = 0; c < dv; ++c)
                S[i * dv + c] += (double)in->c[(size_t)j * dk + i] * (double)in->w[(size_t)j * dv + c];
}

/* ------------------------------------------------------------------ */
/* Windowed decode of many independent heads [Leap-W].                */
/* ------------------------------------------------------------------ */

typedef struct {
    int8_t *codes; float *m; float *s; float *c; float *w; uint16_t *hp;
} lqo_views; /* the same arrays for nh heads, head-major */

static void view_of(const lqo_cfg *cfg, const lqo_views *vs, int h, lqo_view *v)
{
    const size_t dk = cfg->dk, dv = cfg->dv, r = cfg->r, P = cfg->P;
    v->codes = vs->codes + h * dk * dv;
    v->m = vs->m + h * dk;
    v->s = vs->s + h * dv;
    v->c = vs->c + h * r * dk;
    v->w = vs->w + h * r * dv;
    v->hp = vs->hp ? vs->hp + h * P * dv : NULL;
}

static void to_float(const double *S, float *F, int n)
{
    for (int e = 0; e < n; ++e) F[e] = (float)S[e];
}

/*
 * Run T tokens for nh heads.
 *   from_view = 0: the initial view is Q(S0) (INT8 mode) or S0 itself (FP32).
 *   from_view = 1: the initial view is taken from `view` (INT8 mode only).
 * Inputs are token-major: q,k [T][nh][dk], v [T][nh][dv], beta [T][nh],
 * alpha [T][nh][1 or dk].  hp_rows [nh][P].
 * Outputs: o [T][nh][dv]; `view` holds the last quantized view; S_out
 * [nh][dk][dv] the state after the last token (after a final flush if one was
 * made); S_pre [nh][dk][dv] (nullable) the state right before the last flush;
 * n_out [nh] the tokens buffered since the last window start.
 * flush_last: flush when the last token completes a window.
 * phase [nh] (nullable): staggered windows -- head h's first window ends after
 * W - phase[h] tokens, every later one after W (the page's rule of one
 * requantization per W tokens of a sequence, with the sequences' window ends
 * shifted against each other); NULL: every first window holds W tokens.
 */
void lqo_run(const lqo_cfg *cfg, int nh, const int *hp_rows, int from_view,
             const float *S0, lqo_views *view, int T, const float *q,
             const float *k, const float *v, const float *beta,
             const float *alpha, double *o, double *S_out, double *S_pre,
             int *n_out, int flush_last, int nthreads, const int *phase)
{
    const int dk = cfg->dk, dv = cfg->dv, ga = cfg->gate ? dk : 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int h = 0; h < nh; ++h) {
        lqo_cfg hc = *cfg;     /* this head's static scales, if any */
        if (cfg->smoothing == 2) {
            hc.static_m = cfg->static_m + (size_t)h * dk;
            hc.static_s = cfg->static_s + (size_t)h * dv;
        }
        const lqo_cfg *hcfg = &hc;
        double *S = S_out + (size_t)h * dk * dv;
        float *F = (float *)malloc(sizeof(float) * dk * dv);
        const int *hr = hp_rows ? hp_rows + (size_t)h * hcfg->P : NULL;
        lqo_view vh;
        view_of(hcfg, view, h, &vh);
        if (hcfg->quantize) {
            if (!from_view) lqo_quantize(hcfg, hr, S0 + (size_t)h * dk * dv, &vh, NULL);
            lqo_dequantize(hcfg, hr, &vh, S);
        } else {
            for (int e = 0; e < dk * dv; ++e) S[e] = (double)S0[(size_t)h * dk * dv + e];
        }
        int n = 0;
        int len = hcfg->W - (phase ? phase[h] : 0);   /* tokens of the current window */
        float gam[512];
        for (int j = 0; j < ga; ++j) gam[j] = 1.0f;
        for (int t = 0; t < T; ++t) {
            const size_t th = (size_t)t * nh + h;
            if (hcfg->quantize && hcfg->bf16_buffer) {
                if (n == 0)
                    for (int j = 0; j < ga; ++j) gam[j] = 1.0f;
                lqo_step_bf16(hcfg, S, gam, q + th * dk, k + th * dk, v + th * dv, beta[th],
                              alpha + th * ga, o + th * dv);
            } else {
                lqo_step(hcfg, S, q + th * dk, k + th * dk, v + th * dv, beta[th],
                         alpha + th * ga, o + th * dv);
            }
            n += 1;
            if (hcfg->quantize && n == len && (t < T - 1 || flush_last)) {
                if (S_pre) memcpy(S_pre + (size_t)h * dk * dv, S, sizeof(double) * dk * dv);
                to_float(S, F, dk * dv);
                lqo_quantize(hcfg, hr, F, &vh, NULL);
                lqo_dequantize(hcfg, hr, &vh, S);
                n = 0;
                len = hcfg->W;
            }
        }
        if (n_out) n_out[h] = n;
        free(F);
    }
}

/* ------------------------------------------------------------------ */
/* DAMP channel risk [DAMP].                                           */
/* ------------------------------------------------------------------ */

/* Quantization-error energy per key row, summed over n calibration states of
 * one head: E_i += sum_c (R_ic - Deq_ic)^2, where R is the residual after the
 * compensators and Deq its INT8 reconstruction (no BF16 rows). */
void lqo_damp_energy(const lqo_cfg *cfg, int n, const float *states, double *E)
{
    const int dk = cfg->dk, dv = cfg->dv, r = cfg->r;
    lqo_cfg c2 = *cfg;
    c2.P = 0;
    lqo_view v;
    v.codes = (int8_t *)malloc(dk * dv);
    v.m = (float *)malloc(sizeof(float) * dk);
    v.s = (float *)malloc(sizeof(float) * dv);
    v.c = (float *)malloc(sizeof(float) * (r > 0 ? r : 1) * dk);
    v.w = (float *)malloc(sizeof(float) * (r > 0 ? r : 1) * dv);
    v.hp = NULL;
    double *R = (double *)malloc(sizeof(double) * dk * dv);
    for (int i = 0; i < dk; ++i) E[i] = 0.0;
    for (int t = 0; t < n; ++t) {
        const float *S = states + (size_t)t * dk * dv;
        lqo_quantize(&c2, NULL, S, &v, NULL);
        /* residual in float, as handed to the quantizer */
        for (int e = 0; e < dk * dv; ++e) R[e] = (double)S[e];
        for (int j = 0; j < r; ++j)
            for (int i = 0; i < dk; ++i)
                for (int c = 0; c < dv; ++c)
                    R[i * dv + c] -= (double)v.c[j * dk + i] * (double)v.w[j * dv + c];
        for (int i = 0; i < dk; ++i) {
            double e = 0.0;
            for (int c = 0; c < dv; ++c) {
                const float rr = (float)R[i * dv + c];
                const float dq = ((float)v.codes[i * dv + c] * v.s[c]) * v.m[i];
                const double d = (double)rr - (double)dq;
                e += d * d;
            }
            E[i] += e;
        }
    }
    free(v.codes); free(v.m); free(v.s); free(v.c); free(v.w); free(R);
}

/* DAMP's risk score of every key row of one head [DAMP]: the calibration
 * error energy E_i times the row's decay persistence 1 / (1 - a_i), with a_i
 * the mean decay over the n calibration samples gates [n][ga] -- of the row's
 * own channel for KDA (ga = dk), of the head for GDN (ga = 1, the same factor
 * for every row).  Means accumulate in double in sample order. */
void lqo_damp_score(int dk, int ga, int n, const float *gates, const double *E, double *score)
{
    for (int i = 0; i < dk; ++i) {
        const int c = ga == 1 ? 0 : i;
        double mean = 0.0;
        for (int s = 0; s < n; ++s) mean += (double)gates[(size_t)s * ga + c];
        mean /= (double)n;
        score[i] = E[i] * (1.0 / (1.0 - mean));
    }
}

/* Top-P rows by score, ties to the lower index, returned in increasing row
 * order. */
void lqo_damp_select(int dk, int P, const double *score, int *rows)
{
    char *taken = (char *)calloc(dk, 1);
    for (int p = 0; p < P; ++p) {
        int best = -1;
        for (int i = 0; i < dk; ++i) {
            if (taken[i]) continue;
            if (best < 0 || score[i] > score[best]) best = i;
        }
        taken[best] = 1;
    }
    int n = 0;
    for (int i = 0; i < dk; ++i)
        if (taken[i]) rows[n++] = i;
    free(taken);
}

/* ------------------------------------------------------------------ */
/* Static key-row / value-column scales fitted offline [STEP].         */
/* ------------------------------------------------------------------ */

/*
 * The STEPQuant article says the scales are fitted jointly, offline, from
 * state distributions and each key row's impact on the output error, with no
 * formula.  Reading taken here (the plainest one that fits the quantizer
 * above):
 *  - fitted per head on n calibration states, on the residual the quantizer
 *    sees (after the cfg->r compensators);
 *  - objective: sum over states, rows, columns of weight_i (R_ic - Deq_ic)^2,
 *    Deq_ic = (clamp(rne((R_ic / m_i) / s_c)) s_c) m_i as at run time; the
 *    row weight carries the row's impact (the caller passes e.g. the decay
 *    persistence 1 / (1 - mean gate), NULL = 1);
 *  - start: m_i = RMS of row i over all states (1 if 0), s_c = the largest
 *    |R_ic / m_i| over all states and rows / qmax;
 *  - LQO_FIT_ROUNDS rounds of coordinate descent, each first over the
 *    columns then over the rows: s_c takes the best of s_c0 x (1 - j/16),
 *    j = 0..11, for the current m; then m_i the best of m_i0 x {1/2, 5/8, 3/4,
 *    7/8, 1, 5/4, 3/2, 7/4, 2} for the current s (ties to the first
 *    candidate); the current value is always a candidate, so the objective
 *    never increases.
 * Errors are accumulated in double, states outer, then rows (column step) or
 * columns (row step); every float step is the quantizer's.
 */
#define LQO_FIT_ROUNDS 3
#define LQO_FIT_NCOL 12
#define LQO_FIT_NROW 9
static const float lqo_fit_rowgrid[LQO_FIT_NROW] = {0.5f, 0.625f, 0.75f, 0.875f, 1.0f, 1.25f, 1.5f, 1.75f, 2.0f};

static double lqo_fit_err(float R, float m, float s, float qmax)
{
    float dq = 0.0f;
    if (s != 0.0f) {
        const float x = R / m;
        float rq = rintf(x / s);
        if (rq > qmax) rq = qmax;
        if (rq < -qmax) rq = -qmax;
        dq = (rq * s) * m;
    }
    const double d = (double)R - (double)dq;
    return d * d;
}

/* Residuals R [n][dk][dv] (float) of n states after the r compensators. */
static void lqo_residuals(const lqo_cfg *cfg, int n, const float *states, float *R)
{
    const int dk = cfg->dk, dv = cfg->dv, r = cfg->r;
    lqo_cfg c2 = *cfg;
    c2.P = 0;
    c2.smoothing = 1;
    lqo_view v;
    v.codes = (int8_t *)malloc(dk * dv);
    v.m = (float *)malloc(sizeof(float) * dk);
    v.s = (float *)malloc(sizeof(float) * dv);
    v.c = (float *)malloc(sizeof(float) * (r > 0 ? r : 1) * dk);
    v.w = (float *)malloc(sizeof(float) * (r > 0 ? r : 1) * dv);
    v.hp = NULL;
    double *D = (double *)malloc(sizeof(double) * dk * dv);
    for (int t = 0; t < n; ++t) {
        const float *S = states + (size_t)t * dk * dv;
        lqo_quantize(&c2, NULL, S, &v, NULL);
        for (int e = 0; e < dk * dv; ++e) D[e] = (double)S[e];
        for (int j = 0; j < r; ++j)
            for (int i = 0; i < dk; ++i)
                for (int c = 0; c < dv; ++c)
                    D[i * dv + c] -= (double)v.c[j * dk + i] * (double)v.w[j * dv + c];
        for (int e = 0; e < dk * dv; ++e) R[(size_t)t * dk * dv + e] = (float)D[e];
    }
    free(v.codes); free(v.m); free(v.s); free(v.c); free(v.w); free(D);
}

/* Fit one head: m [dk], s [dv]; obj [LQO_FIT_ROUNDS + 1] (nullable) receives
 * the objective at the start and after every round. */
void lqo_fit_static(const lqo_cfg *cfg, int n, const float *states, const double *weight,
                    float *m, float *s, double *obj)
{
    const int dk = cfg->dk, dv = cfg->dv;
    const float qmax = (float)lqo_qmax(cfg);
    float *R = (float *)malloc(sizeof(float) * (size_t)n * dk * dv);
    float *m0 = (float *)malloc(sizeof(float) * dk);
    float *s0 = (float *)malloc(sizeof(float) * dv);
    lqo_residuals(cfg, n, states, R);
#define RES(t, i, c) R[((size_t)(t) * dk + (i)) * dv + (c)]
    for (int i = 0; i < dk; ++i) {
        double ss = 0.0;
        for (int t = 0; t < n; ++t)
            for (int c = 0; c < dv; ++c) ss += (double)RES(t, i, c) * (double)RES(t, i, c);
        float mi = (float)sqrt(ss / ((double)n * dv));
        if (mi == 0.0f) mi = 1.0f;
        m0[i] = m[i] = mi;
    }
    for (int c = 0; c < dv; ++c) {
        float a = 0.0f;
        for (int t = 0; t < n; ++t)
            for (int i = 0; i < dk; ++i) {
                const float ax = fabsf(RES(t, i, c) / m[i]);
                if (ax > a) a = ax;
            }
        s0[c] = s[c] = a / qmax;
    }
    for (int round = 0; round <= LQO_FIT_ROUNDS; ++round) {
        if (obj) {
            double e = 0.0;
            for (int t = 0; t < n; ++t)
                for (int i = 0; i < dk; ++i)
                    for (int c = 0; c < dv; ++c)
                        e += (weight ? weight[i] : 1.0) * lqo_fit_err(RES(t, i, c), m[i], s[c], qmax);
            obj[round] = e;
        }
        if (round == LQO_FIT_ROUNDS) break;
        for (int c = 0; c < dv; ++c) {
            double best = INFINITY;
            float sb = s[c];
            for (int j = 0; j < LQO_FIT_NCOL; ++j) {
                const float sc = s0[c] * (1.0f - (float)j / 16.0f);
                double e = 0.0;
                for (int t = 0; t < n; ++t)
                    for (int i = 0; i < dk; ++i)
                        e += (weight ? weight[i] : 1.0) * lqo_fit_err(RES(t, i, c), m[i], sc, qmax);
                if (e < best) { best = e; sb = sc; }
            }
            s[c] = sb;
        }
        for (int i = 0; i < dk; ++i) {
            double best = INFINITY;
            float mb = m[i];
            for (int j = 0; j < LQO_FIT_NROW; ++j) {
                const float mi = m0[i] * lqo_fit_rowgrid[j];
                double e = 0.0;
                for (int t = 0; t < n; ++t)
                    for (int c = 0; c < dv; ++c) e += lqo_fit_err(RES(t, i, c), mi, s[c], qmax);
                if (e < best) { best = e; mb = mi; }
            }
            m[i] = mb;
        }
    }
#undef RES
    free(R); free(m0); free(s0);
}

/* The fit's objective for given scales m [dk], s [dv] on one head's states. */
double lqo_fit_objective(const lqo_cfg *cfg, int n, const float *states, const double *weight,
                         const float *m, const float *s)
{
    const int dk = cfg->dk, dv = cfg->dv;
    const float qmax = (float)lqo_qmax(cfg);
    float *R = (float *)malloc(sizeof(float) * (size_t)n * dk * dv);
    lqo_residuals(cfg, n, states, R);
    double e = 0.0;
    for (int t = 0; t < n; ++t)
        for (int i = 0; i < dk; ++i)
            for (int c = 0; c < dv; ++c)
                e += (weight ? weight[i] : 1.0) * lqo_fit_err(R[((size_t)t * dk + i) * dv + c], m[i], s[c], qmax);
    free(R);
    return e;
}
