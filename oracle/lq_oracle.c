/*
 * lq_oracle.c -- plain, slow CPU oracle of the LeapQuant decode path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline / reference leg load this library.  The product path (the CUDA
 * library and its Python binding) never calls it and shares no code with it.
 *
 * Sources (the pages print no equations; the recurrences are the standard
 * Gated DeltaNet / Kimi Delta Attention delta rule):
 *   [NEWS]  news post "Linear attention has to move state every token it
 *           generates; LeapQuant compresses it to 8-bit without losing
 *           accuracy": the paragraphs on per-window quantization, on
 *           Compensator Tokens and on residual smoothing.
 *   [ABS]   "LeapQuant: Efficient Linear Attention with Accurate Recurrent
 *           State Quantization", original abstract.
 *
 * Conventions.  One head's state S is dk x dv, row i = key channel, column j =
 * value channel, stored row-major S[i*dv + j].  Codes are value-major:
 * codes[j*dk + i] quantizes residual entry (i, j).  All arithmetic is FP64
 * except where a floating-point result decides an integer (a quantization
 * code, a quantization scale); those decisions are taken in FP32, the
 * precision the state is stored and quantized in, with IEEE correctly rounded
 * division.  Build with -ffp-contract=off and without fast-math.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - the GDN step  S <- a S + k u^T,  u = beta (v - (a S)^T k),  o = S^T q
 *     after the update; KDA uses diag(a) S with a per key channel;
 *   - compensators are one-hot rank-one lines: greedy, r rounds, the key row
 *     or value column with the largest residual L2 energy (ties: larger
 *     energy, then row before column, then lower index);
 *   - smoothing divides each key row of the residual by the power of two at
 *     or above its absolute maximum (1 for an all-zero row);
 *   - quantization is symmetric per value column of the smoothed residual,
 *     scale = fl32(absmax / Qmax) rounded to the storage dtype, codes =
 *     clamp(rint(fl32(R'/scale)), -Qmax, Qmax), ties to even;
 *   - the naive per-step baselines of the accuracy table (BF16, FP8) store the
 *     whole FP32-rounded state after every token: BF16 entry by entry, FP8 as
 *     E4M3 codes with one FP32 scale fl32(absmax / 448) per value column.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t dk, dv;
    int32_t window;     /* W: tokens per quantization window */
    int32_t num_comp;   /* r: compensator lines kept in FP32 */
    int32_t bits;       /* 8, 6, 4; 32 = unquantized FP32 state */
    int32_t kda;        /* 0: scalar decay per head, 1: per key channel */
    int32_t smoothing;  /* 0/1 */
    int32_t scale_f16;  /* 0: scales stored in f32, 1: in f16 */
    int32_t per_step;   /* 1: the naive per-step baselines: a dense state stored
                           after every token as BF16 (bits 16) or as FP8 E4M3
                           codes with one FP32 scale per value column (bits 8) */
} lqo_params;

#define LQO_KIND_COL 0x80000000u
#define LQO_NONE 0xFFFFFFFFu

static int qmax_of(int bits) { return (1 << (bits - 1)) - 1; }

/* ------------------------------------------------------------------------ */
/* IEEE binary16 rounding, written from the format's definition: 11
 * significant bits, exponent >= -14 (below that, a fixed quantum of 2^-24),
 * largest finite 65504, round to nearest with ties to even.  Returns the
 * rounded value as a double (exact).                                        */
double lqo_round_f16(double x)
{
    if (x != x) return x;
    double ax = fabs(x);
    if (ax >= 65520.0) return x > 0 ? INFINITY : -INFINITY;
    if (ax == 0.0) return x;
    int e;
    frexp(ax, &e);              /* ax = f * 2^e, f in [0.5, 1) */
    int ex = e - 1;             /* floor(log2(ax)) */
    if (ex < -14) ex = -14;     /* subnormal range */
    double quantum = ldexp(1.0, ex - 10);
    double r = nearbyint(ax / quantum) * quantum;   /* ax/quantum is exact */
    return x < 0 ? -r : r;
}

/* smallest power of two >= m, for finite m > 0 */
static double pow2_ceil(double m)
{
    int e;
    double f = frexp(m, &e);    /* m = f * 2^e, f in [0.5, 1) */
    return (f == 0.5) ? ldexp(1.0, e - 1) : ldexp(1.0, e);
}

/* ------------------------------------------------------------------------ */
/* Compress: one head's FP32 state -> compensators + smoothed, quantized
 * residual.  [NEWS] Compensator Tokens paragraph (the largest outliers leave
 * as a few rank-one high-precision pairs, the rest is quantized), residual
 * smoothing paragraph (balance each key row before quantizing; the scales are
 * refreshed at the window boundary); [ABS].
 *
 *   S         [dk*dv]   input state (row = key channel)
 *   forced    [r] or NULL: if given, forced[c] is the line taken in round c
 *             (kind bit | index, LQO_NONE to stop); used only to compare the
 *             rest of the result once a near tie has been shown valid
 *   codes     [dv*dk]   out, value-major, values in [-Qmax, Qmax]
 *   qs        [dv]      out, quantization scale per value column (as stored)
 *   sm        [dk]      out, smoothing scale per key row (power of two)
 *   meta      [r]       out, kind bit | index per round, LQO_NONE if unused
 *   vec       [r*maxd]  out, the line's values (row: w over dv; col: p over dk)
 *   top2      [2r] or NULL: out, per round the best and runner-up energies
 *   R_out     [dk*dv] or NULL: out, the residual after extraction (pre-smoothing)
 * Returns the number of compensators taken.                                */
int lqo_compress(const lqo_params *p, const float *S, const uint32_t *forced,
                 int8_t *codes, float *qs, float *sm, uint32_t *meta, float *vec,
                 double *top2, double *R_out)
{
    const int dk = p->dk, dv = p->dv, r = p->num_comp;
    const int maxd = dk > dv ? dk : dv;
    const int qmax = qmax_of(p->bits);
    double *R = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *rowE = (double *)malloc(sizeof(double) * dk);
    double *colE = (double *)malloc(sizeof(double) * dv);
    for (int i = 0; i < dk * dv; ++i) R[i] = (double)S[i];
    for (int c = 0; c < r; ++c) {
        meta[c] = LQO_NONE;
        for (int x = 0; x < maxd; ++x) vec[(size_t)c * maxd + x] = 0.0f;
    }

    /* greedy extraction of one-hot rank-one lines */
    int ncomp = 0;
    for (int c = 0; c < r; ++c) {
        for (int i = 0; i < dk; ++i) {
            double e = 0.0;
            for (int j = 0; j < dv; ++j) e += R[i * dv + j] * R[i * dv + j];
            rowE[i] = e;
        }
        for (int j = 0; j < dv; ++j) {
            double e = 0.0;
            for (int i = 0; i < dk; ++i) e += R[i * dv + j] * R[i * dv + j];
            colE[j] = e;
        }
        /* scan rows then columns, ascending index; only a strictly larger
         * energy replaces the incumbent, which realises the tie order */
        double best = -1.0, second = -1.0;
        uint32_t pick = LQO_NONE;
        for (int i = 0; i < dk; ++i) {
            if (rowE[i] > best) { second = best; best = rowE[i]; pick = (uint32_t)i; }
            else if (rowE[i] > second) second = rowE[i];
        }
        for (int j = 0; j < dv; ++j) {
            if (colE[j] > best) { second = best; best = colE[j]; pick = LQO_KIND_COL | (uint32_t)j; }
            else if (colE[j] > second) second = colE[j];
        }
        if (top2) { top2[2 * c] = best; top2[2 * c + 1] = second; }
        if (forced) pick = forced[c];
        if (pick == LQO_NONE) break;
        double chosen = (pick & LQO_KIND_COL) ? colE[pick & 0x7FFFFFFFu] : rowE[pick];
        if (!(chosen > 0.0)) break;          /* nothing left to extract */
        float *w = vec + (size_t)c * maxd;
        if (pick & LQO_KIND_COL) {
            int j0 = (int)(pick & 0x7FFFFFFFu);
            for (int i = 0; i < dk; ++i) { w[i] = (float)R[i * dv + j0]; R[i * dv + j0] = 0.0; }
        } else {
            int i0 = (int)pick;
            for (int j = 0; j < dv; ++j) { w[j] = (float)R[i0 * dv + j]; R[i0 * dv + j] = 0.0; }
        }
        meta[c] = pick;
        ++ncomp;
    }
    if (R_out) memcpy(R_out, R, sizeof(double) * (size_t)dk * dv);

    /* residual smoothing: one power of two per key row */
    const double sm_lo = p->scale_f16 ? ldexp(1.0, -14) : ldexp(1.0, -126);
    const double sm_hi = p->scale_f16 ? ldexp(1.0, 15) : ldexp(1.0, 127);
    for (int i = 0; i < dk; ++i) {
        double m = 0.0;
        for (int j = 0; j < dv; ++j) m = fmax(m, fabs(R[i * dv + j]));
        double s = 1.0;
        if (p->smoothing && m > 0.0) {
            s = pow2_ceil(m);
            if (s < sm_lo) s = sm_lo;
            if (s > sm_hi) s = sm_hi;
        }
        sm[i] = (float)s;
        for (int j = 0; j < dv; ++j)    /* FP32 division by a power of two: exact */
            R[i * dv + j] = (double)((float)R[i * dv + j] / (float)s);
    }

    /* symmetric quantization per value column, decisions in FP32 */
    const double q_min = p->scale_f16 ? ldexp(1.0, -24) : ldexp(1.0, -149);
    for (int j = 0; j < dv; ++j) {
        double m = 0.0;
        for (int i = 0; i < dk; ++i) m = fmax(m, fabs(R[i * dv + j]));
        float s = (float)m / (float)qmax;
        if (p->scale_f16) s = (float)lqo_round_f16((double)s);
        if (m > 0.0 && s == 0.0f) s = (float)q_min;
        qs[j] = s;
        for (int i = 0; i < dk; ++i) {
            int c = 0;
            if (s != 0.0f) {
                float t = (float)R[i * dv + j] / s;
                double n = nearbyint((double)t);        /* ties to even */
                if (n > qmax) n = qmax;
                if (n < -qmax) n = -qmax;
                c = (int)n;
            }
            codes[(size_t)j * dk + i] = (int8_t)c;
        }
    }
    free(R); free(rowE); free(colE);
    return ncomp;
}

/* Dequantize one head's compact state to FP64 (exact: every product of a
 * power of two, an FP32 scale and a code of <= 8 bits fits in 53 bits).
 * [ABS]: outputs come from the fixed low-bit state; the compensators are
 * rank-one pairs added back.                                                */
void lqo_dequant(const lqo_params *p, const int8_t *codes, const float *qs, const float *sm,
                 const uint32_t *meta, const float *vec, double *S)
{
    const int dk = p->dk, dv = p->dv, maxd = dk > dv ? dk : dv;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[i * dv + j] = (double)sm[i] * (double)qs[j] * (double)codes[(size_t)j * dk + i];
    for (int c = 0; c < p->num_comp; ++c) {
        if (meta[c] == LQO_NONE) continue;
        const float *w = vec + (size_t)c * maxd;
        if (meta[c] & LQO_KIND_COL) {
            int j0 = (int)(meta[c] & 0x7FFFFFFFu);
            for (int i = 0; i < dk; ++i) S[i * dv + j0] += (double)w[i];
        } else {
            int i0 = (int)meta[c];
            for (int j = 0; j < dv; ++j) S[i0 * dv + j] += (double)w[j];
        }
    }
}

/* The window-end state evaluated in FP32, in the order the definition reads
 * left to right:  S_ij = g_i * ( sm_i*qs_j*C_ji  +  sum_c p_c,i w_c,j
 *                               + sum_m khat_m,i u_m,j )
 * with the base product taken as (qs_j * C_ji) * sm_i, the compensators added
 * in round order, the pairs accumulated by fused multiply-add in buffer order
 * and the decay applied last.  This is the FP32 state that the window-end
 * requantization sees ([NEWS] per-window paragraph: the fixed low-precision
 * state plus the cached high-precision updates).
 *   pairs [count*(dk+dv)]: pair m is khat_m (dk values) then u_m (dv values)
 *   g     [dk]: decay accumulated since the window start                   */
void lqo_reconstruct_f32(const lqo_params *p, const int8_t *codes, const float *qs,
                         const float *sm, const uint32_t *meta, const float *vec,
                         int count, const float *pairs, const float *g, float *S)
{
    const int dk = p->dk, dv = p->dv, maxd = dk > dv ? dk : dv, pd = dk + dv;
    for (int i = 0; i < dk; ++i) {
        for (int j = 0; j < dv; ++j) {
            float acc = (qs[j] * (float)codes[(size_t)j * dk + i]) * sm[i];
            for (int c = 0; c < p->num_comp; ++c) {
                if (meta[c] == LQO_NONE) continue;
                const float *w = vec + (size_t)c * maxd;
                if (meta[c] & LQO_KIND_COL) {
                    if ((int)(meta[c] & 0x7FFFFFFFu) == j) acc = acc + w[i];
                } else {
                    if ((int)meta[c] == i) acc = acc + w[j];
                }
            }
            for (int m = 0; m < count; ++m)
                acc = fmaf(pairs[(size_t)m * pd + i], pairs[(size_t)m * pd + dk + j], acc);
            S[i * dv + j] = g[i] * acc;
        }
    }
}

/* One delta-rule decode step in FP64, in place.  GDN: a_i = alpha for every
 * key row; KDA: a_i per key channel.
 *   S' = diag(a) S;  u = beta (v - S'^T k);  S = S' + k u^T;  o = S^T q      */
void lqo_step(int dk, int dv, double *S, const double *q, const double *k, const double *v,
              double beta, const double *a, double *o, double *u_out)
{
    double *u = (double *)malloc(sizeof(double) * dv);
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a[i];
    for (int j = 0; j < dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < dk; ++i) s += S[i * dv + j] * k[i];
        u[j] = beta * (v[j] - s);
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] += k[i] * u[j];
    for (int j = 0; j < dv; ++j) {
        double s = 0.0;
        for (int i = 0; i < dk; ++i) s += S[i * dv + j] * q[i];
        o[j] = s;
    }
    if (u_out) memcpy(u_out, u, sizeof(double) * dv);
    free(u);
}

/* Round an FP64 state to the FP32 state that is stored and requantized. */
static void to_f32(int n, const double *x, float *y)
{
    for (int i = 0; i < n; ++i) y[i] = (float)x[i];
}

/* Rounding to a binary floating-point format with `sig` significant bits
 * (the implicit bit included) and smallest normal 2^emin, below which values
 * keep the fixed quantum 2^(emin - sig + 1); round to nearest, ties to even.
 * Written from the formats' definitions; returns the rounded value exactly. */
static double round_format(double x, int sig, int emin)
{
    if (x != x || x == 0.0) return x;
    double ax = fabs(x);
    int e;
    frexp(ax, &e);              /* ax = f * 2^e, f in [0.5, 1) */
    int ex = e - 1;             /* floor(log2(ax)) */
    if (ex < emin) ex = emin;
    double quantum = ldexp(1.0, ex - (sig - 1));
    double r = nearbyint(ax / quantum) * quantum;   /* ax/quantum is exact */
    return x < 0 ? -r : r;
}

/* bfloat16: 8 significant bits, the exponent range of binary32 (largest
 * finite 0x1.FEp127; beyond it the rounding gives infinity). */
double lqo_round_bf16(double x)
{
    double r = round_format(x, 8, -126);
    if (fabs(r) > 0x1.FEp127) return x > 0 ? INFINITY : -INFINITY;
    return r;
}

/* FP8 E4M3 (the "fn" variant: no infinities, largest finite 448):
 * 4 significant bits, smallest normal 2^-6; magnitudes that round beyond 448
 * saturate to 448 (the saturating conversion the state uses). */
double lqo_round_e4m3(double x)
{
    double r = round_format(x, 4, -6);
    if (r > 448.0) return 448.0;
    if (r < -448.0) return -448.0;
    return r;
}

/* Per-value-column FP8 quantization of an FP32 state (row-major, dk x dv):
 * scale_j = fl32(max_i |S_ij| / 448), val_ij = e4m3(fl32(S_ij / scale_j))
 * (ties to even, saturating); an all-zero column has scale 0 and values 0.
 * The divisions are the correctly rounded FP32 quotients (a binary64 quotient
 * of two floats rounded once more to binary32 is correctly rounded). */
void lqo_fp8_columns(int dk, int dv, const float *S32, float *scale, float *val)
{
    for (int j = 0; j < dv; ++j) {
        float m = 0.f;
        for (int i = 0; i < dk; ++i) m = fmaxf(m, fabsf(S32[i * dv + j]));
        const float sc = (float)((double)m / 448.0);
        scale[j] = sc;
        for (int i = 0; i < dk; ++i)
            val[i * dv + j] = sc == 0.f ? 0.f
                                        : (float)lqo_round_e4m3((double)(float)((double)S32[i * dv + j] / (double)sc));
    }
}

/* The naive per-step baselines ([NEWS] accuracy table: BF16 and FP8 states):
 * after every token the state is rounded to FP32 and stored in the narrow
 * format, and the next token starts from the stored values.  BF16: each entry
 * rounded to bfloat16.  FP8: per-value-column E4M3 codes, dequantized as
 * fl32(code * scale).                                                      */
static void per_step_store(const lqo_params *p, double *S, float *buf32, float *scale, float *val)
{
    const int n = p->dk * p->dv;
    to_f32(n, S, buf32);
    if (p->bits == 16) {
        for (int x = 0; x < n; ++x) S[x] = lqo_round_bf16((double)buf32[x]);
        return;
    }
    lqo_fp8_columns(p->dk, p->dv, buf32, scale, val);
    for (int i = 0; i < p->dk; ++i)
        for (int j = 0; j < p->dv; ++j)
            S[i * p->dv + j] = (double)(float)((double)val[i * p->dv + j] * (double)scale[j]);
}

/* Compress then dequantize, in place: the state after a window boundary. */
static void requantize(const lqo_params *p, double *S, float *buf32, int8_t *codes, float *qs,
                       float *sm, uint32_t *meta, float *vec)
{
    to_f32(p->dk * p->dv, S, buf32);
    lqo_compress(p, buf32, NULL, codes, qs, sm, meta, vec, NULL, NULL);
    lqo_dequant(p, codes, qs, sm, meta, vec, S);
}

/* Run whole decode sequences, one head at a time (OpenMP over heads).
 * [NEWS] per-window paragraph, [ABS]: the state is quantized when the
 * sequence enters (the prefill state), stays fixed within a window while the
 * token updates are kept in high precision, and is requantized once at the end
 * of every window of W tokens.  The buffered form is exact algebra, so the
 * plain result is the dense recurrence restarted from the dequantized state at
 * every boundary, which is what this computes.  bits == 32: no quantization at
 * all (the FP32-state reference).  A partial final window stays unquantized.
 * per_step: the naive baselines instead, the whole state stored in BF16 or
 * FP8 after every token (per_step_store).
 *
 *   S0    [nh*dk*dv] float         q,k [T*nh*dk]   v [T*nh*dv]
 *   beta  [T*nh]     decay [T*nh] (GDN) or [T*nh*dk] (KDA)
 *   o     [T*nh*dv] out            S_end [nh*dk*dv] out (FP64), may be NULL
 * Returns the number of threads used.                                       */
int lqo_run(const lqo_params *p, int nh, int T, const float *S0, const float *q,
            const float *k, const float *v, const float *beta, const float *decay,
            double *o, double *S_end, int threads)
{
    const int dk = p->dk, dv = p->dv, maxd = dk > dv ? dk : dv;
    int used = 1;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
    }
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h) {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        float *buf32 = (float *)malloc(sizeof(float) * (size_t)dk * dv);
        int8_t *codes = (int8_t *)malloc((size_t)dk * dv);
        float *qs = (float *)malloc(sizeof(float) * dv);
        float *sm = (float *)malloc(sizeof(float) * dk);
        uint32_t *meta = (uint32_t *)malloc(sizeof(uint32_t) * (p->num_comp + 1));
        float *vec = (float *)malloc(sizeof(float) * (size_t)(p->num_comp + 1) * maxd);
        double *qd = (double *)malloc(sizeof(double) * dk), *kd = (double *)malloc(sizeof(double) * dk);
        double *vd = (double *)malloc(sizeof(double) * dv), *ad = (double *)malloc(sizeof(double) * dk);
        double *od = (double *)malloc(sizeof(double) * dv);

        float *val = (float *)malloc(sizeof(float) * (size_t)dk * dv);
        for (int x = 0; x < dk * dv; ++x) S[x] = (double)S0[(size_t)h * dk * dv + x];
        if (p->per_step) per_step_store(p, S, buf32, qs, val);
        else if (p->bits != 32) requantize(p, S, buf32, codes, qs, sm, meta, vec);
        int in_window = 0;
        for (int t = 0; t < T; ++t) {
            size_t th = (size_t)t * nh + h;
            for (int i = 0; i < dk; ++i) { qd[i] = q[th * dk + i]; kd[i] = k[th * dk + i]; }
            for (int j = 0; j < dv; ++j) vd[j] = v[th * dv + j];
            for (int i = 0; i < dk; ++i) ad[i] = p->kda ? decay[th * dk + i] : decay[th];
            lqo_step(dk, dv, S, qd, kd, vd, (double)beta[th], ad, od, NULL);
            for (int j = 0; j < dv; ++j) o[th * dv + j] = od[j];
            if (p->per_step) {
                per_step_store(p, S, buf32, qs, val);
            } else if (p->bits != 32 && ++in_window == p->window) {
                requantize(p, S, buf32, codes, qs, sm, meta, vec);
                in_window = 0;
            }
        }
        if (S_end) memcpy(S_end + (size_t)h * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(buf32); free(codes); free(qs); free(sm); free(meta); free(vec); free(val);
        free(qd); free(kd); free(vd); free(ad); free(od);
    }
    return used;
}

/* Prompt handoff.  [NEWS] per-window paragraph: the state a prefill leaves
 * enters the quantized cache, and decoding starts from it.  Per head, the
 * FP64 delta rule (lqo_step) over its first len[h] prompt tokens from S0;
 * outputs of tokens at or past len[h] are 0.  S_end is the FP64 final state;
 * the caller compresses its FP32 rounding (lqo_compress), as at a window
 * boundary.  Layouts as lqo_run; len [nh] (NULL: all T).
 * Returns the number of threads used.                                       */
int lqo_prefill(int dk, int dv, int kda, int nh, int T, const int *len, const float *S0,
                const float *q, const float *k, const float *v, const float *beta,
                const float *decay, double *o, double *S_end, int threads)
{
    int used = 1;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
    }
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h) {
        double *S = S_end + (size_t)h * dk * dv;
        double *qd = (double *)malloc(sizeof(double) * dk), *kd = (double *)malloc(sizeof(double) * dk);
        double *vd = (double *)malloc(sizeof(double) * dv), *ad = (double *)malloc(sizeof(double) * dk);
        double *od = (double *)malloc(sizeof(double) * dv);
        const int n = len ? (len[h] < 0 ? 0 : (len[h] > T ? T : len[h])) : T;
        for (int x = 0; x < dk * dv; ++x) S[x] = (double)S0[(size_t)h * dk * dv + x];
        for (int t = 0; t < T; ++t) {
            size_t th = (size_t)t * nh + h;
            if (t >= n) {
                for (int j = 0; j < dv; ++j) o[th * dv + j] = 0.0;
                continue;
            }
            for (int i = 0; i < dk; ++i) { qd[i] = q[th * dk + i]; kd[i] = k[th * dk + i]; }
            for (int j = 0; j < dv; ++j) vd[j] = v[th * dv + j];
            for (int i = 0; i < dk; ++i) ad[i] = kda ? decay[th * dk + i] : decay[th];
            lqo_step(dk, dv, S, qd, kd, vd, (double)beta[th], ad, od, NULL);
            for (int j = 0; j < dv; ++j) o[th * dv + j] = od[j];
        }
        free(qd); free(kd); free(vd); free(ad); free(od);
    }
    return used;
}

/* The buffered window form, FP64, with explicit decay products (no
 * division): within a window starting from S_base,
 *   S'_t = P_t S_base + sum_{m<t} (Q_{m,t} k_m) u_m^T,   P_t = prod_{s<=t} D_s,
 *   Q_{m,t} = prod_{m<s<=t} D_s,
 *   u_t = beta_t (v_t - S'_t^T k_t),  o_t = S'_t^T q_t + (k_t . q_t) u_t.
 * [ABS]: outputs come from the fixed state together with the buffered
 * high-precision updates.  Used to pin that this form equals the dense
 * recurrence.  Inputs for one head: q,k [T*dk], v [T*dv], beta [T],
 * a [T*dk] (per-token decay per key channel; GDN repeats alpha).             */
void lqo_window_buffered(int dk, int dv, int T, const double *S_base, const double *q,
                         const double *k, const double *v, const double *beta,
                         const double *a, double *o, double *S_end)
{
    double *U = (double *)calloc((size_t)T * dv, sizeof(double));
    double *P = (double *)malloc(sizeof(double) * dk);
    double *Q = (double *)malloc(sizeof(double) * dk);
    double *accK = (double *)malloc(sizeof(double) * dv), *accQ = (double *)malloc(sizeof(double) * dv);
    for (int i = 0; i < dk; ++i) P[i] = 1.0;
    for (int t = 0; t < T; ++t) {
        const double *kt = k + (size_t)t * dk, *qt = q + (size_t)t * dk;
        for (int i = 0; i < dk; ++i) P[i] *= a[(size_t)t * dk + i];
        for (int j = 0; j < dv; ++j) {
            double sk = 0.0, sq = 0.0;
            for (int i = 0; i < dk; ++i) {
                sk += S_base[i * dv + j] * P[i] * kt[i];
                sq += S_base[i * dv + j] * P[i] * qt[i];
            }
            accK[j] = sk; accQ[j] = sq;
        }
        for (int m = 0; m < t; ++m) {
            for (int i = 0; i < dk; ++i) {
                double prod = 1.0;
                for (int s = m + 1; s <= t; ++s) prod *= a[(size_t)s * dk + i];
                Q[i] = prod * k[(size_t)m * dk + i];
            }
            double ck = 0.0, cq = 0.0;
            for (int i = 0; i < dk; ++i) { ck += Q[i] * kt[i]; cq += Q[i] * qt[i]; }
            for (int j = 0; j < dv; ++j) {
                accK[j] += ck * U[(size_t)m * dv + j];
                accQ[j] += cq * U[(size_t)m * dv + j];
            }
        }
        double kq = 0.0;
        for (int i = 0; i < dk; ++i) kq += kt[i] * qt[i];
        for (int j = 0; j < dv; ++j) {
            double u = beta[t] * (v[(size_t)t * dv + j] - accK[j]);
            U[(size_t)t * dv + j] = u;
            o[(size_t)t * dv + j] = accQ[j] + kq * u;
        }
    }
    if (S_end) {
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S_end[i * dv + j] = P[i] * S_base[i * dv + j];
        for (int m = 0; m < T; ++m) {
            for (int i = 0; i < dk; ++i) {
                double prod = 1.0;
                for (int s = m + 1; s < T; ++s) prod *= a[(size_t)s * dk + i];
                Q[i] = prod * k[(size_t)m * dk + i];
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S_end[i * dv + j] += Q[i] * U[(size_t)m * dv + j];
        }
    }
    free(U); free(P); free(Q); free(accK); free(accQ);
}

/* ------------------------------------------------------------------------ */
/* Packed code rows.  A row is the dk codes of one value column, key index
 * ascending, in groups of 16 codes:
 *   8-bit: 16 bytes, byte b = code b (two's complement).
 *   4-bit:  8 bytes, byte b holds code 2b in its low nibble and code 2b+1 in
 *           its high nibble (4-bit two's complement).
 *   6-bit: 12 bytes = three little-endian 32-bit words w0, w1, w2.  Codes
 *           4q..4q+3 (q = 0, 1, 2) sit in bits 0..5 of bytes 0..3 of w_q.
 *           Code 12+b (b = 0..3) is split over bits 6..7 of byte b of w0
 *           (code bits 0..1), of w1 (bits 2..3) and of w2 (bits 4..5).
 *           Every code is 6-bit two's complement; 4 codes per 3 bytes.       */
int lqo_row_bytes(int bits, int dk) { return dk * bits / 8; }

void lqo_pack_rows(int bits, int dk, int rows, const int8_t *codes, uint8_t *out)
{
    const int rb = lqo_row_bytes(bits, dk);
    for (int j = 0; j < rows; ++j) {
        const int8_t *c = codes + (size_t)j * dk;
        uint8_t *o = out + (size_t)j * rb;
        for (int g = 0; g < dk / 16; ++g) {
            const int8_t *cg = c + 16 * g;
            if (bits == 8) {
                for (int b = 0; b < 16; ++b) o[16 * g + b] = (uint8_t)cg[b];
            } else if (bits == 4) {
                for (int b = 0; b < 8; ++b)
                    o[8 * g + b] = (uint8_t)(((uint8_t)cg[2 * b] & 0xF) | (((uint8_t)cg[2 * b + 1] & 0xF) << 4));
            } else {
                uint8_t *og = o + 12 * g;
                for (int q = 0; q < 3; ++q)
                    for (int b = 0; b < 4; ++b) {
                        unsigned lo = (unsigned)(uint8_t)cg[4 * q + b] & 0x3F;
                        unsigned hi = (((unsigned)(uint8_t)cg[12 + b] & 0x3F) >> (2 * q)) & 0x3;
                        og[4 * q + b] = (uint8_t)(lo | (hi << 6));
                    }
            }
        }
    }
}

static int sext(unsigned x, int nbits)
{
    int s = (int)(x & ((1u << nbits) - 1));
    return (s & (1 << (nbits - 1))) ? s - (1 << nbits) : s;
}

void lqo_unpack_rows(int bits, int dk, int rows, const uint8_t *in, int8_t *codes)
{
    const int rb = lqo_row_bytes(bits, dk);
    for (int j = 0; j < rows; ++j) {
        const uint8_t *r = in + (size_t)j * rb;
        int8_t *c = codes + (size_t)j * dk;
        for (int g = 0; g < dk / 16; ++g) {
            int8_t *cg = c + 16 * g;
            if (bits == 8) {
                for (int b = 0; b < 16; ++b) cg[b] = (int8_t)r[16 * g + b];
            } else if (bits == 4) {
                for (int b = 0; b < 8; ++b) {
                    cg[2 * b] = (int8_t)sext(r[8 * g + b] & 0xF, 4);
                    cg[2 * b + 1] = (int8_t)sext(r[8 * g + b] >> 4, 4);
                }
            } else {
                const uint8_t *rg = r + 12 * g;
                for (int q = 0; q < 3; ++q)
                    for (int b = 0; b < 4; ++b) cg[4 * q + b] = (int8_t)sext(rg[4 * q + b] & 0x3F, 6);
                for (int b = 0; b < 4; ++b) {
                    unsigned x = (unsigned)(rg[b] >> 6) | ((unsigned)(rg[4 + b] >> 6) << 2) |
                                 ((unsigned)(rg[8 + b] >> 6) << 4);
                    cg[12 + b] = (int8_t)sext(x, 6);
                }
            }
        }
    }
}
