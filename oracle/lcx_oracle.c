/*
 * lcx_oracle.c -- plain, slow, fp64 CPU oracle for RoPE with context-extension
 * frequency scaling and causal softmax attention prefill.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; the two meet only through
 * the seeded input tensors handed to both.
 *
 * Every function restates the pages' definitions directly, in fp64, with no
 * blocking, fusion or reordering beyond the definition.  Threads are used only
 * to run independent rows / keys side by side; each row's arithmetic is the
 * plain definition.
 *
 * Sources (page title, section):
 *  - "Long Context: RoPE / YaRN / NTK / MLA" (mathieu0905.github.io), sections
 *    2.1-2.4 (RoPE), 4.2/4.4 (PI), 5.2/5.4 (NTK-aware), 6.2-6.6 (YaRN),
 *    10.1 (sliding window), 10.2 (attention sinks), 2.4 rope_attention.
 *  - "8.3 长上下文技术" (paper.xwysyy.cn, llm-fullstack-book 08_3), sections
 *    8.3.1 (theta_d = b^(-2d/D)), 8.3.2 (PI, NTK-aware gamma), 8.3.3
 *    (NTK-by-parts ramp, YaRN five-step recipe, sqrt(1/t) = 0.1 ln s + 1),
 *    8.3.4 (FlashAttention is exact: online softmax equals softmax).
 *
 * Parity pins: every function here is pinned by tests/test_oracle_pins.py
 * (printed worked values, closed forms, invariants, brute force).  No function
 * is "parity unpinned".  tests/test_oracle_mutants.py plants single mistakes in
 * copies of this file and checks that those pins fail on each.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>
#include <unistd.h>

#define ORC_NONE 0
#define ORC_PLAIN 1
#define ORC_PI 2
#define ORC_NTK 3
#define ORC_YARN 4
#define ORC_DYNAMIC_NTK 5
#define ORC_FACTORS 6

#define ORC_PAIR_HALF 0
#define ORC_PAIR_INTERLEAVED 1

#define ORC_PI_D 3.14159265358979323846

int orc_version(void) { return 1; }

/*
 * Per-pair angular frequency theta'_i of the chosen mode, in fp64, and the
 * attention scale sqrt(1/t).
 *
 *   theta_i = b^(-2i/D), i in [0, D/2)          (RoPE, 2.1 / 8.3.1)
 *   PLAIN : theta'_i = theta_i
 *   PI    : theta'_i = theta_i / s               (4.2: dividing every theta by
 *                                                 s equals m -> m/s)
 *   NTK   : b' = b * s^(D/(D-2)), theta'_i = b'^(-2i/D)          (5.2 boxed)
 *   YARN  : lambda_i = 2 pi / theta_i, r_i = L_train / lambda_i,
 *           ramp_i = clip((r_i - alpha)/(beta - alpha), 0, 1),
 *           theta'_i = (1 - ramp_i) * theta_i / s + ramp_i * theta_i      (6.2)
 *   NONE  : theta'_i = 0 (identity rotation)
 *   mscale = sqrt(1/t) = 0.1 ln s + 1 for YARN with s > 1, else 1   (6.3, 6.6)
 *
 * Returns 0 on success, 1 on an invalid argument.
 */
int orc_rope_theta_fp64(int mode, int D, double base, double s, int64_t L_train,
                        double alpha, double beta, double *theta_prime, double *mscale)
{
    if (D <= 0 || (D % 2) != 0) return 1;
    if (mode < ORC_NONE || mode > ORC_YARN) return 1;
    if (mode != ORC_NONE && !(base > 1.0)) return 1;
    if ((mode == ORC_PI || mode == ORC_NTK || mode == ORC_YARN) && !(s > 0.0)) return 1;
    if (mode == ORC_NTK && D < 4) return 1;
    if (mode == ORC_YARN && (!(beta > alpha) || L_train <= 0)) return 1;

    int half = D / 2;
    for (int i = 0; i < half; i++) {
        double theta = pow(base, -2.0 * (double)i / (double)D);
        double tp = 0.0;
        if (mode == ORC_NONE) {
            tp = 0.0;
        } else if (mode == ORC_PLAIN) {
            tp = theta;
        } else if (mode == ORC_PI) {
            tp = theta / s;
        } else if (mode == ORC_NTK) {
            double new_base = base * pow(s, (double)D / (double)(D - 2));
            tp = pow(new_base, -2.0 * (double)i / (double)D);
        } else { /* ORC_YARN */
            double wavelength = 2.0 * ORC_PI_D / theta;
            double r = (double)L_train / wavelength;
            double ramp = (r - alpha) / (beta - alpha);
            if (ramp < 0.0) ramp = 0.0;
            if (ramp > 1.0) ramp = 1.0;
            tp = (1.0 - ramp) * (theta / s) + ramp * theta;
        }
        theta_prime[i] = tp;
    }
    *mscale = (mode == ORC_YARN && s > 1.0) ? (0.1 * log(s) + 1.0) : 1.0;
    return 0;
}

/*
 * Table variants that depend on the actual context length seq_len:
 *   DYNAMIC_NTK ("AI Day 9: 长上下文技术", RoPE extension list, item 4 Dynamic
 *     NTK: the base is adjusted at inference time to the actual sequence
 *     length; no change for short sequences): s = seq_len / L_train when
 *     seq_len > L_train, else 1, and the NTK-aware base b' = b s^(D/(D-2)).
 *   FACTORS ("Long Context: RoPE / YaRN / NTK / MLA", 7.3-7.4, LongRoPE):
 *     theta'_i = theta_i / lambda_i with per-pair factors lambda_i; with a
 *     second (short) table, that table is used while seq_len <= L_train.
 *   Both keep mscale = 1.  Other modes ignore seq_len and the factor tables.
 */
int orc_rope_theta_ext(int mode, int D, double base, double s, int64_t L_train, double alpha,
                       double beta, int64_t seq_len, const double *factors,
                       const double *factors_short, double *theta_prime, double *mscale)
{
    if (mode == ORC_DYNAMIC_NTK) {
        if (D < 4 || (D % 2) != 0 || !(base > 1.0) || L_train <= 0 || seq_len <= 0) return 1;
        double se = (seq_len > L_train) ? (double)seq_len / (double)L_train : 1.0;
        if (se == 1.0) return orc_rope_theta_fp64(ORC_PLAIN, D, base, 1.0, L_train, alpha, beta,
                                                  theta_prime, mscale);
        return orc_rope_theta_fp64(ORC_NTK, D, base, se, L_train, alpha, beta, theta_prime,
                                   mscale);
    }
    if (mode == ORC_FACTORS) {
        if (D <= 0 || (D % 2) != 0 || !(base > 1.0) || !factors) return 1;
        const double *lam = (factors_short && seq_len <= L_train) ? factors_short : factors;
        for (int i = 0; i < D / 2; i++) {
            if (!(lam[i] > 0.0) || !isfinite(lam[i])) return 1;
            theta_prime[i] = pow(base, -2.0 * (double)i / (double)D) / lam[i];
        }
        *mscale = 1.0;
        return 0;
    }
    return orc_rope_theta_fp64(mode, D, base, s, L_train, alpha, beta, theta_prime, mscale);
}

/*
 * 1 if the fp64 value v lies within a relative 2^-40 of a midpoint between two
 * adjacent fp32 numbers (where its fp32 rounding could depend on the last bits
 * of the fp64 evaluation), else 0.
 */
static int near_fp32_midpoint(double v)
{
    if (v == 0.0 || !isfinite(v)) return 0;
    float f = (float)v;
    float up = nextafterf(f, INFINITY);
    float dn = nextafterf(f, -INFINITY);
    double mid_up = 0.5 * ((double)f + (double)up);
    double mid_dn = 0.5 * ((double)f + (double)dn);
    double tol = fabs(v) * ldexp(1.0, -40);
    return (fabs(v - mid_up) < tol || fabs(v - mid_dn) < tol) ? 1 : 0;
}

/*
 * The fp32 RoPE table: each theta'_i and mscale rounded once, to nearest even,
 * from fp64.  flags[i] (nullable) is set to 1 where that rounding sits too
 * close to an fp32 midpoint to be trusted bit for bit.
 */
int orc_rope_table_ext(int mode, int D, double base, double s, int64_t L_train,
                       double alpha, double beta, int64_t seq_len, const double *factors,
                       const double *factors_short, float *table, float *mscale,
                       double *theta_fp64, int *flags)
{
    if (D <= 0 || D > 4096 || (D % 2) != 0) return 1;
    double tp[2048];
    double ms;
    int rc = orc_rope_theta_ext(mode, D, base, s, L_train, alpha, beta, seq_len, factors,
                                factors_short, tp, &ms);
    if (rc) return rc;
    for (int i = 0; i < D / 2; i++) {
        table[i] = (float)tp[i];
        if (theta_fp64) theta_fp64[i] = tp[i];
        if (flags) flags[i] = near_fp32_midpoint(tp[i]);
    }
    *mscale = (float)ms;
    if (flags) flags[D / 2] = near_fp32_midpoint(ms);
    return 0;
}

int orc_rope_table(int mode, int D, double base, double s, int64_t L_train,
                   double alpha, double beta, float *table, float *mscale,
                   double *theta_fp64, int *flags)
{
    return orc_rope_table_ext(mode, D, base, s, L_train, alpha, beta, 0, NULL, NULL, table,
                              mscale, theta_fp64, flags);
}

/*
 * Rotate one row x[0..D) at integer position m (2.2 real form):
 *   phi = m * theta_i (exact in fp64: m < 2^31, theta_i an fp32 value),
 *   (x_p, x_q) -> ms * (x_p cos phi - x_q sin phi, x_p sin phi + x_q cos phi),
 * with (p, q) = (i, i + D/2) for HALF pairing (2.4, HuggingFace halves) or
 * (2i, 2i + 1) for INTERLEAVED pairing (2.1 adjacent pairs).
 */
static void rotate_row(const double *x, double *y, int D, int64_t m,
                       const float *table, double ms, int pairing)
{
    int half = D / 2;
    for (int i = 0; i < half; i++) {
        int p = (pairing == ORC_PAIR_HALF) ? i : 2 * i;
        int q = (pairing == ORC_PAIR_HALF) ? i + half : 2 * i + 1;
        double phi = (double)m * (double)table[i];
        double c = cos(phi), sn = sin(phi);
        double xp = x[p], xq = x[q];
        y[p] = ms * (xp * c - xq * sn);
        y[q] = ms * (xp * sn + xq * c);
    }
}

/*
 * y[r] = rotate(x[r]) at position pos[r], for n_rows rows of D fp32 inputs;
 * fp64 outputs.  Returns 0, or 1 on an invalid argument.
 */
int orc_rotate_rows(const float *x, double *y, int64_t n_rows, int D,
                    const int64_t *pos, const float *table, float mscale, int pairing)
{
    if (D <= 0 || (D % 2) != 0 || D > 4096) return 1;
    if (pairing != ORC_PAIR_HALF && pairing != ORC_PAIR_INTERLEAVED) return 1;
    double xr[4096];
    for (int64_t r = 0; r < n_rows; r++) {
        for (int d = 0; d < D; d++) xr[d] = (double)x[r * D + d];
        rotate_row(xr, y + r * D, D, pos[r], table, (double)mscale, pairing);
    }
    return 0;
}

/*
 * Visibility of key j to query i in prefill (queries and keys share
 * positions 0..L-1):
 *   causal      : j <= i                                       (2.4 mask)
 *   window W > 0: i - j < W (W counts the query itself)       (10.1)
 *   sinks S     : keys j < S stay visible to every i >= j      (10.2)
 * causal == 0 means every key j < L is visible (window and sinks unused).
 */
int orc_visible(int64_t i, int64_t j, int64_t L, int causal, int64_t window, int64_t sinks)
{
    if (j < 0 || j >= L || i < 0 || i >= L) return 0;
    if (!causal) return 1;
    if (j > i) return 0;
    if (window <= 0) return 1;
    if (i - j < window) return 1;
    if (j < sinks) return 1;
    return 0;
}

/* Fill an [L, L] byte mask with orc_visible. */
void orc_mask(int64_t L, int causal, int64_t window, int64_t sinks, uint8_t *mask)
{
    for (int64_t i = 0; i < L; i++)
        for (int64_t j = 0; j < L; j++)
            mask[i * L + j] = (uint8_t)orc_visible(i, j, L, causal, window, sinks);
}

/* ------------------------------------------------------------------------ */
/* simple parallel-for over [0, n) with pthreads                             */

typedef void (*orc_body_fn)(void *ctx, int64_t idx);
typedef struct {
    orc_body_fn fn;
    void *ctx;
    int64_t n;
    int64_t next;
    pthread_mutex_t mu;
} orc_pool;

static void *orc_worker(void *arg)
{
    orc_pool *p = (orc_pool *)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        int64_t idx = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (idx >= p->n) break;
        p->fn(p->ctx, idx);
    }
    return NULL;
}

static int orc_threads(int nthreads)
{
    if (nthreads > 0) return nthreads;
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}

static void orc_parallel_for(int64_t n, int nthreads, orc_body_fn fn, void *ctx)
{
    orc_pool p;
    p.fn = fn; p.ctx = ctx; p.n = n; p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    int nt = orc_threads(nthreads);
    if (nt > 256) nt = 256;
    if ((int64_t)nt > n) nt = (int)(n > 0 ? n : 1);
    if (nt <= 1) {
        orc_worker(&p);
    } else {
        pthread_t th[256];
        for (int t = 0; t < nt; t++) pthread_create(&th[t], NULL, orc_worker, &p);
        for (int t = 0; t < nt; t++) pthread_join(th[t], NULL);
    }
    pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------------ */
/* attention rows                                                            */

typedef struct {
    const float *k;          /* [B, Hkv, L, D] contiguous */
    double *kr;              /* [L, D] rotated keys of one (b, kv head) */
    int64_t b, g, Hkv, L, D;
    int64_t pos_offset;
    const float *table;
    double ms;
    int pairing;
} rot_keys_ctx;

static void rot_keys_body(void *vctx, int64_t j)
{
    rot_keys_ctx *c = (rot_keys_ctx *)vctx;
    const float *src = c->k + (((c->b * c->Hkv) + c->g) * c->L + j) * c->D;
    double x[4096];
    for (int64_t d = 0; d < c->D; d++) x[d] = (double)src[d];
    rotate_row(x, c->kr + j * c->D, (int)c->D, c->pos_offset + j, c->table, c->ms, c->pairing);
}

typedef struct {
    const float *q;          /* [nrows, D] raw query rows */
    const int64_t *row_i;    /* query index i of each row */
    const int64_t *sel;      /* rows of this (b, kv head) */
    const double *kr;        /* [L, D] rotated keys */
    const float *v;          /* [B, Hkv, L, D] */
    int64_t b, g, Hkv, L, D;
    int64_t pos_offset;
    const float *table;
    double ms;
    int pairing, causal;
    int64_t window, sinks;
    int64_t k_begin, k_end;  /* only keys k_begin <= j < k_end take part */
    double scale;
    double *o;               /* [nrows, D] */
    double *lse;             /* [nrows] */
} row_ctx;

/*
 * One query row by the plain definition (2.4 rope_attention):
 *   s_j = scale * <q'_i, k'_j> for visible j, p = softmax(s) (two passes:
 *   max, then exp and sum), o_i = sum_j p_j v_j, lse_i = max + ln sum exp.
 */
static void row_body(void *vctx, int64_t t)
{
    row_ctx *c = (row_ctx *)vctx;
    int64_t r = c->sel[t];
    int64_t i = c->row_i[r];
    int64_t D = c->D, L = c->L;
    double qr[4096], x[4096];
    for (int64_t d = 0; d < D; d++) x[d] = (double)c->q[r * D + d];
    rotate_row(x, qr, (int)D, c->pos_offset + i, c->table, c->ms, c->pairing);

    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; j++) {
        if (j < c->k_begin || j >= c->k_end ||
            !orc_visible(i, j, L, c->causal, c->window, c->sinks)) { s[j] = -INFINITY; continue; }
        double dot = 0.0;
        const double *kj = c->kr + j * D;
        for (int64_t d = 0; d < D; d++) dot += qr[d] * kj[d];
        s[j] = c->scale * dot;
        if (s[j] > mx) mx = s[j];
    }
    double *o = c->o + r * D;
    for (int64_t d = 0; d < D; d++) o[d] = 0.0;
    if (mx == -INFINITY) {           /* no visible key: empty sum */
        c->lse[r] = -INFINITY;
        free(s);
        return;
    }
    double Z = 0.0;
    const float *vb = c->v + ((c->b * c->Hkv) + c->g) * L * D;
    for (int64_t j = 0; j < L; j++) {
        if (s[j] == -INFINITY) continue;
        double p = exp(s[j] - mx);
        Z += p;
        const float *vj = vb + j * D;
        for (int64_t d = 0; d < D; d++) o[d] += p * (double)vj[d];
    }
    for (int64_t d = 0; d < D; d++) o[d] /= Z;
    c->lse[r] = mx + log(Z);
    free(s);
}

/*
 * Attention outputs for selected query rows.
 *   q      : [nrows, D] raw (un-rotated) query rows, fp32 values
 *   row_b, row_h, row_i : batch, query head and query index of each row
 *   k, v   : [B, Hkv, L, D] contiguous raw keys / values, fp32 values
 *   table, mscale, pairing : the RoPE table (see orc_rope_table)
 *   pos_offset : position of index 0 (prefill: 0)
 *   scale  : softmax scale (typically 1/sqrt(D))
 *   GQA    : query head h reads kv head floor(h / (Hq / Hkv))
 * Outputs o [nrows, D] and lse [nrows] in fp64.  Keys of one (b, kv head) are
 * rotated once and reused by all selected rows of that head.
 */
int orc_attn_rows_keys(const float *q, const int64_t *row_b, const int64_t *row_h,
                       const int64_t *row_i, int64_t nrows,
                       const float *k, const float *v,
                       int64_t B, int64_t Hq, int64_t Hkv, int64_t L, int64_t D,
                       const float *table, float mscale, int pairing, int64_t pos_offset,
                       int causal, int64_t window, int64_t sinks, int64_t k_begin,
                       int64_t k_end, double scale, double *o, double *lse, int nthreads)
{
    if (k_begin < 0 || k_end < k_begin || k_end > L) return 1;
    if (D <= 0 || D > 4096 || (D % 2) != 0) return 1;
    if (Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0 || L <= 0 || B <= 0) return 1;
    if (!causal && (window != 0 || sinks != 0)) return 1;
    if (window < 0 || sinks < 0) return 1;
    int64_t G = Hq / Hkv;
    for (int64_t r = 0; r < nrows; r++) {
        if (row_b[r] < 0 || row_b[r] >= B || row_h[r] < 0 || row_h[r] >= Hq ||
            row_i[r] < 0 || row_i[r] >= L) return 1;
    }
    int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nrows > 0 ? nrows : 1));
    double *kr = (double *)malloc(sizeof(double) * (size_t)(L * D));
    if (!sel || !kr) { free(sel); free(kr); return 2; }

    for (int64_t b = 0; b < B; b++) {
        for (int64_t g = 0; g < Hkv; g++) {
            int64_t ns = 0;
            for (int64_t r = 0; r < nrows; r++)
                if (row_b[r] == b && row_h[r] / G == g) sel[ns++] = r;
            if (ns == 0) continue;
            rot_keys_ctx rk = {k, kr, b, g, Hkv, L, D, pos_offset, table, (double)mscale, pairing};
            orc_parallel_for(L, nthreads, rot_keys_body, &rk);
            row_ctx rc = {q, row_i, sel, kr, v, b, g, Hkv, L, D, pos_offset, table,
                          (double)mscale, pairing, causal, window, sinks, k_begin, k_end,
                          scale, o, lse};
            orc_parallel_for(ns, nthreads, row_body, &rc);
        }
    }
    free(sel);
    free(kr);
    return 0;
}

/* orc_attn_rows_keys over all keys. */
int orc_attn_rows(const float *q, const int64_t *row_b, const int64_t *row_h,
                  const int64_t *row_i, int64_t nrows,
                  const float *k, const float *v,
                  int64_t B, int64_t Hq, int64_t Hkv, int64_t L, int64_t D,
                  const float *table, float mscale, int pairing, int64_t pos_offset,
                  int causal, int64_t window, int64_t sinks, double scale,
                  double *o, double *lse, int nthreads)
{
    return orc_attn_rows_keys(q, row_b, row_h, row_i, nrows, k, v, B, Hq, Hkv, L, D, table,
                              mscale, pairing, pos_offset, causal, window, sinks, 0, L, scale,
                              o, lse, nthreads);
}

/*
 * Combine partial attention results of the same query rows over disjoint key
 * sets ("8.3 长上下文技术", 8.3.4 online softmax and 8.3.5 Ring Attention step 3:
 * partial outputs are merged by rescaling with their softmax statistics).
 * Part s of a row holds o_s = sum_{j in K_s} e^{s_j} v_j / Z_s and
 * lse_s = ln Z_s (Z_s = sum_{j in K_s} e^{s_j}; an empty K_s has lse_s = -inf).
 * Then Z = sum_s Z_s = e^m sum_s e^{lse_s - m} with m = max_s lse_s, and
 *   o = sum_s Z_s o_s / Z = sum_s e^{lse_s - m} o_s / sum_s e^{lse_s - m},
 *   lse = m + ln sum_s e^{lse_s - m}.
 * o_parts [n_parts, rows, D], lse_parts [n_parts, rows]; o [rows, D], lse [rows].
 * A row whose parts are all empty gets o = 0, lse = -inf.
 */
int orc_merge(const double *o_parts, const double *lse_parts, int64_t n_parts, int64_t rows,
              int64_t D, double *o, double *lse)
{
    if (n_parts <= 0 || rows < 0 || D <= 0) return 1;
    for (int64_t r = 0; r < rows; r++) {
        double m = -INFINITY;
        for (int64_t s = 0; s < n_parts; s++)
            if (lse_parts[s * rows + r] > m) m = lse_parts[s * rows + r];
        double *orow = o + r * D;
        for (int64_t d = 0; d < D; d++) orow[d] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        double z = 0.0;
        for (int64_t s = 0; s < n_parts; s++) {
            double l = lse_parts[s * rows + r];
            if (l == -INFINITY) continue;
            double w = exp(l - m);
            z += w;
            const double *op = o_parts + (s * rows + r) * D;
            for (int64_t d = 0; d < D; d++) orow[d] += w * op[d];
        }
        for (int64_t d = 0; d < D; d++) orow[d] /= z;
        lse[r] = m + log(z);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* decoupled RoPE ("Long Context: RoPE / YaRN / NTK / MLA", 9.5 and 9.7):     */
/* a query is [q_C ; q_R], the key of head h is [k_C^(h) ; k_R] with one      */
/* rotary key k_R shared by all heads, only the d_R-dim parts are rotated    */
/* (RoPE of dimension d_R, mscale on the rotated parts as cos/sin carry it), */
/* scores use 1/sqrt(d_C + d_R) unless a scale is given, values are v^(h).   */

typedef struct {
    const float *q;          /* [nrows, Dc + Dr] raw query rows */
    const int64_t *row_b, *row_h, *row_i;
    const float *kc;         /* [B, Hkv, L, Dc] */
    const double *krr;       /* [B, L, Dr] rotated shared rope keys */
    const float *v;          /* [B, Hkv, L, Dv] */
    int64_t B, Hq, Hkv, L, Dc, Dr, Dv;
    int64_t pos_offset;
    const float *table;
    double ms;
    int pairing, causal;
    int64_t window, sinks;
    double scale;
    double *o, *lse;
} mla_ctx;

static void mla_row(void *vctx, int64_t r)
{
    mla_ctx *c = (mla_ctx *)vctx;
    const int64_t b = c->row_b[r], h = c->row_h[r], i = c->row_i[r];
    const int64_t g = h / (c->Hq / c->Hkv), Dq = c->Dc + c->Dr, L = c->L;
    double xr[4096], qr[4096];
    for (int64_t d = 0; d < c->Dr; d++) xr[d] = (double)c->q[r * Dq + c->Dc + d];
    rotate_row(xr, qr, (int)c->Dr, c->pos_offset + i, c->table, c->ms, c->pairing);
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; j++) {
        if (!orc_visible(i, j, L, c->causal, c->window, c->sinks)) { s[j] = -INFINITY; continue; }
        const float *kc = c->kc + (((b * c->Hkv) + g) * L + j) * c->Dc;
        const double *kr = c->krr + (b * L + j) * c->Dr;
        double dot = 0.0;
        for (int64_t d = 0; d < c->Dc; d++) dot += (double)c->q[r * Dq + d] * (double)kc[d];
        for (int64_t d = 0; d < c->Dr; d++) dot += qr[d] * kr[d];
        s[j] = c->scale * dot;
        if (s[j] > mx) mx = s[j];
    }
    double *o = c->o + r * c->Dv;
    for (int64_t d = 0; d < c->Dv; d++) o[d] = 0.0;
    if (mx == -INFINITY) { c->lse[r] = -INFINITY; free(s); return; }
    double Z = 0.0;
    for (int64_t j = 0; j < L; j++) {
        if (s[j] == -INFINITY) continue;
        double p = exp(s[j] - mx);
        Z += p;
        const float *vj = c->v + (((b * c->Hkv) + g) * L + j) * c->Dv;
        for (int64_t d = 0; d < c->Dv; d++) o[d] += p * (double)vj[d];
    }
    for (int64_t d = 0; d < c->Dv; d++) o[d] /= Z;
    c->lse[r] = mx + log(Z);
    free(s);
}

/*
 * Attention rows with decoupled RoPE.
 *   q  : [nrows, Dc + Dr] raw query rows ([q_C ; q_R])
 *   kc : [B, Hkv, L, Dc] per-head non-rotary keys (Dc may be 0)
 *   kr : [B, L, Dr] raw rotary keys shared by every head
 *   v  : [B, Hkv, L, Dv]
 *   table, mscale, pairing : a RoPE table of dimension Dr
 *   scale : score scale (the caller passes 1/sqrt(Dc + Dr) for the default)
 * Other arguments as orc_attn_rows.  Outputs o [nrows, Dv], lse [nrows].
 */
int orc_attn_rows_mla(const float *q, const int64_t *row_b, const int64_t *row_h,
                      const int64_t *row_i, int64_t nrows, const float *kc, const float *kr,
                      const float *v, int64_t B, int64_t Hq, int64_t Hkv, int64_t L,
                      int64_t Dc, int64_t Dr, int64_t Dv, const float *table, float mscale,
                      int pairing, int64_t pos_offset, int causal, int64_t window,
                      int64_t sinks, double scale, double *o, double *lse, int nthreads)
{
    if (Dc < 0 || Dr <= 0 || (Dr % 2) != 0 || Dv <= 0 || Dc + Dr > 4096 || Dr > 4096) return 1;
    if (Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0 || L <= 0 || B <= 0) return 1;
    if (!causal && (window != 0 || sinks != 0)) return 1;
    if (window < 0 || sinks < 0) return 1;
    for (int64_t r = 0; r < nrows; r++)
        if (row_b[r] < 0 || row_b[r] >= B || row_h[r] < 0 || row_h[r] >= Hq ||
            row_i[r] < 0 || row_i[r] >= L) return 1;
    double *krr = (double *)malloc(sizeof(double) * (size_t)(B * L * Dr));
    if (!krr) return 2;
    double xr[4096];
    for (int64_t t = 0; t < B * L; t++) {
        for (int64_t d = 0; d < Dr; d++) xr[d] = (double)kr[t * Dr + d];
        rotate_row(xr, krr + t * Dr, (int)Dr, pos_offset + t % L, table, (double)mscale,
                   pairing);
    }
    mla_ctx c = {q, row_b, row_h, row_i, kc, krr, v, B, Hq, Hkv, L, Dc, Dr, Dv, pos_offset,
                 table, (double)mscale, pairing, causal, window, sinks, scale, o, lse};
    orc_parallel_for(nrows, nthreads, mla_row, &c);
    free(krr);
    return 0;
}

/* Number of threads orc_attn_rows uses for a given request (0 = all cores). */
int orc_num_threads(int nthreads) { return orc_threads(nthreads); }
