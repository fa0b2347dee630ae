/*
 * tri_oracle.c - plain, slow CPU oracle for TriAttention key scoring, top-B
 * selection and K/V compaction.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no source,
 * header, table or helper with the CUDA library, and neither one includes or
 * links the other.
 *
 * Arithmetic is fp64 with long double (x87 80-bit) phases: every RoPE angle
 * omega_f * n is formed in long double and handed to cosl/sinl, so an angle of
 * 2.6e5 rad carries ~1e-14 rad of error instead of the ~3e-11 of plain double.
 *
 * What the method computes, and where it is stated:
 *  - "TriAttention：基于三角函数 KV 压缩的高效长推理" (whatsmy.fun paper digest),
 *    section 流程详解 (pipeline):
 *      step 1: pre-RoPE query/key centres are extracted ahead of time;
 *      step 2: the pre-RoPE q.k inner product is a sum of sinusoids in the
 *              token distance, which scores each cached key;
 *      step 3: the distance score is combined with Q/K norm magnitudes;
 *      step 4: only the most important KV pairs are kept.
 *    section 核心洞见 (key insight): pre-RoPE Q and K cluster around fixed,
 *    position-stable centres.
 *  - "WeianMao/triattention" project card, section "How it works": keys are
 *    scored from the query centres and norms through a trigonometric series.
 *  The pages give the method in words only.  The exact rule written out below
 *  (the method statement this library implements) is
 *
 *    S_j = (1/G) sum_g [ sum_f |qbar_f^g| |k_f| sum_delta cos(w_f (p_now + delta - j) + phi_f^g)
 *                        + sum_f (E|q_f^g| - |qbar_f^g|) |k_f| ],
 *    w_f = theta^(-2f/d),  phi_f^g = arg qbar_f^g - arg k_f,
 *
 *  with k the pre-RoPE key at position j, pairs (f, f + d/2) (rotate-half
 *  RoPE) or (2f, 2f + 1) (interleaved RoPE), g over the G query heads of one
 *  KV head, and delta over the offset set.  Selection keeps the last W slots plus the top (B - W) of the rest,
 *  ordered by (score descending, slot descending); compaction is a stable
 *  gather by the kept slots.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef long double ldbl;

/* w_f = theta^(-2f/d), the RoPE angular frequency of pair f. */
static ldbl omega_l(double theta, int d, int f)
{
    return powl((ldbl)theta, -2.0L * (ldbl)f / (ldbl)d);
}

double ora_omega(double theta, int d, int f) { return (double)omega_l(theta, d, f); }

int ora_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* The two dimensions of frequency pair f: (f, f + d/2) for rotate-half RoPE
 * (GPT-NeoX / Llama-HF / Qwen layout), (2f, 2f + 1) for interleaved RoPE
 * (GPT-J / Meta-Llama complex layout).  The first is the real part. */
static void pair_dims(int d, int interleaved, int f, int *ire, int *iim)
{
    if (interleaved) {
        *ire = 2 * f;
        *iim = 2 * f + 1;
    } else {
        *ire = f;
        *iim = f + d / 2;
    }
}

/* Pre-RoPE pair f of a cached key.  post_rope != 0: the cache holds
 * k_post_f = k_pre_f * e^{i w_f pos}, so multiply by e^{-i w_f pos}. */
static void key_pair(int d, int il, const double *key, int f, int post_rope, ldbl w,
                     int64_t pos, ldbl *re, ldbl *im)
{
    int ire, iim;
    pair_dims(d, il, f, &ire, &iim);
    ldbl xr = key[ire], xi = key[iim];
    if (post_rope) {
        ldbl a = w * (ldbl)pos;
        ldbl c = cosl(a), s = sinl(a);
        *re = xr * c + xi * s;
        *im = xi * c - xr * s;
    } else {
        *re = xr;
        *im = xi;
    }
}

/*
 * One term of the trigonometric series, for one query centre and one key:
 *   T = sum_f |qbar_f| |k_f| cos(w_f * dist + arg qbar_f - arg k_f)
 * qbar: [F][2] (re, im); k: [d] pre-RoPE key, pairs as pair_dims(il).
 * This is the pre-RoPE form of the q.k logit at token distance `dist`
 * (digest, 流程详解 step 2).
 */
double ora_trig_series(int d, int il, double theta, const double *qbar, const double *k, int64_t dist)
{
    const int F = d / 2;
    ldbl s = 0.0L;
    for (int f = 0; f < F; f++) {
        ldbl w = omega_l(theta, d, f);
        ldbl qr = qbar[2 * f], qi = qbar[2 * f + 1];
        int ire, iim;
        pair_dims(d, il, f, &ire, &iim);
        ldbl kr = k[ire], ki = k[iim];
        ldbl phi = atan2l(qi, qr) - atan2l(ki, kr);
        s += hypotl(qr, qi) * hypotl(kr, ki) * cosl(w * (ldbl)dist + phi);
    }
    return (double)s;
}

/*
 * Calibration (digest, 流程详解 step 1): per frequency pair f of one query
 * head, the complex mean of the pre-RoPE queries and the mean of their
 * magnitudes.
 *   q: [nq][d] pre-RoPE queries (pairs as pair_dims(il)); centre: [F][2];
 *   mnorm: [F].
 */
void ora_calib(int d, int il, int64_t nq, const double *q, double *centre, double *mnorm)
{
    const int F = d / 2;
    for (int f = 0; f < F; f++) {
        ldbl sr = 0.0L, si = 0.0L, sn = 0.0L;
        int ire, iim;
        pair_dims(d, il, f, &ire, &iim);
        for (int64_t t = 0; t < nq; t++) {
            ldbl xr = q[t * d + ire], xi = q[t * d + iim];
            sr += xr;
            si += xi;
            sn += hypotl(xr, xi);
        }
        centre[2 * f] = (double)(sr / (ldbl)nq);
        centre[2 * f + 1] = (double)(si / (ldbl)nq);
        mnorm[f] = (double)(sn / (ldbl)nq);
    }
}

/*
 * Literal score: the triple sum over query heads g, pairs f and offsets delta,
 * exactly as the rule above is written (one cosine per (g, f, delta)).
 *   qbar: [G][F][2], mnorm: [G][F] - calibration of the G query heads that
 *         share this KV head.
 *   keys: [n][d] cached keys, pos: [n] their positions.
 *   post_rope: 1 if the cache holds RoPE-rotated keys (they are de-rotated
 *         by their own position first), 0 if it holds pre-RoPE keys.
 *   offsets: [n_off] future offsets delta.
 *   il: 1 for interleaved RoPE pairs, 0 for rotate-half (pair_dims).
 *   out: [n] scores.
 */
void ora_score_literal(int d, int il, double theta, int G, const double *qbar, const double *mnorm,
                       int64_t n, const double *keys, const int64_t *pos, int post_rope,
                       int64_t p_now, int n_off, const int64_t *offsets, double *out)
{
    const int F = d / 2;
    ldbl *w = malloc(sizeof(ldbl) * F);
    ldbl *qn = malloc(sizeof(ldbl) * G * F);
    ldbl *qa = malloc(sizeof(ldbl) * G * F);
    for (int f = 0; f < F; f++) w[f] = omega_l(theta, d, f);
    for (int g = 0; g < G; g++)
        for (int f = 0; f < F; f++) {
            ldbl qr = qbar[(g * F + f) * 2], qi = qbar[(g * F + f) * 2 + 1];
            qn[g * F + f] = hypotl(qr, qi);
            qa[g * F + f] = atan2l(qi, qr);
        }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++) {
        ldbl total = 0.0L;
        for (int g = 0; g < G; g++) {
            ldbl sg = 0.0L;
            for (int f = 0; f < F; f++) {
                ldbl kr, ki;
                key_pair(d, il, keys + j * d, f, post_rope, w[f], pos[j], &kr, &ki);
                ldbl kn = hypotl(kr, ki);
                ldbl phi = qa[g * F + f] - atan2l(ki, kr);
                ldbl trig = 0.0L;
                for (int e = 0; e < n_off; e++)
                    trig += cosl(w[f] * (ldbl)(p_now + offsets[e] - pos[j]) + phi);
                sg += qn[g * F + f] * kn * trig + ((ldbl)mnorm[g * F + f] - qn[g * F + f]) * kn;
            }
            total += sg;
        }
        out[j] = (double)(total / (ldbl)G);
    }
    free(w);
    free(qn);
    free(qa);
}

/*
 * Collapsed score: the same rule with the delta sum folded by angle addition,
 *   sum_delta cos(x + w_f delta) = Re(e^{ix} * sum_delta e^{i w_f delta}),
 * so there is one (cos, sin) per (key, g, f) of x = w_f (p_now - j) + phi.
 * Arguments as for ora_score_literal.
 */
void ora_score_collapsed(int d, int il, double theta, int G, const double *qbar, const double *mnorm,
                         int64_t n, const double *keys, const int64_t *pos, int post_rope,
                         int64_t p_now, int n_off, const int64_t *offsets, double *out)
{
    const int F = d / 2;
    ldbl *w = malloc(sizeof(ldbl) * F);
    ldbl *sr = malloc(sizeof(ldbl) * F);
    ldbl *si = malloc(sizeof(ldbl) * F);
    ldbl *qn = malloc(sizeof(ldbl) * G * F);
    ldbl *qa = malloc(sizeof(ldbl) * G * F);
    for (int f = 0; f < F; f++) {
        w[f] = omega_l(theta, d, f);
        sr[f] = 0.0L;
        si[f] = 0.0L;
        for (int e = 0; e < n_off; e++) {
            sr[f] += cosl(w[f] * (ldbl)offsets[e]);
            si[f] += sinl(w[f] * (ldbl)offsets[e]);
        }
    }
    for (int g = 0; g < G; g++)
        for (int f = 0; f < F; f++) {
            ldbl qr = qbar[(g * F + f) * 2], qi = qbar[(g * F + f) * 2 + 1];
            qn[g * F + f] = hypotl(qr, qi);
            qa[g * F + f] = atan2l(qi, qr);
        }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++) {
        ldbl total = 0.0L;
        for (int g = 0; g < G; g++) {
            ldbl sg = 0.0L;
            for (int f = 0; f < F; f++) {
                ldbl kr, ki;
                key_pair(d, il, keys + j * d, f, post_rope, w[f], pos[j], &kr, &ki);
                ldbl kn = hypotl(kr, ki);
                ldbl x = w[f] * (ldbl)(p_now - pos[j]) + qa[g * F + f] - atan2l(ki, kr);
                ldbl trig = cosl(x) * sr[f] - sinl(x) * si[f];
                sg += qn[g * F + f] * kn * trig + ((ldbl)mnorm[g * F + f] - qn[g * F + f]) * kn;
            }
            total += sg;
        }
        out[j] = (double)(total / (ldbl)G);
    }
    free(w);
    free(sr);
    free(si);
    free(qn);
    free(qa);
}

/*
 * Absorbed score: the rule rewritten as a linear form in the cached pair plus
 * the norm term,
 *   S_j = sum_f Re(A_f * conj(k_f)) + c_f |k_f|,
 *   A_f = (1/G) sum_g qbar_f^g * e^{i w_f p_now} * sum_delta e^{i w_f delta}
 *         (post_rope = 1: k_f is the cached, rotated pair; the key's own
 *          rotation e^{i w_f j} cancels the -j of the distance),
 *   A_f = (1/G) sum_g qbar_f^g * sum_delta e^{i w_f delta} * e^{i w_f (p_now - j)}
 *         (post_rope = 0: the cache holds pre-RoPE pairs),
 *   c_f = (1/G) sum_g (E|q_f^g| - |qbar_f^g|).
 * Kept only to cross-check that identity against the literal form.
 */
void ora_score_absorbed(int d, int il, double theta, int G, const double *qbar, const double *mnorm,
                        int64_t n, const double *keys, const int64_t *pos, int post_rope,
                        int64_t p_now, int n_off, const int64_t *offsets, double *out)
{
    const int F = d / 2;
    ldbl *w = malloc(sizeof(ldbl) * F);
    ldbl *ar = malloc(sizeof(ldbl) * F);
    ldbl *ai = malloc(sizeof(ldbl) * F);
    ldbl *cf = malloc(sizeof(ldbl) * F);
    for (int f = 0; f < F; f++) {
        w[f] = omega_l(theta, d, f);
        ldbl sr = 0.0L, si = 0.0L;
        for (int e = 0; e < n_off; e++) {
            sr += cosl(w[f] * (ldbl)offsets[e]);
            si += sinl(w[f] * (ldbl)offsets[e]);
        }
        ldbl mr = 0.0L, mi = 0.0L, c = 0.0L;
        for (int g = 0; g < G; g++) {
            ldbl qr = qbar[(g * F + f) * 2], qi = qbar[(g * F + f) * 2 + 1];
            mr += qr;
            mi += qi;
            c += (ldbl)mnorm[g * F + f] - hypotl(qr, qi);
        }
        mr /= (ldbl)G;
        mi /= (ldbl)G;
        /* (mr + i mi) * (sr + i si) */
        ldbl tr = mr * sr - mi * si, ti = mr * si + mi * sr;
        if (post_rope) {
            ldbl a = w[f] * (ldbl)p_now, ec = cosl(a), es = sinl(a);
            ar[f] = tr * ec - ti * es;
            ai[f] = tr * es + ti * ec;
        } else {
            ar[f] = tr;
            ai[f] = ti;
        }
        cf[f] = c / (ldbl)G;
    }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++) {
        ldbl s = 0.0L;
        for (int f = 0; f < F; f++) {
            int ire, iim;
            pair_dims(d, il, f, &ire, &iim);
            ldbl kr = keys[j * d + ire], ki = keys[j * d + iim];
            ldbl br = ar[f], bi = ai[f];
            if (!post_rope) {
                ldbl a = w[f] * (ldbl)(p_now - pos[j]), ec = cosl(a), es = sinl(a);
                br = ar[f] * ec - ai[f] * es;
                bi = ar[f] * es + ai[f] * ec;
            }
            s += br * kr + bi * ki + cf[f] * hypotl(kr, ki);
        }
        out[j] = (double)s;
    }
    free(w);
    free(ar);
    free(ai);
    free(cf);
}

/* ---------------------------------------------------------------- select */

typedef struct {
    double s;
    int64_t i;
} ora_entry;

/* Strict total order, "better first": larger score first; equal scores keep
 * the higher (more recent) slot first; NaN ranks below every number. */
static int better_first(const void *pa, const void *pb)
{
    const ora_entry *a = pa, *b = pb;
    int an = isnan(a->s), bn = isnan(b->s);
    if (an != bn) return an ? 1 : -1;
    if (!an && a->s != b->s) return a->s > b->s ? -1 : 1;
    if (a->i != b->i) return a->i > b->i ? -1 : 1;
    return 0;
}

/*
 * Keep-set of one row (digest, 流程详解 step 4; the budget B counts the
 * protected window):
 *   N <= B: every slot is kept;
 *   else:   slots N-W .. N-1 (the W most recent) are kept, plus the B-W best
 *           of slots 0 .. N-W-1 under better_first.
 * kept: [min(N, B)] slots in ascending order.  Returns the count, or -1 when
 * the arguments are invalid (B < 1, W < 0, W > B).
 */
int64_t ora_select(int64_t n, const double *score, int64_t B, int64_t W, int64_t *kept)
{
    if (B < 1 || W < 0 || W > B || n < 0) return -1;
    if (n <= B) {
        for (int64_t j = 0; j < n; j++) kept[j] = j;
        return n;
    }
    const int64_t M = n - W, K = B - W;
    ora_entry *e = malloc(sizeof(ora_entry) * (size_t)(M > 0 ? M : 1));
    unsigned char *keep = calloc((size_t)n, 1);
    for (int64_t j = 0; j < M; j++) {
        e[j].s = score[j];
        e[j].i = j;
    }
    qsort(e, (size_t)M, sizeof(ora_entry), better_first);
    for (int64_t t = 0; t < K; t++) keep[e[t].i] = 1;
    for (int64_t j = M; j < n; j++) keep[j] = 1;
    int64_t c = 0;
    for (int64_t j = 0; j < n; j++)
        if (keep[j]) kept[c++] = j;
    free(e);
    free(keep);
    return c;
}

/* -------------------------------------------------------------- compaction */

/* Stable gather of fixed-width records: dst[t] = src[idx[t]] for t < n. */
void ora_gather_bytes(int64_t n, const int64_t *idx, int64_t width, const unsigned char *src,
                      unsigned char *dst)
{
    for (int64_t t = 0; t < n; t++)
        memcpy(dst + t * width, src + idx[t] * width, (size_t)width);
}

/* ------------------------------------------------- calibration, continued */

/*
 * Online (decode-time) centre update, written as the weighted statistics it
 * maintains.  Queries arrive in n_updates batches; query t came with batch
 * update_of[t] (0 .. n_updates-1), and each later batch multiplies the weight
 * of everything seen before it by `decay` (0 < decay <= 1; 1 keeps the plain
 * mean of every query seen).  So query t carries the weight
 *   w_t = decay^(n_updates - 1 - update_of[t]),
 * and per pair f
 *   centre_f = sum_t w_t q_f(t) / sum_t w_t,   mnorm_f = sum_t w_t |q_f(t)| / sum_t w_t,
 * the centres of digest step 1 over a (decayed) stream of queries.
 *   q: [nq][d] pre-RoPE queries of one head; centre: [F][2]; mnorm: [F].
 */
void ora_calib_online(int d, int il, int64_t nq, const double *q, const int64_t *update_of,
                      int64_t n_updates, double decay, double *centre, double *mnorm)
{
    const int F = d / 2;
    for (int f = 0; f < F; f++) {
        int ire, iim;
        pair_dims(d, il, f, &ire, &iim);
        ldbl sr = 0.0L, si = 0.0L, sn = 0.0L, sw = 0.0L;
        for (int64_t t = 0; t < nq; t++) {
            ldbl w = powl((ldbl)decay, (ldbl)(n_updates - 1 - update_of[t]));
            ldbl xr = q[t * d + ire], xi = q[t * d + iim];
            sr += w * xr;
            si += w * xi;
            sn += w * hypotl(xr, xi);
            sw += w;
        }
        centre[2 * f] = (double)(sr / sw);
        centre[2 * f + 1] = (double)(si / sw);
        mnorm[f] = (double)(sn / sw);
    }
}

/*
 * Key centres (digest, 流程详解 step 1: the pre-RoPE centres of Q *and* K): per
 * pair f of one cache row, the complex mean of the pre-RoPE keys and the mean
 * of their magnitudes.  post_rope != 0: the cached keys are de-rotated by their
 * own positions first (key_pair).  An empty row has centre 0 and mnorm 0.
 *   keys: [n][d], pos: [n]; centre: [F][2]; mnorm: [F].
 */
void ora_key_centres(int d, int il, double theta, int64_t n, const double *keys, const int64_t *pos,
                     int post_rope, double *centre, double *mnorm)
{
    const int F = d / 2;
    for (int f = 0; f < F; f++) {
        ldbl w = omega_l(theta, d, f);
        ldbl sr = 0.0L, si = 0.0L, sn = 0.0L;
        for (int64_t j = 0; j < n; j++) {
            ldbl kr, ki;
            key_pair(d, il, keys + j * d, f, post_rope, w, pos[j], &kr, &ki);
            sr += kr;
            si += ki;
            sn += hypotl(kr, ki);
        }
        centre[2 * f] = n ? (double)(sr / (ldbl)n) : 0.0;
        centre[2 * f + 1] = n ? (double)(si / (ldbl)n) : 0.0;
        mnorm[f] = n ? (double)(sn / (ldbl)n) : 0.0;
    }
}

/*
 * Concentration and drift of one head's statistics (the pages name Q/K
 * concentration as the premise, digest section 核心洞见, and the sensitivity
 * of the calibration to a shift between calibration and deployment data as an
 * open risk, digest sections 不足 and 复现注意事项):
 *   conc[f]  = |centre_f| / mnorm_f      (1: every query on the centre's
 *              direction; near 0: directions spread out; 0 when mnorm_f = 0)
 *   head[0]  = sum_f |centre_f| / sum_f mnorm_f      (0 when the sum is 0)
 *   head[1]  = sum_f (|centre_f - ref_f| + |mnorm_f - ref_mnorm_f|) / sum_f ref_mnorm_f
 *              (0 without a reference or when its norm sum is 0): the
 *              relative L1 change of the two statistics the score uses.
 *   centre, ref: [F][2]; mnorm, ref_mnorm: [F]; conc: [F]; head: [2].
 */
void ora_calib_stats(int F, const double *centre, const double *mnorm, const double *ref,
                     const double *ref_mnorm, double *conc, double *head)
{
    ldbl sc = 0.0L, sm = 0.0L, dd = 0.0L, rm = 0.0L;
    for (int f = 0; f < F; f++) {
        ldbl a = hypotl(centre[2 * f], centre[2 * f + 1]);
        conc[f] = mnorm[f] > 0.0 ? (double)(a / (ldbl)mnorm[f]) : 0.0;
        sc += a;
        sm += mnorm[f];
        if (ref) {
            dd += hypotl((ldbl)centre[2 * f] - ref[2 * f], (ldbl)centre[2 * f + 1] - ref[2 * f + 1]);
            dd += fabsl((ldbl)mnorm[f] - ref_mnorm[f]);
            rm += ref_mnorm[f];
        }
    }
    head[0] = sm > 0.0L ? (double)(sc / sm) : 0.0;
    head[1] = (ref && rm > 0.0L) ? (double)(dd / rm) : 0.0;
}

/* ------------------------------------------------ attention over the cache */

/*
 * Decode attention of one query over one (compressed) cache row (digest,
 * 流程详解 step 5: all later attention runs over the compressed cache):
 *   s_j = scale * (q . k_j),   out = sum_j e^{s_j} v_j / sum_j e^{s_j},
 *   lse = log sum_j e^{s_j}
 * taken with the maximum subtracted first (softmax definition; long double).
 * An empty row gives out = 0 and lse = -inf.
 *   q: [d] (already RoPE'd at its position); keys, values: [n][d]; out: [d].
 */
void ora_attention(int d, int64_t n, const double *q, const double *keys, const double *values, double scale,
                   double *out, double *lse)
{
    for (int t = 0; t < d; t++) out[t] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return;
    }
    ldbl *s = malloc(sizeof(ldbl) * (size_t)n);
    ldbl m = -INFINITY;
    for (int64_t j = 0; j < n; j++) {
        ldbl a = 0.0L;
        for (int t = 0; t < d; t++) a += (ldbl)q[t] * (ldbl)keys[j * d + t];
        s[j] = (ldbl)scale * a;
        if (s[j] > m) m = s[j];
    }
    ldbl den = 0.0L;
    ldbl *acc = calloc((size_t)d, sizeof(ldbl));
    for (int64_t j = 0; j < n; j++) {
        ldbl p = expl(s[j] - m);
        den += p;
        for (int t = 0; t < d; t++) acc[t] += p * (ldbl)values[j * d + t];
    }
    for (int t = 0; t < d; t++) out[t] = (double)(acc[t] / den);
    *lse = (double)(m + logl(den));
    free(s);
    free(acc);
}
