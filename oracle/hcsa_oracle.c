/*
 * CPU oracle for hybrid compressed attention (CSA / HCA) -- TEST
 * INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library; the product path never
 * does.  It shares no code with the CUDA library.
 *
 * Plain, slow and literal: every value is a double, every loop follows the
 * definition, results are rounded to the storage format (fp32 or bf16,
 * round-to-nearest-even) exactly where the layer stores a tensor.  OpenMP
 * only splits independent entries / queries across threads.
 *
 * What is computed (DeepSeek-V4 hybrid attention as described on the pages
 * "DeepSeek-V4: interleaved compressed attention ..." (TL;DR, three-tier
 * diagram) and "DeepSeek-V4 ... KV cache compressed attention" (sections
 * "CSA: compresion 4x ...", "HCA: compresion 128x ...", "Ventana
 * deslizante"), with the operator fixed by the CSA fp32 T=2048 workload
 * definition):
 *
 *   pool (learned compressor, CSA m=4 width 8 / HCA m=128 width 128):
 *     entry j pools tokens i in [m j - (W - m), m j + m) intersected with [0, T);
 *     per channel c: c_j[c] = sum_i softmax_i(g[i,c] + B[i - m j + (W - m), c]) kv[i,c]
 *     indexer key  k_j[d]  = the same pool over ki[i,d], gate channel d (d < di)
 *   indexer score (lightning indexer, CSA):
 *     s[t,j] = sum_h w[t,h] * max(0, sum_d qi[t,h,d] k_j[d]),  j visible iff m j + m <= t
 *   top-k: the min(k, visible) largest s[t,j], equal scores broken by lower j
 *   attention (MQA): keys = selected entries' first half, values = second half,
 *     united with the raw tokens i in (t - window, t] (key / value = halves of kv[i]);
 *     one softmax over the union with scale tau.
 *   HCA attention: the same with every visible entry selected.
 *
 * parity pins live in the tests (closed forms, library special cases, brute
 * force); nothing here is unpinned.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ST_F64 = 0, ST_F32 = 1, ST_BF16 = 2 };

/* round a double to the nearest value of the storage format (ties to even) */
static double store(double v, int st) {
    if (st == ST_F32) return (double)(float)v;
    if (st == ST_BF16) {
        if (v == 0.0 || !isfinite(v)) return v;
        int e;
        frexp(v, &e);                 /* |v| in [2^(e-1), 2^e) */
        int ulp_exp = e - 8;          /* 8 significant bits */
        if (e - 1 < -126) ulp_exp = -133;
        double ulp = ldexp(1.0, ulp_exp);
        return nearbyint(v / ulp) * ulp;
    }
    return v;
}

/* threads the OpenMP loops below use (reported next to the oracle's timings) */
int orc_num_threads(void) { return omp_get_max_threads(); }

void orc_round(double *a, int64_t n, int st) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) a[i] = store(a[i], st);
}

/* ---------------------------------------------------------------------------------------------
 * Low-precision cache storage (page "DeepSeek-V4 ... KV cache ...", section "FP8 y FP4": most of
 * each compressed entry in FP8, the indexer keys in FP4).  The pages fix neither the formats' flavour
 * nor the scaling; the readings taken:
 *   FP8 entries: OCP E4M3 (bias 7, no infinities, largest 448, subnormals down to 2^-9).  Every entry
 *     row is cut into blocks of `block` (32) channels sharing a power-of-two scale 2^e, e the smallest
 *     integer with amax / 2^e <= 448 (no value is clipped); x is stored as the E4M3 value nearest to
 *     x / 2^e (ties to even), times 2^e.  Power-of-two block scales over 32 elements are the shared
 *     scales of the OCP Microscaling formats; a stored value is then exactly a bf16 number.
 *   FP4 indexer keys: OCP E2M1 (0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives).  A block of `block`
 *     channels shares a power-of-two scale 2^e, e the smallest integer with amax / 2^e <= 6 (no value
 *     is clipped); x is stored as the E2M1 value nearest to x / 2^e (ties to the even mantissa), times 2^e.
 * These functions return the stored values (dequantized) in place of the inputs.
 * --------------------------------------------------------------------------------------------- */

/* nearest E4M3 value (ties to even), saturating at +-448 */
static double round_e4m3(double v) {
    if (v == 0.0 || isnan(v)) return v;
    const double a = fabs(v);
    double ulp;
    if (a < ldexp(1.0, -6)) {
        ulp = ldexp(1.0, -9);                 /* subnormals: m / 8 * 2^-6 */
    } else {
        int e;
        frexp(a, &e);                         /* a in [2^(e-1), 2^e) */
        ulp = ldexp(1.0, e - 1 - 3);          /* 3 mantissa bits */
    }
    double q = nearbyint(a / ulp) * ulp;
    if (q > 448.0) q = 448.0;
    return v < 0 ? -q : q;
}

/* nearest E2M1 value (ties to the even mantissa), saturating at +-6 */
static double round_e2m1(double v) {
    if (v == 0.0 || isnan(v)) return v;
    const double a = fabs(v);
    const double ulp = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    double q = nearbyint(a / ulp) * ulp;
    if (q > 6.0) q = 6.0;
    return v < 0 ? -q : q;
}

void orc_round_e4m3(double *a, int64_t n) {
    for (int64_t i = 0; i < n; ++i) a[i] = round_e4m3(a[i]);
}

void orc_round_e2m1(double *a, int64_t n) {
    for (int64_t i = 0; i < n; ++i) a[i] = round_e2m1(a[i]);
}

/* smallest e with amax / 2^e <= top (amax > 0) */
static int block_exponent(double amax, double top) {
    int e = (int)ceil(log2(amax / top));
    while (amax / ldexp(1.0, e) > top) ++e;          /* guard log2 rounding */
    while (amax / ldexp(1.0, e - 1) <= top) --e;
    return e;
}

/* FP8 (E4M3) storage of rows [rows, cols] (row-major, leading dimension cols) in blocks of `block`
 * channels with power-of-two scales; exps[rows][cols / block] receives the scale exponents (may be NULL). */
void orc_store_fp8_rows(double *a, int64_t rows, int cols, int block, int32_t *exps) {
    const int nb = (cols + block - 1) / block;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int b = 0; b < nb; ++b) {
            double *x = a + r * cols + (int64_t)b * block;
            const int n = (b + 1) * block <= cols ? block : cols - b * block;
            double amax = 0.0;
            for (int i = 0; i < n; ++i) amax = fmax(amax, fabs(x[i]));
            const int e = amax > 0.0 ? block_exponent(amax, 448.0) : 0;
            if (exps) exps[r * nb + b] = e;
            const double s = ldexp(1.0, e);
            for (int i = 0; i < n; ++i) x[i] = amax > 0.0 ? round_e4m3(x[i] / s) * s : 0.0;
        }
    }
}

/* FP4 (E2M1) storage of rows [rows, cols] in blocks of `block` channels with power-of-two scales;
 * exps[rows][cols / block] receives the scale exponents (may be NULL). */
void orc_store_fp4_rows(double *a, int64_t rows, int cols, int block, int32_t *exps) {
    const int nb = (cols + block - 1) / block;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int b = 0; b < nb; ++b) {
            double *x = a + r * cols + (int64_t)b * block;
            const int n = (b + 1) * block <= cols ? block : cols - b * block;
            double amax = 0.0;
            for (int i = 0; i < n; ++i) amax = fmax(amax, fabs(x[i]));
            const int e = amax > 0.0 ? block_exponent(amax, 6.0) : 0;
            if (exps) exps[r * nb + b] = e;
            const double s = ldexp(1.0, e);
            for (int i = 0; i < n; ++i) x[i] = amax > 0.0 ? round_e2m1(x[i] / s) * s : 0.0;
        }
    }
}

/* One gated-softmax pool over n tokens for channels [0, nch): the learned
 * compressor of "CSA: compresion 4x mas recuperacion dispersa" (learned pool,
 * overlapping windows) and "HCA: compresion 128x" (m'=128), per channel.
 * kv_rows[i], g_rows[i], b_rows[i] point at token i's value row, gate-logit row
 * and bias row; out[c] receives the pooled value (unrounded). */
static void pool(int n, int nch, const double *const *kv_rows, const double *const *g_rows,
                 const double *const *b_rows, double *out) {
    for (int c = 0; c < nch; ++c) {
        double mx = -INFINITY;
        for (int i = 0; i < n; ++i) {
            double l = g_rows[i][c] + b_rows[i][c];
            if (l > mx) mx = l;
        }
        double z = 0.0, acc = 0.0;
        for (int i = 0; i < n; ++i) {
            double e = exp(g_rows[i][c] + b_rows[i][c] - mx);
            z += e;
            acc += e * kv_rows[i][c];
        }
        out[c] = acc / z;
    }
}

/* Prefill compressor over a whole sequence (CSA m=4 width 8, HCA m=128 width 128;
 * edge entries pool only the tokens inside [0, T), with the bias row given by
 * the token's offset inside the pool window).
 * kv[T, ld_kv] (C used), g[T, ld_g] (C used), bias[W, C], ki[T, ld_ki] (di used, may be NULL).
 * entries[N, C], idx_keys[N, di] with N = ceil(T / m). */
void orc_compress(int64_t T, int C, int m, int W, const double *kv, int64_t ld_kv, const double *g,
                  int64_t ld_g, const double *bias, const double *ki, int64_t ld_ki, int di,
                  double *entries, double *idx_keys, int st) {
    int64_t N = (T + m - 1) / m;
    if (W > 512 || W < m) return;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t j = 0; j < N; ++j) {
        int64_t lo = m * j - (W - m), hi = m * j + m;
        int64_t a = lo < 0 ? 0 : lo, b = hi > T ? T : hi;
        int n = (int)(b - a);
        const double *kvr[512], *gr[512], *br[512], *kir[512];
        for (int i = 0; i < n; ++i) {
            int64_t tok = a + i;
            kvr[i] = kv + tok * ld_kv;
            gr[i] = g + tok * ld_g;
            br[i] = bias + (tok - lo) * C;    /* bias row: position inside the pool window */
            if (ki) kir[i] = ki + tok * ld_ki;
        }
        double *e = entries + j * C;
        pool(n, C, kvr, gr, br, e);
        for (int c = 0; c < C; ++c) e[c] = store(e[c], st);
        if (ki && idx_keys) {
            double *k = idx_keys + j * di;
            pool(n, di, kir, gr, br, k);      /* gate channels [0, di) */
            for (int d = 0; d < di; ++d) k[d] = store(k[d], st);
        }
    }
}

/* Single pool over explicit token rows (decode append): kv_tok/g_tok/b_tok are
 * [n, ld] arrays holding the n tokens in order; out[nch] is rounded to storage. */
void orc_pool_rows(int n, int nch, const double *kv_tok, int64_t ld_kv, const double *g_tok, int64_t ld_g,
                   const double *b_tok, int64_t ld_b, double *out, int st) {
    const double *kvr[512], *gr[512], *br[512];
    if (n > 512) return;
    for (int i = 0; i < n; ++i) {
        kvr[i] = kv_tok + i * ld_kv;
        gr[i] = g_tok + i * ld_g;
        br[i] = b_tok + i * ld_b;
    }
    pool(n, nch, kvr, gr, br, out);
    for (int c = 0; c < nch; ++c) out[c] = store(out[c], st);
}

/* Lightning-indexer scores ("CSA: ... Lightning Indexer para puntuarlos"), ReLU of
 * each head's dot product weighted by the query's head weight, no scale.  qi[nq, Hi*di], w[nq, Hi], keys[N, di];
 * n_vis[q] entries are visible to query q; scores[q, j] = NAN for j >= n_vis[q]. */
void orc_index_scores(int nq, int Hi, int di, const double *qi, const double *w, const double *keys,
                      int64_t N, const int64_t *n_vis, double *scores) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < nq; ++q) {
        const double *qq = qi + (int64_t)q * Hi * di;
        const double *ww = w + (int64_t)q * Hi;
        double *s = scores + (int64_t)q * N;
        for (int64_t j = 0; j < N; ++j) {
            if (j >= n_vis[q]) { s[j] = NAN; continue; }
            const double *k = keys + j * di;
            double acc = 0.0;
            for (int h = 0; h < Hi; ++h) {
                double dot = 0.0;
                for (int d = 0; d < di; ++d) dot += qq[h * di + d] * k[d];
                acc += ww[h] * (dot > 0.0 ? dot : 0.0);
            }
            s[j] = acc;
        }
    }
}

typedef struct { double s; int64_t j; } scored;

/* descending score, then ascending index (so equal scores keep the lower j first) */
static int by_score_then_index(const void *pa, const void *pb) {
    const scored *a = (const scored *)pa, *b = (const scored *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_index(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Top-k selection (page "DeepSeek-V4 ... KV cache ...", section "CSA": the indexer's best-scoring
 * compressed entries are kept), exact, via a library sort on (score descending, index ascending).
 * sel[q, 0..k) = the min(k, n_vis) best entries in ascending j, -1 padded.
 * kth_gap[q] (may be NULL) receives (s_(k) - s_(k+1)) / |s_(k)| (INFINITY when n_vis <= k). */
void orc_topk(int nq, const double *scores, int64_t N, const int64_t *n_vis, int k, int32_t *sel,
              double *kth_gap, double *kth_score) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < nq; ++q) {
        int64_t n = n_vis[q];
        const double *s = scores + (int64_t)q * N;
        scored *v = (scored *)malloc(sizeof(scored) * (n > 0 ? n : 1));
        for (int64_t j = 0; j < n; ++j) { v[j].s = s[j]; v[j].j = j; }
        qsort(v, (size_t)n, sizeof(scored), by_score_then_index);
        int64_t take = n < k ? n : k;
        int32_t *out = sel + (int64_t)q * k;
        for (int64_t i = 0; i < take; ++i) out[i] = (int32_t)v[i].j;
        qsort(out, (size_t)take, sizeof(int32_t), by_index);
        for (int64_t i = take; i < k; ++i) out[i] = -1;
        if (kth_gap) kth_gap[q] = (n > k) ? (v[k - 1].s - v[k].s) / fabs(v[k - 1].s) : INFINITY;
        if (kth_score) kth_score[q] = (n >= k && k > 0) ? v[k - 1].s : (n > 0 ? v[n - 1].s : NAN);
        free(v);
    }
}

/* Attention for nq queries (MQA) over the compressed branch united with the raw
 * sliding window ("Ventana deslizante": compressed long-range K/V concatenated
 * with sliding-window K/V), one softmax over the union.
 * q[nq, ld_q] holds H heads of dh; entries[N, C] and raw[*, ld_raw] hold key|value rows (C = 2 dh used).
 * For query q the key set is { entries[sel[q, i]] : sel[q, i] >= 0 } (sel row length nsel), or, when
 * sel == NULL, entries [0, n_vis[q]); united with { raw[win_rows[q, i]] : win_rows[q, i] >= 0 }
 * (row length nwin).  out[nq, H*dh] rounded to storage. */
void orc_attend(int nq, int H, int dh, double scale, const double *q, int64_t ld_q, const double *entries,
                int C, const int32_t *sel, int nsel, const int64_t *n_vis, const double *raw, int64_t ld_raw,
                const int64_t *win_rows, int nwin, double *out, int st) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int qq = 0; qq < nq; ++qq) {
        int64_t ne = sel ? nsel : n_vis[qq];
        int64_t cap = ne + nwin;
        const double **rows = (const double **)malloc(sizeof(double *) * (cap > 0 ? cap : 1));
        int64_t nk = 0;
        for (int64_t i = 0; i < ne; ++i) {
            int64_t j = sel ? sel[(int64_t)qq * nsel + i] : i;
            if (j >= 0) rows[nk++] = entries + j * C;
        }
        for (int i = 0; i < nwin; ++i) {
            int64_t r = win_rows[(int64_t)qq * nwin + i];
            if (r >= 0) rows[nk++] = raw + r * ld_raw;
        }
        double *logit = (double *)malloc(sizeof(double) * (nk > 0 ? nk : 1));
        for (int h = 0; h < H; ++h) {
            const double *qh = q + (int64_t)qq * ld_q + (int64_t)h * dh;
            double mx = -INFINITY;
            for (int64_t r = 0; r < nk; ++r) {
                double dot = 0.0;
                for (int d = 0; d < dh; ++d) dot += qh[d] * rows[r][d];
                logit[r] = dot * scale;
                if (logit[r] > mx) mx = logit[r];
            }
            double *o = out + (int64_t)qq * H * dh + (int64_t)h * dh;
            for (int d = 0; d < dh; ++d) o[d] = 0.0;
            double z = 0.0;
            for (int64_t r = 0; r < nk; ++r) {
                double p = exp(logit[r] - mx);
                z += p;
                for (int d = 0; d < dh; ++d) o[d] += p * rows[r][C / 2 + d];
            }
            for (int d = 0; d < dh; ++d) o[d] = store(nk ? o[d] / z : 0.0, st);
        }
        free(logit);
        free(rows);
    }
}
