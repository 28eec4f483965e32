/*
 * CPU oracle for decode-step combined sparse attention.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its binding) never calls it, and it shares no code,
 * header or table with that path.
 *
 * Plain, slow, single-threaded C in double precision.  Inputs are the bf16
 * bit patterns the GPU sees (uint16_t), widened exactly to double.  Each
 * function restates one step of the method, in the order the method takes
 * them:
 *
 *   "Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs Without
 *   Retraining", abstract: each remaining full-attention layer attends to a
 *   pinned prefix, a sliding window of recent tokens, and a fixed budget of
 *   the most relevant tokens of the context.
 *
 *   "Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining", section "The
 *   method: sliding window + prefix + query-aware pages, searched per
 *   layer": the relevant tokens are picked per query by Quest-style paged
 *   selection over the (vLLM paged) KV cache.
 *
 * The pages give no formula.  The readings taken here:
 *   - pages hold 16 tokens; a sequence of L tokens has n = ceil(L/16) pages;
 *   - prefix and window are page-granular: every page that overlaps the
 *     first P tokens, or the last W tokens, is attended whole;
 *   - a page's relevance is the Quest upper bound of q.k over the page,
 *     built from the elementwise min and max of its keys:
 *       s_j = sum over the query heads h' of the kv head's group,
 *             sum over d of max(q_h'd * kmin_jd, q_h'd * kmax_jd);
 *   - the budget counts pages; the top-budget candidate pages by
 *     (score descending, page index ascending) are kept, one set per
 *     (sequence, kv head) shared by the group's query heads;
 *   - attention over the kept tokens is ordinary softmax(scale * q.k) v,
 *     scale = 1/sqrt(d).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PAGE 16

static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Step: page index ranges of one sequence of L tokens.
 *   n            = number of pages holding tokens
 *   [0, np)      = pinned-prefix pages (overlap tokens [0, P))
 *   [ws, n)      = sliding-window pages (overlap tokens [L-W, L)), clamped
 *                  so they do not overlap the prefix pages
 *   [np, ws)     = candidate pages, the only ones that are scored.        */
void oracle_page_ranges(int L, int prefix, int window, int *n_out, int *np_out,
                        int *ws_out)
{
    int n = L > 0 ? (L + PAGE - 1) / PAGE : 0;
    int np = (prefix + PAGE - 1) / PAGE;
    if (np > n)
        np = n;
    int ws;
    if (window <= 0) {
        ws = n; /* no window */
    } else {
        int first = L - window;
        if (first < 0)
            first = 0;
        ws = first / PAGE;
    }
    if (ws < np)
        ws = np;
    if (ws > n)
        ws = n;
    *n_out = n;
    *np_out = np;
    *ws_out = ws;
}

/* Step: per-page key bounds.  For sequence b, kv head h and logical page j,
 * kmin/kmax[d] are the min/max of K[t, h, d] over the tokens t of the page
 * that are < L_b.  Output layout [B][Hkv][max_pages][D]; entries of pages
 * j >= n_b are left as they are.  Returns 0, or -1 on a block-table entry
 * outside the pool. */
int oracle_page_bounds(const uint16_t *k_cache, int num_pages, int hkv, int dim,
                       const int32_t *block_table, int max_pages,
                       const int32_t *seq_lens, int batch, double *kmin,
                       double *kmax)
{
    for (int b = 0; b < batch; b++) {
        int L = seq_lens[b];
        int n = L > 0 ? (L + PAGE - 1) / PAGE : 0;
        for (int j = 0; j < n; j++) {
            int phys = block_table[(int64_t)b * max_pages + j];
            if (phys < 0 || phys >= num_pages)
                return -1;
            int valid = L - j * PAGE;
            if (valid > PAGE)
                valid = PAGE;
            for (int h = 0; h < hkv; h++) {
                double *lo = kmin + (((int64_t)b * hkv + h) * max_pages + j) * dim;
                double *hi = kmax + (((int64_t)b * hkv + h) * max_pages + j) * dim;
                for (int d = 0; d < dim; d++) {
                    double mn = INFINITY, mx = -INFINITY;
                    for (int t = 0; t < valid; t++) {
                        int64_t at = (((int64_t)phys * hkv + h) * PAGE + t) * dim + d;
                        double v = widen_bf16(k_cache[at]);
                        if (v < mn)
                            mn = v;
                        if (v > mx)
                            mx = v;
                    }
                    lo[d] = mn;
                    hi[d] = mx;
                }
            }
        }
    }
    return 0;
}

/* Low-precision page metadata (the bounds stored in 8 bits, a quarter of
 * the bytes the scoring reads at head_dim 128; cf. "Faster Than Flash: Fudan
 * FFD Hits 11.6x Kernel Speedup, Pushes Long-Context Decoding to 256K",
 * section "The Hard Constraint on an Old Problem": a low-bit scan of the
 * blocks).  Format: 8-bit floating point E4M3 ("FN" form: 1 sign bit, 4
 * exponent bits with bias 7, 3 mantissa bits; exponent field 0 is
 * subnormal; no infinities; 0x7F / 0xFF are NaN).  To keep the score an
 * upper bound the bounds round OUTWARD: kmin to the largest E4M3 value <=
 * kmin, kmax to the smallest E4M3 value >= kmax.  A bound beyond the format's
 * range (|x| > 448) is stored as the NaN code of its sign and read back as
 * the largest bf16 value of that sign (so it still bounds any bf16 key).
 * Zero is always code 0x00. */

#define BF16_MAX 3.3895313892515355e38 /* 0x7F7F */

/* The value of an E4M3 code, from the format definition (NaN codes: the
 * out-of-range bound of their sign, +-BF16_MAX). */
double oracle_fp8_value(int code)
{
    int sgn = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        v = BF16_MAX;
    else if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -v : v;
}

typedef struct {
    double v;
    int code;
} fp8_entry_t;

static fp8_entry_t fp8_table[256];
static int fp8_count = 0;

static int fp8_cmp(const void *x, const void *y)
{
    double a = ((const fp8_entry_t *)x)->v, b = ((const fp8_entry_t *)y)->v;
    return (a > b) - (a < b);
}

/* Every finite E4M3 value once, ascending (-0 left out: zero is 0x00). */
static void fp8_build_table(void)
{
    if (fp8_count)
        return;
    int n = 0;
    for (int c = 0; c < 256; c++) {
        if ((c & 0x7F) == 0x7F || c == 0x80)
            continue;
        fp8_table[n].v = oracle_fp8_value(c);
        fp8_table[n].code = c;
        n++;
    }
    qsort(fp8_table, n, sizeof(fp8_entry_t), fp8_cmp);
    fp8_count = n;
}

/* Outward rounding of x to E4M3: up != 0 gives the smallest value >= x
 * (0x7F if x > 448), else the largest value <= x (0xFF if x < -448). */
int oracle_fp8_round(double x, int up)
{
    fp8_build_table();
    /* binary search: first entry with value >= x */
    int lo = 0, hi = fp8_count;
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (fp8_table[mid].v < x)
            lo = mid + 1;
        else
            hi = mid;
    }
    if (up)
        return lo < fp8_count ? fp8_table[lo].code : 0x7F;
    if (lo < fp8_count && fp8_table[lo].v == x)
        return fp8_table[lo].code;
    return lo > 0 ? fp8_table[lo - 1].code : 0xFF;
}

/* Step: E4M3 page bounds.  The exact bounds of oracle_page_bounds, each
 * rounded outward: kmin down, kmax up.  Codes [B][Hkv][max_pages][D] for
 * pages j < n_b (others left as they are).  Returns 0, or -1 on a
 * block-table entry outside the pool. */
int oracle_page_bounds_fp8(const uint16_t *k_cache, int num_pages, int hkv, int dim,
                           const int32_t *block_table, int max_pages,
                           const int32_t *seq_lens, int batch, uint8_t *kmin8,
                           uint8_t *kmax8)
{
    int64_t nb = (int64_t)batch * hkv * max_pages * dim;
    double *kmin = (double *)malloc(sizeof(double) * (nb > 0 ? nb : 1));
    double *kmax = (double *)malloc(sizeof(double) * (nb > 0 ? nb : 1));
    int rc = oracle_page_bounds(k_cache, num_pages, hkv, dim, block_table, max_pages,
                                seq_lens, batch, kmin, kmax);
    for (int b = 0; b < batch && rc == 0; b++) {
        int L = seq_lens[b];
        int n = L > 0 ? (L + PAGE - 1) / PAGE : 0;
        for (int h = 0; h < hkv; h++)
            for (int j = 0; j < n; j++) {
                int64_t base = (((int64_t)b * hkv + h) * max_pages + j) * dim;
                for (int d = 0; d < dim; d++) {
                    kmin8[base + d] = (uint8_t)oracle_fp8_round(kmin[base + d], 0);
                    kmax8[base + d] = (uint8_t)oracle_fp8_round(kmax[base + d], 1);
                }
            }
    }
    free(kmin);
    free(kmax);
    return rc;
}

/* Step: score every candidate page with the Quest bound, summed over the
 * query heads that share the kv head.  Written literally, one max per
 * (query head, dimension).  Output [B][Hkv][max_pages]; non-candidate
 * entries are set to NaN. */
void oracle_page_scores(const uint16_t *q, int hq, int hkv, int dim,
                        const double *kmin, const double *kmax, int max_pages,
                        const int32_t *seq_lens, int batch, int prefix,
                        int window, double *scores)
{
    int group = hq / hkv;
    for (int b = 0; b < batch; b++) {
        int n, np, ws;
        oracle_page_ranges(seq_lens[b], prefix, window, &n, &np, &ws);
        for (int h = 0; h < hkv; h++) {
            double *s = scores + ((int64_t)b * hkv + h) * max_pages;
            for (int j = 0; j < max_pages; j++)
                s[j] = NAN;
            for (int j = np; j < ws; j++) {
                const double *lo = kmin + (((int64_t)b * hkv + h) * max_pages + j) * dim;
                const double *hi = kmax + (((int64_t)b * hkv + h) * max_pages + j) * dim;
                double acc = 0.0;
                for (int g = 0; g < group; g++) {
                    const uint16_t *qh = q + ((int64_t)b * hq + h * group + g) * dim;
                    for (int d = 0; d < dim; d++) {
                        double qd = widen_bf16(qh[d]);
                        double a = qd * lo[d], c = qd * hi[d];
                        acc += a > c ? a : c;
                    }
                }
                s[j] = acc;
            }
        }
    }
}

typedef struct {
    double score;
    int page;
} ranked_t;

/* Total order of the selection: higher score first, then lower page. */
static int rank_cmp(const void *x, const void *y)
{
    const ranked_t *a = (const ranked_t *)x, *b = (const ranked_t *)y;
    if (a->score > b->score)
        return -1;
    if (a->score < b->score)
        return 1;
    return (a->page > b->page) - (a->page < b->page);
}

static int int_cmp(const void *x, const void *y)
{
    int a = *(const int *)x, b = *(const int *)y;
    return (a > b) - (a < b);
}

/* Step: fixed-budget selection.  For each (sequence, kv head), sort the
 * candidate pages by (score desc, page asc) and keep the first
 * min(budget, #candidates).  Output sel [B][Hkv][budget] in ascending page
 * order, padded with -1; nsel [B][Hkv]. */
void oracle_select_pages(const double *scores, int hkv, int max_pages,
                         const int32_t *seq_lens, int batch, int prefix,
                         int window, int budget, int32_t *sel, int32_t *nsel)
{
    ranked_t *buf = (ranked_t *)malloc(sizeof(ranked_t) * (max_pages > 0 ? max_pages : 1));
    int *keep = (int *)malloc(sizeof(int) * (budget > 0 ? budget : 1));
    for (int b = 0; b < batch; b++) {
        int n, np, ws;
        oracle_page_ranges(seq_lens[b], prefix, window, &n, &np, &ws);
        for (int h = 0; h < hkv; h++) {
            const double *s = scores + ((int64_t)b * hkv + h) * max_pages;
            int m = 0;
            for (int j = np; j < ws; j++) {
                buf[m].score = s[j];
                buf[m].page = j;
                m++;
            }
            qsort(buf, m, sizeof(ranked_t), rank_cmp);
            int k = budget < m ? budget : m;
            for (int i = 0; i < k; i++)
                keep[i] = buf[i].page;
            qsort(keep, k, sizeof(int), int_cmp);
            int32_t *out = sel + ((int64_t)b * hkv + h) * budget;
            for (int i = 0; i < budget; i++)
                out[i] = i < k ? keep[i] : -1;
            nsel[b * hkv + h] = k;
        }
    }
    free(buf);
    free(keep);
}

/* Top-delta selection ("Faster Than Flash: Fudan FFD Hits 11.6x Kernel
 * Speedup, Pushes Long-Context Decoding to 256K", section "top-delta: Tearing
 * Down "Global Synchronization" Too"): per (sequence, kv head), the d
 * candidate pages with the highest scores (the order of oracle_select_pages)
 * together with every candidate page whose score is within delta of the
 * highest candidate score (s_max - s_j <= delta).  Readings: d and delta are
 * given per call; the union is written in ascending page order, -1 padded to
 * cap, and if it holds more than cap pages the cap best of it (score desc,
 * page asc) are kept.  nsel receives the count written. */
void oracle_select_pages_delta(const double *scores, int hkv, int max_pages,
                               const int32_t *seq_lens, int batch, int prefix,
                               int window, int d, double delta, int cap,
                               int32_t *sel, int32_t *nsel)
{
    ranked_t *buf = (ranked_t *)malloc(sizeof(ranked_t) * (max_pages > 0 ? max_pages : 1));
    int *keep = (int *)malloc(sizeof(int) * (max_pages > 0 ? max_pages : 1));
    for (int b = 0; b < batch; b++) {
        int n, np, ws;
        oracle_page_ranges(seq_lens[b], prefix, window, &n, &np, &ws);
        for (int h = 0; h < hkv; h++) {
            const double *s = scores + ((int64_t)b * hkv + h) * max_pages;
            int m = 0;
            double smax = -INFINITY;
            for (int j = np; j < ws; j++) {
                buf[m].score = s[j];
                buf[m].page = j;
                if (s[j] > smax)
                    smax = s[j];
                m++;
            }
            qsort(buf, m, sizeof(ranked_t), rank_cmp);
            /* the union, in rank order: the first d ranked pages, and every
             * page within delta of the top */
            int k = 0;
            for (int i = 0; i < m; i++) {
                const int in_top = i < d;
                const int near = smax - buf[i].score <= delta;
                if ((in_top || near) && k < cap)
                    keep[k++] = buf[i].page;
            }
            qsort(keep, k, sizeof(int), int_cmp);
            int32_t *out = sel + ((int64_t)b * hkv + h) * cap;
            for (int i = 0; i < cap; i++)
                out[i] = i < k ? keep[i] : -1;
            nsel[b * hkv + h] = k;
        }
    }
    free(buf);
    free(keep);
}

/* Softmax attention of one query head over an explicit token list. */
static void attend_tokens(const uint16_t *qh, const uint16_t *k_cache,
                          const uint16_t *v_cache, int hkv, int h, int dim,
                          const int32_t *bt_row, const int *tokens, int ntok,
                          double scale, double *z, double *out)
{
    for (int d = 0; d < dim; d++)
        out[d] = 0.0;
    if (ntok == 0)
        return;
    double zmax = -INFINITY;
    for (int i = 0; i < ntok; i++) {
        int t = tokens[i];
        int phys = bt_row[t / PAGE];
        const uint16_t *kt = k_cache + (((int64_t)phys * hkv + h) * PAGE + t % PAGE) * dim;
        double dot = 0.0;
        for (int d = 0; d < dim; d++)
            dot += widen_bf16(qh[d]) * widen_bf16(kt[d]);
        z[i] = scale * dot;
        if (z[i] > zmax)
            zmax = z[i];
    }
    double denom = 0.0;
    for (int i = 0; i < ntok; i++) {
        z[i] = exp(z[i] - zmax);
        denom += z[i];
    }
    for (int i = 0; i < ntok; i++) {
        int t = tokens[i];
        int phys = bt_row[t / PAGE];
        const uint16_t *vt = v_cache + (((int64_t)phys * hkv + h) * PAGE + t % PAGE) * dim;
        double p = z[i] / denom;
        for (int d = 0; d < dim; d++)
            out[d] += p * widen_bf16(vt[d]);
    }
}

/* Step: attention over the attended set.  For each (sequence, kv head) the
 * attended pages are prefix pages, window pages and the selected pages
 * sel[b][h][0..nsel) (any order; -1 entries ignored); the attended tokens
 * are the tokens t < L_b of those pages.  dense != 0 attends every token.
 * Output out [B][Hq][D].  scale <= 0 means 1/sqrt(D).  Returns 0, or -1 on
 * a block-table entry outside the pool. */
int oracle_attend(const uint16_t *q, const uint16_t *k_cache,
                  const uint16_t *v_cache, int num_pages, int hq, int hkv,
                  int dim, const int32_t *block_table, int max_pages,
                  const int32_t *seq_lens, int batch, int prefix, int window,
                  const int32_t *sel, int budget, int dense, double scale,
                  double *out)
{
    int group = hq / hkv;
    if (scale <= 0.0)
        scale = 1.0 / sqrt((double)dim);
    int maxtok = max_pages * PAGE;
    int *tokens = (int *)malloc(sizeof(int) * (maxtok > 0 ? maxtok : 1));
    double *z = (double *)malloc(sizeof(double) * (maxtok > 0 ? maxtok : 1));
    unsigned char *use = (unsigned char *)malloc(max_pages > 0 ? max_pages : 1);
    int rc = 0;
    for (int b = 0; b < batch && rc == 0; b++) {
        int L = seq_lens[b];
        int n, np, ws;
        oracle_page_ranges(L, prefix, window, &n, &np, &ws);
        const int32_t *bt_row = block_table + (int64_t)b * max_pages;
        for (int j = 0; j < n; j++) {
            if (bt_row[j] < 0 || bt_row[j] >= num_pages)
                rc = -1;
        }
        if (rc)
            break;
        for (int h = 0; h < hkv; h++) {
            memset(use, 0, max_pages > 0 ? max_pages : 1);
            if (dense) {
                for (int j = 0; j < n; j++)
                    use[j] = 1;
            } else {
                for (int j = 0; j < np; j++)
                    use[j] = 1;
                for (int j = ws; j < n; j++)
                    use[j] = 1;
                const int32_t *s = sel + ((int64_t)b * hkv + h) * budget;
                for (int i = 0; i < budget; i++)
                    if (s[i] >= 0 && s[i] < n)
                        use[s[i]] = 1;
            }
            int ntok = 0;
            for (int t = 0; t < L; t++)
                if (use[t / PAGE])
                    tokens[ntok++] = t;
            for (int g = 0; g < group; g++) {
                int head = h * group + g;
                attend_tokens(q + ((int64_t)b * hq + head) * dim, k_cache, v_cache,
                              hkv, h, dim, bt_row, tokens, ntok, scale, z,
                              out + ((int64_t)b * hq + head) * dim);
            }
        }
    }
    free(tokens);
    free(z);
    free(use);
    return rc;
}

/* The whole decode step: bounds -> scores -> selection -> attention.
 * sel [B][Hkv][budget], nsel [B][Hkv] receive the selection; out [B][Hq][D]. */
int oracle_sparse_decode(const uint16_t *q, const uint16_t *k_cache,
                         const uint16_t *v_cache, int num_pages, int hq, int hkv,
                         int dim, const int32_t *block_table, int max_pages,
                         const int32_t *seq_lens, int batch, int prefix,
                         int window, int budget, double scale, double *out,
                         int32_t *sel, int32_t *nsel)
{
    int64_t nb = (int64_t)batch * hkv * max_pages;
    double *kmin = (double *)malloc(sizeof(double) * (nb * dim > 0 ? nb * dim : 1));
    double *kmax = (double *)malloc(sizeof(double) * (nb * dim > 0 ? nb * dim : 1));
    double *scores = (double *)malloc(sizeof(double) * (nb > 0 ? nb : 1));
    int rc = oracle_page_bounds(k_cache, num_pages, hkv, dim, block_table,
                                max_pages, seq_lens, batch, kmin, kmax);
    if (rc == 0) {
        oracle_page_scores(q, hq, hkv, dim, kmin, kmax, max_pages, seq_lens,
                           batch, prefix, window, scores);
        oracle_select_pages(scores, hkv, max_pages, seq_lens, batch, prefix,
                            window, budget, sel, nsel);
        rc = oracle_attend(q, k_cache, v_cache, num_pages, hq, hkv, dim,
                           block_table, max_pages, seq_lens, batch, prefix,
                           window, sel, budget, 0, scale, out);
    }
    free(kmin);
    free(kmax);
    free(scores);
    return rc;
}
