/*
 * BasisKV decode-attention oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, float64 CPU restatement of what one decode step of the
 * BasisKV hot path computes.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library; the product path
 * (the CUDA library) never does, and the two share no code.
 *
 * Source of the method: "BasisKV: Value Latents for Communication and Key
 * Routing" (arXiv 2026-11), English abstract:
 *   - the Value cache is held only as low-rank latents Z (per KV head basis
 *     B_v turns a latent back into a value);
 *   - the compressed Value cache predicts part of the Key information used
 *     for routing, and a Key-specific residual R stores what Value cannot
 *     recover -- so the routing key is  Khat = Z.W_zk + R.B_r;
 *   - pages are chosen by that routing key, and the original Keys are read
 *     only for the selected pages to compute exact QK scores.
 * The abstract gives no formulas; the plain readings used here are:
 *   page score  S_j = max over the G query heads of the group and over the
 *                     valid tokens t of page j of  q_h . Khat_t   (unscaled);
 *   selection       = the k_b = min(k, n_b) pages of largest S_j, equal
 *                     scores going to the lower page index, listed ascending;
 *   attention       = softmax over the valid tokens of the selected pages of
 *                     scale * q_h . K_t, weighted sum of the latents Z_t,
 *                     then expansion by B_v.
 *
 * Every stored value is widened exactly to double (bf16 bits are shifted
 * into the high half of an IEEE single; fp32 converts exactly), and every
 * sum is accumulated in double.  Khat is formed explicitly per token.
 *
 * Pool layouts (row-major):  z_pool [slots][Hkv][P][r]
 *                            r_pool [slots][Hkv][P][s]
 *                            k_pool [slots][Hkv][P][d]
 *   Keys may instead be stored as int8 codes with one fp32 scale per token
 *   (k_format = ORACLE_KEYS_INT8): k_pool [slots][Hkv][P][d] int8 and
 *   k_scale [slots][Hkv][P]; the key is then K_t = k_scale_t * code_t.  This
 *   follows the lossy key compression with fused decompression of "PackKV:
 *   Reducing KV Cache Memory Footprint through LLM-Aware Lossy Compression"
 *   (abstract), read as symmetric per-token int8; the oracle widens code and
 *   scale exactly and forms their product in double.
 *   query q [B][Hkv*G][d] in the pool dtype; query head h of KV head kvh is
 *   q[b][kvh*G + h].  Bases are fp32: w_zk [Hkv][r][d], b_r [Hkv][s][d],
 *   b_v [Hkv][r][d].  page_table [B][ld_pt] holds the slot of logical page j
 *   of sequence b; seq_lens [B] is the token count L_b.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_F32 = 1 };
enum { ORACLE_KEYS_NATIVE = 0, ORACLE_KEYS_INT8 = 1 };

/* Shape and pointers of one problem.  Mirrored field by field by the ctypes
 * structure in oracle.py. */
typedef struct {
    int32_t batch, num_kv_heads, gqa_group, head_dim, page_size;
    int32_t rank_r, rank_s, topk, dtype, num_slots, ld_pt;
    int32_t latent; /* nonzero: out holds zbar [G][r] per unit, before B_v */
    int32_t k_format; /* ORACLE_KEYS_*: keys in the pool dtype, or int8 codes */
    double softmax_scale;
    const void *q, *z_pool, *r_pool, *k_pool;
    const float *k_scale; /* [slots][Hkv][P] when k_format = ORACLE_KEYS_INT8 */
    const float *w_zk, *b_r, *b_v;
    const int32_t *page_table, *seq_lens;
    const uint8_t *unit_mask; /* [B][Hkv], nonzero = compute; NULL = all */
} oracle_problem;

static double widen(const void *base, size_t idx, int dtype)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Element c of the key stored in pool row `row` (row = offset of the row's
 * element 0 divided by d): the pool value, or code times the row's scale. */
static double key_value(const oracle_problem *p, size_t row, int c)
{
    const size_t idx = row * (size_t)p->head_dim + c;
    if (p->k_format == ORACLE_KEYS_INT8)
        return (double)((const int8_t *)p->k_pool)[idx] * (double)p->k_scale[row];
    return widen(p->k_pool, idx, p->dtype);
}

/* Offset of element 0 of token i of page `slot`, KV head kvh, in a pool whose
 * rows are `width` wide. */
static size_t pool_row(const oracle_problem *p, int slot, int kvh, int i, int width)
{
    return (((size_t)slot * p->num_kv_heads + kvh) * p->page_size + i) * (size_t)width;
}

static int check_problem(const oracle_problem *p)
{
    if (p->batch < 0 || p->num_kv_heads <= 0 || p->gqa_group <= 0 || p->head_dim <= 0 ||
        p->page_size <= 0 || p->rank_r <= 0 || p->rank_s < 0 || p->topk <= 0 ||
        p->num_slots < 0 || p->ld_pt < 0)
        return -1;
    if (p->dtype != ORACLE_BF16 && p->dtype != ORACLE_F32)
        return -1;
    if (p->k_format != ORACLE_KEYS_NATIVE && (p->k_format != ORACLE_KEYS_INT8 || !p->k_scale))
        return -1;
    for (int b = 0; b < p->batch; ++b) {
        int L = p->seq_lens[b];
        if (L < 0) return -1;
        int n = (L + p->page_size - 1) / p->page_size;
        if (n > p->ld_pt) return -1;
        for (int j = 0; j < n; ++j) {
            int slot = p->page_table[(size_t)b * p->ld_pt + j];
            if (slot < 0 || slot >= p->num_slots) return -2;
        }
    }
    return 0;
}

/* Ordering used for the selection: larger score first, lower page first on
 * equal scores. */
typedef struct { double score; int page; } ranked_page;

static int rank_cmp(const void *a, const void *b)
{
    const ranked_page *x = (const ranked_page *)a, *y = (const ranked_page *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->page > y->page) - (x->page < y->page);
}

static int int_cmp(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* Routing for one (sequence b, KV head kvh):
 *   page_scores[j] = S_j for j < n_b, -inf after;
 *   sel[0..k_b) ascending pages, -1 after;  *gap = S_(k_b) - S_(k_b+1)
 *   in the ranked order (+inf when every page is selected). */
static void route_unit(const oracle_problem *p, int b, int kvh,
                       double *page_scores, int32_t *sel, double *gap)
{
    const int G = p->gqa_group, d = p->head_dim, P = p->page_size;
    const int r = p->rank_r, s = p->rank_s;
    const int L = p->seq_lens[b];
    const int n = (L + P - 1) / P;
    const int kb = n < p->topk ? n : p->topk;

    double *khat = (double *)malloc(sizeof(double) * (size_t)d);
    double *qh = (double *)malloc(sizeof(double) * (size_t)G * d);
    ranked_page *order = (ranked_page *)malloc(sizeof(ranked_page) * (size_t)(n > 0 ? n : 1));
    const float *W = p->w_zk + (size_t)kvh * r * d;
    const float *Br = p->b_r + (size_t)kvh * s * d;

    for (int h = 0; h < G; ++h)
        for (int c = 0; c < d; ++c)
            qh[(size_t)h * d + c] =
                widen(p->q, ((size_t)b * p->num_kv_heads * G + (size_t)kvh * G + h) * d + c, p->dtype);

    for (int j = 0; j < p->ld_pt; ++j)
        page_scores[j] = -INFINITY;

    for (int j = 0; j < n; ++j) {
        const int slot = p->page_table[(size_t)b * p->ld_pt + j];
        double best = -INFINITY;
        for (int i = 0; i < P; ++i) {
            const int t = j * P + i;
            if (t >= L) break;
            /* Khat_t = Z_t . W_zk + R_t . B_r, one output channel at a time */
            const size_t zrow = pool_row(p, slot, kvh, i, r);
            const size_t rrow = pool_row(p, slot, kvh, i, s);
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int a = 0; a < r; ++a)
                    acc += widen(p->z_pool, zrow + a, p->dtype) * (double)W[(size_t)a * d + c];
                for (int a = 0; a < s; ++a)
                    acc += widen(p->r_pool, rrow + a, p->dtype) * (double)Br[(size_t)a * d + c];
                khat[c] = acc;
            }
            for (int h = 0; h < G; ++h) {
                double u = 0.0;
                for (int c = 0; c < d; ++c)
                    u += qh[(size_t)h * d + c] * khat[c];
                if (u > best) best = u;
            }
        }
        page_scores[j] = best;
        order[j].score = best;
        order[j].page = j;
    }

    qsort(order, (size_t)n, sizeof(ranked_page), rank_cmp);
    int *chosen = (int *)malloc(sizeof(int) * (size_t)(kb > 0 ? kb : 1));
    for (int i = 0; i < kb; ++i)
        chosen[i] = order[i].page;
    qsort(chosen, (size_t)kb, sizeof(int), int_cmp);
    for (int i = 0; i < p->topk; ++i)
        sel[i] = i < kb ? chosen[i] : -1;
    if (gap)
        *gap = kb < n ? order[kb - 1].score - order[kb].score : INFINITY;

    free(chosen);
    free(order);
    free(qh);
    free(khat);
}

/* Exact attention over the valid tokens of the given pages for every query
 * head of (b, kvh); out is [G][d], or [G][r] in latent mode (the weighted
 * latent zbar itself, the quantity BasisKV keeps in rank-r form until the
 * output projection).  sel holds up to topk page indices, -1 entries are
 * skipped.  A sequence with no selected token gets out = 0. */
static void attend_unit(const oracle_problem *p, int b, int kvh, const int32_t *sel, double *out)
{
    const int G = p->gqa_group, d = p->head_dim, P = p->page_size, r = p->rank_r;
    const int L = p->seq_lens[b];
    const float *Bv = p->b_v + (size_t)kvh * r * d;

    int ntok = 0;
    for (int i = 0; i < p->topk; ++i)
        if (sel[i] >= 0) ntok += P;
    double *score = (double *)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
    size_t *zrow = (size_t *)malloc(sizeof(size_t) * (size_t)(ntok > 0 ? ntok : 1));
    double *qh = (double *)malloc(sizeof(double) * (size_t)d);
    double *zbar = (double *)malloc(sizeof(double) * (size_t)r);

    for (int h = 0; h < G; ++h) {
        const size_t qoff = ((size_t)b * p->num_kv_heads * G + (size_t)kvh * G + h) * d;
        for (int c = 0; c < d; ++c)
            qh[c] = widen(p->q, qoff + c, p->dtype);

        /* exact scores scale * q_h . K_t over the selected valid tokens */
        int m = 0;
        for (int i = 0; i < p->topk; ++i) {
            const int j = sel[i];
            if (j < 0) continue;
            const int slot = p->page_table[(size_t)b * p->ld_pt + j];
            for (int a = 0; a < P; ++a) {
                if (j * P + a >= L) break;
                const size_t krow = pool_row(p, slot, kvh, a, 1);
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += qh[c] * key_value(p, krow, c);
                score[m] = p->softmax_scale * dot;
                zrow[m] = pool_row(p, slot, kvh, a, r);
                ++m;
            }
        }

        const int width = p->latent ? r : d;
        double *o = out + (size_t)h * width;
        if (m == 0) {
            for (int c = 0; c < width; ++c) o[c] = 0.0;
            continue;
        }
        /* softmax weights, then the weighted mean of the latents */
        double mx = -INFINITY;
        for (int t = 0; t < m; ++t)
            if (score[t] > mx) mx = score[t];
        double den = 0.0;
        for (int a = 0; a < r; ++a) zbar[a] = 0.0;
        for (int t = 0; t < m; ++t) {
            const double w = exp(score[t] - mx);
            den += w;
            for (int a = 0; a < r; ++a)
                zbar[a] += w * widen(p->z_pool, zrow[t] + a, p->dtype);
        }
        for (int a = 0; a < r; ++a) zbar[a] /= den;
        if (p->latent) {
            for (int a = 0; a < r; ++a) o[a] = zbar[a];
            continue;
        }
        /* value = latent . B_v */
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int a = 0; a < r; ++a)
                acc += zbar[a] * (double)Bv[(size_t)a * d + c];
            o[c] = acc;
        }
    }
    free(zbar);
    free(qh);
    free(zrow);
    free(score);
}

static int unit_wanted(const oracle_problem *p, int u)
{
    return p->unit_mask == NULL || p->unit_mask[u] != 0;
}

/* Routing for every wanted unit.  page_scores [B][Hkv][ld_pt] (nullable),
 * sel [B][Hkv][topk], gap [B][Hkv] (nullable).  Returns 0, -1 for a bad
 * shape, -2 for a page-table entry outside the pool. */
int oracle_route(const oracle_problem *p, double *page_scores, int32_t *sel, double *gap)
{
    int rc = check_problem(p);
    if (rc) return rc;
    const int U = p->batch * p->num_kv_heads;
    double *scratch = NULL;
    if (!page_scores) {
        scratch = (double *)malloc(sizeof(double) * (size_t)(U > 0 ? U : 1) * (p->ld_pt > 0 ? p->ld_pt : 1));
        page_scores = scratch;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < U; ++u) {
        if (!unit_wanted(p, u)) continue;
        route_unit(p, u / p->num_kv_heads, u % p->num_kv_heads,
                   page_scores + (size_t)u * p->ld_pt, sel + (size_t)u * p->topk,
                   gap ? gap + u : NULL);
    }
    free(scratch);
    return 0;
}

/* Exact attention for every wanted unit over the pages listed in
 * sel [B][Hkv][topk]; out [B][Hkv*G][d]. */
int oracle_attend(const oracle_problem *p, const int32_t *sel, double *out)
{
    int rc = check_problem(p);
    if (rc) return rc;
    const int U = p->batch * p->num_kv_heads;
    for (int u = 0; u < U; ++u) {
        const int b = u / p->num_kv_heads;
        const int n = (p->seq_lens[b] + p->page_size - 1) / p->page_size;
        for (int i = 0; i < p->topk; ++i) {
            int j = sel[(size_t)u * p->topk + i];
            if (j >= n) return -1;
        }
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < U; ++u) {
        if (!unit_wanted(p, u)) continue;
        attend_unit(p, u / p->num_kv_heads, u % p->num_kv_heads, sel + (size_t)u * p->topk,
                    out + (size_t)u * p->gqa_group * (p->latent ? p->rank_r : p->head_dim));
    }
    return 0;
}

/* The whole step: routing (skipped as unnecessary for a unit whose every page
 * is selected, in which case page_scores keeps -inf unless want_scores) and
 * exact attention over the selection. */
int oracle_decode(const oracle_problem *p, int want_scores, double *page_scores,
                  int32_t *sel, double *gap, double *out)
{
    int rc = check_problem(p);
    if (rc) return rc;
    const int U = p->batch * p->num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < U; ++u) {
        if (!unit_wanted(p, u)) continue;
        const int b = u / p->num_kv_heads, kvh = u % p->num_kv_heads;
        const int n = (p->seq_lens[b] + p->page_size - 1) / p->page_size;
        int32_t *su = sel + (size_t)u * p->topk;
        if (n <= p->topk && !want_scores) {
            for (int i = 0; i < p->topk; ++i) su[i] = i < n ? i : -1;
            if (page_scores)
                for (int j = 0; j < p->ld_pt; ++j) page_scores[(size_t)u * p->ld_pt + j] = -INFINITY;
            if (gap) gap[u] = INFINITY;
        } else {
            double *ps = page_scores ? page_scores + (size_t)u * p->ld_pt : NULL;
            double *tmp = NULL;
            if (!ps) ps = tmp = (double *)malloc(sizeof(double) * (size_t)(p->ld_pt > 0 ? p->ld_pt : 1));
            route_unit(p, b, kvh, ps, su, gap ? gap + u : NULL);
            free(tmp);
        }
        attend_unit(p, b, kvh, su, out + (size_t)u * p->gqa_group * (p->latent ? p->rank_r : p->head_dim));
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
