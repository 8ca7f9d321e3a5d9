/*
 * pw_oracle.c -- plain, slow CPU oracle for the PageWeaver prefill hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU-baseline
 * legs of bench.py may load this library.  The product path (the CUDA library and its
 * Python binding) never loads, links or calls it, and it shares no code with that path.
 *
 * What it restates (sources are the pages on "PageWeaver: KV-Guided Query Unions for
 * Sparse Attention", arXiv 2610.11201):
 *   - Abstract: each query keeps its own selected KV pages ("original support") and owns its
 *     complete output; query unions share page loads; FP8 KV throughout; a bounded GPU search
 *     produces query IDs.
 *   - AI Radio episode on the paper, paper summary: within a bounded window, queries whose
 *     selected sets add few new pages are collected greedily; execution size g is fixed
 *     (g = 8) independently of the window W.
 * Readings where the pages are silent (fixed sequence-aligned windows, cost = number of new
 * pages, lowest-index seed and tie-break, ascending member and page order, causal limit on
 * the own page) are stated at each function.
 *
 * Precision: attention in IEEE binary64 throughout.  E4M3 and bf16 inputs are decoded
 * exactly from their bit definitions.
 *
 * Status codes returned match the library's: 0 ok, 1 invalid argument, 3 bad selection,
 * 4 capacity exceeded.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PWO_PAGE 64
#define PWO_D 128

enum { PWO_OK = 0, PWO_ERR_INVALID_ARG = 1, PWO_ERR_BAD_SELECTION = 3, PWO_ERR_CAPACITY = 4 };

/* ---------------------------------------------------------------------------------------
 * Number formats
 * ------------------------------------------------------------------------------------- */

/* FP8 E4M3 ("FN" variant: no infinities, S.1111.111 is NaN), from its bit definition:
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal
 * with value m/8 * 2^-6.  The pages use FP8 KV throughout (Abstract). */
double pwo_e4m3_to_double(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* bf16 is the upper 16 bits of an IEEE binary32; the value converts exactly to binary64. */
double pwo_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* binary64 -> bf16, round to nearest, ties to even, straight from binary64 (no double
 * rounding through binary32).  bf16 keeps 8 significant bits, exponent range of binary32,
 * subnormal quantum 2^-133, overflow to infinity. */
uint16_t pwo_double_to_bf16(double x)
{
    if (isnan(x))
        return 0x7FC0;
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    if (isinf(x))
        return signbit(x) ? 0xFF80 : 0x7F80;
    int e2;
    frexp(x, &e2);                 /* |x| in [2^(e2-1), 2^e2) */
    int qexp = e2 - 8;             /* ulp of an 8-significant-bit number in that binade */
    if (qexp < -133)
        qexp = -133;               /* subnormal range */
    double r = ldexp(x, -qexp);    /* exact: power-of-two scaling */
    double n = nearbyint(r);       /* default rounding mode: to nearest, ties to even */
    double y = ldexp(n, qexp);
    float f = (float)y;            /* y is a bf16 value (or overflows to inf): exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------------------------------
 * Selected page sets
 * ------------------------------------------------------------------------------------- */

static int seq_of(const int32_t *cu, int B, int64_t t)
{
    for (int b = 0; b < B; ++b)
        if (t >= cu[b] && t < cu[b + 1])
            return b;
    return -1;
}

/* S(t, h) as a set: the distinct entries of sel[t, h, :] other than -1, ascending.
 * Returns the count written to out (out has room for kmax). */
static int selected_set(const int32_t *sel, int Hkv, int kmax, int64_t t, int h, int32_t *out)
{
    const int32_t *row = sel + ((size_t)t * Hkv + h) * kmax;
    int n = 0;
    for (int j = 0; j < kmax; ++j) {
        int32_t p = row[j];
        if (p < 0)
            continue;
        int dup = 0;
        for (int i = 0; i < n; ++i)
            if (out[i] == p)
                dup = 1;
        if (!dup)
            out[n++] = p;
    }
    /* insertion sort, ascending */
    for (int i = 1; i < n; ++i) {
        int32_t v = out[i];
        int j = i - 1;
        while (j >= 0 && out[j] > v) {
            out[j + 1] = out[j];
            --j;
        }
        out[j + 1] = v;
    }
    return n;
}

/* Every entry is -1 or a page of the query's own causal prefix: 0 <= p <= own page. */
int pwo_validate(const int32_t *sel, const int32_t *cu, int B, int Hkv, int kmax)
{
    for (int b = 0; b < B; ++b)
        for (int64_t t = cu[b]; t < cu[b + 1]; ++t) {
            int64_t own = (t - cu[b]) / PWO_PAGE;
            for (int h = 0; h < Hkv; ++h)
                for (int j = 0; j < kmax; ++j) {
                    int32_t p = sel[((size_t)t * Hkv + h) * kmax + j];
                    if (p < -1 || p > own)
                        return PWO_ERR_BAD_SELECTION;
                }
        }
    return PWO_OK;
}

/* ---------------------------------------------------------------------------------------
 * Bounded-window greedy grouping
 *
 * Per sequence b and kv head h, tokens 0..len_b-1 are cut into fixed windows
 * [wW, min((w+1)W, len_b)).  Inside a window, while some token is unassigned:
 *   seed = lowest unassigned token; group = {seed}; U = S(seed)
 *   while |group| < g and some token is unassigned:
 *       pick the unassigned c minimising |S(c) \ U| (the number of pages c adds to the
 *       union), lowest token index on ties; add c; U = U u S(c)
 *   emit the group (members ascending) and U (pages ascending).
 * Groups are emitted in (b, h, window, seed) order.  qids hold global token indices.
 * gmeta[3*i] = (b, h, window).  pick_order, if not NULL, receives the members in the order
 * the greedy chose them (seed first), for property tests.
 * ------------------------------------------------------------------------------------- */
int pwo_group(const int32_t *sel, const int32_t *cu, int B, int Hkv, int kmax, int W, int g,
              int64_t cap_groups, int64_t union_cap,
              int32_t *qids, int32_t *gsize, int32_t *gmeta, int32_t *union_off,
              int32_t *union_pages, int32_t *pick_order, int64_t *n_groups_out)
{
    if (!sel || !cu || B < 1 || Hkv < 1 || kmax < 1 || W < 1 || g < 1)
        return PWO_ERR_INVALID_ARG;
    int st = pwo_validate(sel, cu, B, Hkv, kmax);
    if (st != PWO_OK)
        return st;

    int64_t ng = 0, nu = 0;
    if (union_off && cap_groups >= 0)
        union_off[0] = 0;
    int32_t *cand_set = (int32_t *)malloc(sizeof(int32_t) * (size_t)W * kmax);
    int *cand_n = (int *)malloc(sizeof(int) * (size_t)W);
    char *assigned = (char *)malloc((size_t)W);
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)g);
    for (int b = 0; b < B; ++b) {
        int64_t len = cu[b + 1] - cu[b];
        int64_t P = (len + PWO_PAGE - 1) / PWO_PAGE;
        char *in_u = (char *)malloc((size_t)(P > 0 ? P : 1));
        for (int h = 0; h < Hkv; ++h) {
            for (int64_t w = 0; w * W < len; ++w) {
                int64_t lo = w * W;
                int64_t hi = lo + W < len ? lo + W : len;
                int n = (int)(hi - lo);
                for (int c = 0; c < n; ++c) {
                    cand_n[c] = selected_set(sel, Hkv, kmax, cu[b] + lo + c, h,
                                             cand_set + (size_t)c * kmax);
                    assigned[c] = 0;
                }
                int remaining = n;
                while (remaining > 0) {
                    if (ng >= cap_groups) {
                        st = PWO_ERR_CAPACITY;
                        goto done;
                    }
                    int seed = 0;
                    while (assigned[seed])
                        ++seed;
                    memset(in_u, 0, (size_t)P);
                    int m = 0;
                    order[m++] = seed;
                    assigned[seed] = 1;
                    --remaining;
                    for (int i = 0; i < cand_n[seed]; ++i)
                        in_u[cand_set[(size_t)seed * kmax + i]] = 1;
                    while (m < g && remaining > 0) {
                        int best = -1, best_cost = 0;
                        for (int c = 0; c < n; ++c) {
                            if (assigned[c])
                                continue;
                            int cost = 0;
                            for (int i = 0; i < cand_n[c]; ++i)
                                if (!in_u[cand_set[(size_t)c * kmax + i]])
                                    ++cost;
                            if (best < 0 || cost < best_cost) { /* strict: lowest index wins ties */
                                best = c;
                                best_cost = cost;
                            }
                        }
                        order[m++] = best;
                        assigned[best] = 1;
                        --remaining;
                        for (int i = 0; i < cand_n[best]; ++i)
                            in_u[cand_set[(size_t)best * kmax + i]] = 1;
                    }
                    /* emit: members ascending */
                    int32_t *q = qids + ng * g;
                    for (int i = 0; i < g; ++i)
                        q[i] = -1;
                    int k = 0;
                    for (int c = 0; c < n; ++c)
                        for (int i = 0; i < m; ++i)
                            if (order[i] == c)
                                q[k++] = (int32_t)(cu[b] + lo + c);
                    if (pick_order)
                        for (int i = 0; i < g; ++i)
                            pick_order[ng * g + i] = i < m ? (int32_t)(cu[b] + lo + order[i]) : -1;
                    gsize[ng] = m;
                    gmeta[3 * ng + 0] = b;
                    gmeta[3 * ng + 1] = h;
                    gmeta[3 * ng + 2] = (int32_t)w;
                    for (int64_t p = 0; p < P; ++p) {
                        if (!in_u[p])
                            continue;
                        if (nu >= union_cap) {
                            st = PWO_ERR_CAPACITY;
                            goto done;
                        }
                        union_pages[nu++] = (int32_t)p;
                    }
                    ++ng;
                    union_off[ng] = (int32_t)nu;
                }
            }
        }
    done:
        free(in_u);
        if (st != PWO_OK)
            break;
    }
    free(cand_set);
    free(cand_n);
    free(assigned);
    free(order);
    if (n_groups_out)
        *n_groups_out = ng;
    return st;
}

/* ---------------------------------------------------------------------------------------
 * Attention of one query row: the plain definition.
 *
 * Query token t (sequence b, position pos, own page o = pos / 64), query head hq, kv head
 * h = hq / (Hq / Hkv).  Its keys are { 64p + i : p in S(t,h), 0 <= i < 64, 64p + i <= pos },
 * visited in ascending page order, then ascending i.  With s_j = sm_scale * k_scale * (q . k_j)
 * and m = max_j s_j:  O = v_scale * sum_j exp(s_j - m) v_j / sum_j exp(s_j - m).
 * An empty key set gives O = 0.
 * ------------------------------------------------------------------------------------- */
typedef struct {
    const uint16_t *Q;
    const uint8_t *K, *V;
    const int32_t *page_table;
    int max_pages;
    const int32_t *cu;
    int B, Hq, Hkv, kmax;
    const int32_t *sel;
    double k_scale, v_scale, sm_scale;
} pwo_attn_args;

/* keys: list of (page, i) pairs already in visiting order; writes O[128]. */
static void attend(const pwo_attn_args *a, int b, int64_t t, int hq, const int32_t *kp,
                   const int32_t *ki, int nkeys, double *scores, double *O)
{
    int G = a->Hq / a->Hkv;
    int h = hq / G;
    double q[PWO_D];
    for (int d = 0; d < PWO_D; ++d)
        q[d] = pwo_bf16_to_double(a->Q[((size_t)t * a->Hq + hq) * PWO_D + d]);
    for (int d = 0; d < PWO_D; ++d)
        O[d] = 0.0;
    if (nkeys == 0)
        return;
    double m = -INFINITY;
    for (int j = 0; j < nkeys; ++j) {
        int32_t phys = a->page_table[(size_t)b * a->max_pages + kp[j]];
        const uint8_t *k = a->K + (((size_t)phys * a->Hkv + h) * PWO_PAGE + ki[j]) * PWO_D;
        double dot = 0.0;
        for (int d = 0; d < PWO_D; ++d)
            dot += q[d] * (pwo_e4m3_to_double(k[d]) * a->k_scale);
        scores[j] = dot * a->sm_scale;
        if (scores[j] > m)
            m = scores[j];
    }
    double l = 0.0;
    for (int j = 0; j < nkeys; ++j) {
        double w = exp(scores[j] - m);
        l += w;
        int32_t phys = a->page_table[(size_t)b * a->max_pages + kp[j]];
        const uint8_t *v = a->V + (((size_t)phys * a->Hkv + h) * PWO_PAGE + ki[j]) * PWO_D;
        for (int d = 0; d < PWO_D; ++d)
            O[d] += w * (pwo_e4m3_to_double(v[d]) * a->v_scale);
    }
    for (int d = 0; d < PWO_D; ++d)
        O[d] /= l;
}

static void row_keys(const pwo_attn_args *a, int b, int64_t t, int h, const int32_t *pages,
                     int npages, int32_t *kp, int32_t *ki, int *nkeys)
{
    int64_t pos = t - a->cu[b];
    int n = 0;
    for (int i = 0; i < npages; ++i)
        for (int r = 0; r < PWO_PAGE; ++r)
            if ((int64_t)pages[i] * PWO_PAGE + r <= pos) {
                kp[n] = pages[i];
                ki[n] = r;
                ++n;
            }
    *nkeys = n;
}

/* O[n, 128] (binary64) for the listed (token, query head) rows, by the definition above. */
int pwo_attn_rows(const uint16_t *Q, const uint8_t *K, const uint8_t *V, const int32_t *page_table,
                  int max_pages, const int32_t *cu, int B, int Hq, int Hkv, int kmax,
                  const int32_t *sel, double k_scale, double v_scale, double sm_scale,
                  const int64_t *rows_t, const int32_t *rows_hq, int64_t nrows, int nthreads,
                  double *O)
{
    if (Hkv < 1 || Hq % Hkv != 0)
        return PWO_ERR_INVALID_ARG;
    pwo_attn_args a = {Q, K, V, page_table, max_pages, cu, B, Hq, Hkv, kmax, sel,
                       k_scale, v_scale, sm_scale};
    int bad = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1) reduction(| : bad)
    {
        int32_t *pages = (int32_t *)malloc(sizeof(int32_t) * (size_t)kmax);
        int32_t *kp = (int32_t *)malloc(sizeof(int32_t) * (size_t)kmax * PWO_PAGE);
        int32_t *ki = (int32_t *)malloc(sizeof(int32_t) * (size_t)kmax * PWO_PAGE);
        double *sc = (double *)malloc(sizeof(double) * (size_t)kmax * PWO_PAGE);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t t = rows_t[r];
            int hq = rows_hq[r];
            int b = seq_of(cu, B, t);
            if (b < 0 || hq < 0 || hq >= Hq) {
                bad = 1;
                continue;
            }
            int h = hq / (Hq / Hkv);
            int np = selected_set(sel, Hkv, kmax, t, h, pages);
            int nk;
            row_keys(&a, b, t, h, pages, np, kp, ki, &nk);
            attend(&a, b, t, hq, kp, ki, nk, sc, O + (size_t)r * PWO_D);
        }
        free(pages);
        free(kp);
        free(ki);
        free(sc);
    }
    return bad ? PWO_ERR_INVALID_ARG : PWO_OK;
}

/* The same attention reached through the groups: for every group, every member t and every
 * query head of the group's kv head, walk the group's union pages in ascending order and keep
 * page p only if p is in the member's own set S(t,h) (membership mask), then apply the causal
 * limit.  Writes O[t, hq, :] for every member row.  Because each member keeps exactly its own
 * pages, in ascending order, the result must equal pwo_attn_rows bit for bit: grouping never
 * changes a query's output (Abstract: original support and complete output ownership). */
int pwo_attn_grouped(const uint16_t *Q, const uint8_t *K, const uint8_t *V,
                     const int32_t *page_table, int max_pages, const int32_t *cu, int B, int Hq,
                     int Hkv, int kmax, const int32_t *sel, double k_scale, double v_scale,
                     double sm_scale, const int32_t *qids, const int32_t *gsize,
                     const int32_t *gmeta, const int32_t *union_off, const int32_t *union_pages,
                     int64_t n_groups, int g, int nthreads, double *O /* [T, Hq, 128] */)
{
    if (Hkv < 1 || Hq % Hkv != 0)
        return PWO_ERR_INVALID_ARG;
    pwo_attn_args a = {Q, K, V, page_table, max_pages, cu, B, Hq, Hkv, kmax, sel,
                       k_scale, v_scale, sm_scale};
    int G = Hq / Hkv;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        int32_t *own = (int32_t *)malloc(sizeof(int32_t) * (size_t)kmax);
        int64_t maxu = 0;
        for (int64_t i = 0; i < n_groups; ++i)
            if (union_off[i + 1] - union_off[i] > maxu)
                maxu = union_off[i + 1] - union_off[i];
        int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxu > 0 ? maxu : 1));
        int32_t *kp = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxu > 0 ? maxu : 1) * PWO_PAGE);
        int32_t *ki = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxu > 0 ? maxu : 1) * PWO_PAGE);
        double *sc = (double *)malloc(sizeof(double) * (size_t)(maxu > 0 ? maxu : 1) * PWO_PAGE);
#pragma omp for schedule(dynamic, 4)
        for (int64_t gi = 0; gi < n_groups; ++gi) {
            int b = gmeta[3 * gi + 0];
            int h = gmeta[3 * gi + 1];
            for (int mi = 0; mi < gsize[gi]; ++mi) {
                int64_t t = qids[gi * g + mi];
                int n_own = selected_set(sel, Hkv, kmax, t, h, own);
                int nk_pages = 0;
                for (int32_t u = union_off[gi]; u < union_off[gi + 1]; ++u) {
                    int member = 0;
                    for (int i = 0; i < n_own; ++i)
                        if (own[i] == union_pages[u])
                            member = 1;
                    if (member)
                        kept[nk_pages++] = union_pages[u];
                }
                int nk;
                row_keys(&a, b, t, h, kept, nk_pages, kp, ki, &nk);
                for (int j = 0; j < G; ++j) {
                    int hq = h * G + j;
                    attend(&a, b, t, hq, kp, ki, nk, sc, O + ((size_t)t * Hq + hq) * PWO_D);
                }
            }
        }
        free(own);
        free(kept);
        free(kp);
        free(ki);
        free(sc);
    }
    return PWO_OK;
}

/* Elementwise pwo_double_to_bf16 over an array (same rounding, one call). */
void pwo_double_to_bf16_n(const double *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = pwo_double_to_bf16(x[i]);
}
