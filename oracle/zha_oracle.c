/*
 * zha_oracle.c -- plain, slow, fp64 CPU oracle of the Zyphra Hierarchical
 * Attention (ZHA) decode path: summary-tree build / append, top-p routing,
 * and exact attention over the routed token set.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA library shares no
 * code, header, table or helper with it, and it never calls the CUDA library.
 *
 * What each function follows (page title, then section):
 *   "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)" (MarkTechPost
 *   article, tradepoint.io copy):
 *     - "Building the tree": the cache is cut into contiguous chunks of c
 *       keys and each chunk is summarised; c sibling summaries are summarised
 *       into a parent, one level at a time (c = 4 and 6 levels put 4,096
 *       tokens under a top node). Every learned reference query gives a chunk
 *       a tangent plane of its log attention mass; the largest plane value is
 *       the node's estimate.
 *     - "How does top-p routing pick tokens": a decode query rates the top
 *       level's nodes, retains the fewest whose estimated mass reaches p of
 *       the total, rates only their children next, and so on down to raw
 *       keys; token 0 (the attention sink) is attended in every case.
 *     - explainer widget, step 5 caption: the final attention is exact, over
 *       the routed raw KV plus the sink and the chunk being written.
 *   "ZHA" (kongchang.com notes): a parent summarises its children, and the
 *       tree grows as the cache does.
 *
 * Readings taken where the pages are loose (each is also listed in the
 * design notes of the repository):
 *   R1 tangent plane of reference r over a chunk with keys k_t, s = 1/sqrt(d):
 *      l_t = s r.k_t, F = log sum_t e^{l_t}, w_t = e^{l_t - F},
 *      mu = sum_t w_t k_t, b = F - s r.mu; plane_r(q) = s q.mu + b.
 *      (This is the first-order expansion of F(q) = log sum_t e^{s q.k_t}
 *      at q = r, since grad F(r) = s mu.)
 *   R2 parent rule: a parent applies R1 to its children, child i acting as
 *      one point at its summary key mu_{i,r} (as stored) carrying, as
 *      log-weight, its log-mass at the SAME reference r,
 *      l_i = F_{i,r} = log sum over the keys under child i of e^{s r.k}
 *      (the child's plane evaluated at r, where it is exact: in exact
 *      arithmetic F_{i,r} = s r.mu_{i,r} + b_{i,r}); F = log sum_i e^{l_i},
 *      mu = sum_i e^{l_i - F} mu_{i,r}, b = F - s r.mu. Every node keeps its
 *      F beside its planes. In exact arithmetic this equals R1 over all raw
 *      keys under the parent.
 *   R3 only complete leaf chunks enter the tree: n_1 = floor(N/c); a node at
 *      level l > 1 exists iff at least one of its children exists, and uses
 *      only the existing ones: n_l = ceil(n_{l-1}/c).
 *   R4 estimate E = max_r plane_r(q).
 *   R5 top-p per query head over all candidates of a level at once: masses
 *      e^{E - max E}, order (E desc, node index asc), keep the shortest
 *      prefix whose running mass reaches p * total (>=); p >= 1 keeps all.
 *   R6 token set = {0} U tokens of kept leaf chunks U current chunk, the
 *      current chunk being [c*floor((N-1)/c), N) (the chunk holding the
 *      newest token, complete or not); tail_only selects the alternative
 *      [c*floor(N/c), N).
 *   R7 attention scale s = 1/sqrt(d) unless given.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_STORE_F64 0
#define ORC_STORE_F32 1
#define ORC_STORE_BF16 2
#define ORC_STORE_MXFP8 3

/* Round-to-nearest-even to the storage format the summaries are kept in,
 * so that parents are built from the same stored children a GPU build
 * would read. bf16 keeps 8 significant bits (normal range only). */
static double store_round(double x, int storage)
{
    if (storage == ORC_STORE_F32)
        return (double)(float)x;
    if (storage == ORC_STORE_BF16) {
        if (x == 0.0 || !isfinite(x))
            return x;
        int e;
        double m = frexp(x, &e);            /* |m| in [0.5, 1) */
        double r = nearbyint(ldexp(m, 8));  /* 8 significant bits, ties even */
        return ldexp(r, e - 8);
    }
    return x;
}

double orc_round_storage(double x, int storage) { return store_round(x, storage); }

/*
 * Low-precision summaries (the MarkTechPost article's TL;DR box says an FP4
 * router variant was also tried, and gives no format; the reading taken
 * here, at 8 bits): mu of every plane is kept in
 * blocks of 32 consecutive coordinates, each block as one power-of-two scale
 * 2^e times 32 FP8 E4M3 values, the block layout of the OCP Microscaling (MX)
 * specification v1.0. E4M3 as defined there: 1 sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; normal magnitudes 2^-6 .. 448, subnormals are
 * multiples of 2^-9. Rounding to nearest, ties to even. The block's e is the
 * smallest integer with max|x| <= 448 * 2^e, so that no element saturates
 * (a choice made here; the MX text allows saturation instead).
 */
static double e4m3_round(double x)
{
    if (x == 0.0 || !isfinite(x))
        return x;
    double a = fabs(x), r;
    if (a < ldexp(1.0, -6)) {
        r = ldexp(nearbyint(ldexp(a, 9)), -9);   /* subnormal grid 2^-9 */
    } else {
        int e;
        double m = frexp(a, &e);                 /* a = m 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(m, 4)), e - 4); /* 4 significant bits */
    }
    if (r > 448.0)
        r = 448.0;
    return x < 0 ? -r : r;
}

double orc_e4m3_round(double x) { return e4m3_round(x); }

/* Exponent e of one block's scale 2^e; 0 for an all-zero block. */
static int mx_block_exponent(const double *x, int n)
{
    double amax = 0.0;
    for (int k = 0; k < n; ++k)
        if (fabs(x[k]) > amax)
            amax = fabs(x[k]);
    if (amax == 0.0)
        return 0;
    int k;
    double f = frexp(amax, &k);      /* amax = f 2^k; 448 = 0.875 2^9 */
    int e = (f <= 0.875) ? k - 9 : k - 8;
    if (e < -126) e = -126;
    if (e > 127) e = 127;
    return e;
}

/* Round a plane (d coordinates, d a multiple of 32) to its MX-FP8 value in place;
 * exps (optional, d/32 entries) receives the block exponents. */
void orc_mx_round(double *x, int d, int *exps)
{
    for (int b0 = 0; b0 < d; b0 += 32) {
        int e = mx_block_exponent(x + b0, 32);
        for (int k = b0; k < b0 + 32; ++k)
            x[k] = ldexp(e4m3_round(ldexp(x[k], -e)), e);
        if (exps)
            exps[b0 / 32] = e;
    }
}

/* Store one plane's mu in the summary format. */
static void store_plane(double *m, int d, int storage)
{
    if (storage == ORC_STORE_MXFP8) {
        orc_mx_round(m, d, NULL);
        return;
    }
    for (int k = 0; k < d; ++k)
        m[k] = store_round(m[k], storage);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double dot(const double *a, const double *b, int d)
{
    double acc = 0.0;
    for (int k = 0; k < d; ++k)
        acc += a[k] * b[k];
    return acc;
}

/* Number of nodes at `level` (1 = leaf chunks) for a cache of N tokens (R3). */
int64_t orc_level_nodes(int64_t N, int c, int level)
{
    int64_t n = N / c;
    for (int l = 2; l <= level; ++l)
        n = (n + c - 1) / c;
    return n;
}

/*
 * R1/R2 for ONE reference r over n points x[i] (each d long) carrying
 * log-weights a[i] (a == NULL: all zero, i.e. raw keys).
 */
static void plane_one_ref(int64_t n, int d, const double *const *x, const double *a,
                          const double *r, double s, double *mu, double *b, double *F_out)
{
    double *l = (double *)malloc((size_t)n * sizeof(double));
    double lmax = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        l[i] = s * dot(r, x[i], d) + (a ? a[i] : 0.0);
        if (l[i] > lmax)
            lmax = l[i];
    }
    double sum = 0.0;
    for (int64_t i = 0; i < n; ++i)
        sum += exp(l[i] - lmax);
    double F = lmax + log(sum);
    for (int k = 0; k < d; ++k)
        mu[k] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double w = exp(l[i] - F);
        for (int k = 0; k < d; ++k)
            mu[k] += w * x[i][k];
    }
    *b = F - s * dot(r, mu, d);
    if (F_out)
        *F_out = F;
    free(l);
}

/*
 * R2 for ONE reference r over n children: points x[i] (their summary keys)
 * whose log-weights are their log-masses lw[i] at r.
 */
static void plane_from_children(int64_t n, int d, const double *const *x, const double *lw,
                                const double *r, double s, double *mu, double *b, double *F_out)
{
    double lmax = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (lw[i] > lmax)
            lmax = lw[i];
    double sum = 0.0;
    for (int64_t i = 0; i < n; ++i)
        sum += exp(lw[i] - lmax);
    double F = lmax + log(sum);
    for (int k = 0; k < d; ++k)
        mu[k] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double w = exp(lw[i] - F);
        for (int k = 0; k < d; ++k)
            mu[k] += w * x[i][k];
    }
    *b = F - s * dot(r, mu, d);
    *F_out = F;
}

/*
 * R1 directly over the raw keys K[t0..t1) for every reference (no tree):
 * the plane a node covering exactly those tokens must equal (R2 identity).
 * mu: [R][d], b: [R].
 */
void orc_direct_planes(const double *K, int64_t t0, int64_t t1, int d,
                       const double *refs, int R, double s, double *mu, double *b)
{
    int64_t n = t1 - t0;
    const double **x = (const double **)malloc((size_t)n * sizeof(double *));
    for (int64_t i = 0; i < n; ++i)
        x[i] = K + (t0 + i) * d;
    for (int r = 0; r < R; ++r)
        plane_one_ref(n, d, x, NULL, refs + (int64_t)r * d, s, mu + (int64_t)r * d, b + r, NULL);
    free(x);
}

/*
 * R2 for one parent from given children: cmu [nch][R][d] and their log-masses
 * cF [nch][R] (for instance the children a GPU stored), with the result
 * stored as `storage` would keep it. mu: [R][d], b: [R], F: [R].
 */
void orc_parent_planes(const double *cmu, const double *cF, int64_t nch, int d,
                       const double *refs, int R, double s, int storage, double *mu, double *b, double *F)
{
    const double **x = (const double **)malloc((size_t)nch * sizeof(double *));
    double *a = (double *)malloc((size_t)nch * sizeof(double));
    for (int r = 0; r < R; ++r) {
        for (int64_t i = 0; i < nch; ++i) {
            x[i] = cmu + (i * R + r) * d;
            a[i] = cF[i * R + r];
        }
        plane_from_children(nch, d, x, a, refs + (int64_t)r * d, s, mu + (int64_t)r * d, b + r, F + r);
        store_plane(mu + (int64_t)r * d, d, storage);
        b[r] = store_round(b[r], storage == ORC_STORE_F64 ? ORC_STORE_F64 : ORC_STORE_F32);
        F[r] = store_round(F[r], storage == ORC_STORE_F64 ? ORC_STORE_F64 : ORC_STORE_F32);
    }
    free(a);
    free(x);
}

/*
 * Build or extend the tree of ONE (sequence, KV head) from old_N to new_N
 * tokens. mu[l-1]: [n_l][R][d], b[l-1]: [n_l][R], F[l-1]: [n_l][R] (each
 * plane's log-mass at its reference) for the caller's capacity.
 * Nodes that a longer cache adds or changes are (R3) the new leaf chunks and,
 * at each level above, every node from the parent of the first changed child
 * to the last node; those are recomputed, everything else is left as is.
 * old_N = 0 is a build from scratch.
 */
void orc_tree_update(const double *K, int64_t old_N, int64_t new_N, int d,
                     const double *refs, int R, int c, int L, double s, int storage,
                     double **mu, double **b, double **F)
{
    int64_t lo = old_N / c;              /* first leaf that is new */
    int64_t hi = new_N / c;              /* leaves after the update */
    if (hi <= lo)
        return;                          /* no chunk completed: tree unchanged */
    /* level 1: leaf chunks */
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t j = lo; j < hi; ++j) {
        const double *x[512];
        const double **xp = (c <= 512) ? x : (const double **)malloc((size_t)c * sizeof(double *));
        for (int i = 0; i < c; ++i)
            xp[i] = K + (j * c + i) * d;
        for (int r = 0; r < R; ++r) {
            double *m = mu[0] + (j * R + r) * d;
            double *bb = b[0] + j * R + r;
            double *ff = F[0] + j * R + r;
            plane_one_ref(c, d, xp, NULL, refs + (int64_t)r * d, s, m, bb, ff);
            store_plane(m, d, storage);
            *bb = store_round(*bb, storage == ORC_STORE_F64 ? ORC_STORE_F64 : ORC_STORE_F32);
            *ff = store_round(*ff, storage == ORC_STORE_F64 ? ORC_STORE_F64 : ORC_STORE_F32);
        }
        if (xp != x)
            free(xp);
    }
    /* levels 2..L: parents from their existing children (R2, R3) */
    int64_t nprev = hi;
    for (int l = 2; l <= L; ++l) {
        lo = lo / c;
        int64_t nl = (nprev + c - 1) / c;
        const double *cmu = mu[l - 2];
        const double *cF = F[l - 2];
#pragma omp parallel for schedule(dynamic, 16)
        for (int64_t p = lo; p < nl; ++p) {
            int64_t c0 = p * c;
            int64_t c1 = c0 + c < nprev ? c0 + c : nprev;
            int64_t nch = c1 - c0;
            const double *x[512];
            double a[512];
            const double **xp = (nch <= 512) ? x : (const double **)malloc((size_t)nch * sizeof(double *));
            double *ap = (nch <= 512) ? a : (double *)malloc((size_t)nch * sizeof(double));
            for (int r = 0; r < R; ++r) {
                for (int64_t i = 0; i < nch; ++i) {
                    xp[i] = cmu + ((c0 + i) * R + r) * d;
                    ap[i] = cF[(c0 + i) * R + r];
                }
                double *m = mu[l - 1] + (p * R + r) * d;
                double *bb = b[l - 1] + p * R + r;
                double *ff = F[l - 1] + p * R + r;
                plane_from_children(nch, d, xp, ap, refs + (int64_t)r * d, s, m, bb, ff);
                store_plane(m, d, storage);
                *bb = store_round(*bb, storage == ORC_STORE_F64 ? ORC_STORE_F64 : ORC_STORE_F32);
                *ff = store_round(*ff, storage == ORC_STORE_F64 ? ORC_STORE_F64 : ORC_STORE_F32);
            }
            if (xp != x)
                free(xp);
            if (ap != a)
                free(ap);
        }
        nprev = nl;
    }
}

/* R4: estimate of one node (planes mu [R][d], b [R]) for query q. */
double orc_estimate(const double *q, const double *mu, const double *b, int R, int d, double s)
{
    double best = -INFINITY;
    for (int r = 0; r < R; ++r) {
        double e = s * dot(q, mu + (int64_t)r * d, d) + b[r];
        if (e > best)
            best = e;
    }
    return best;
}

typedef struct {
    double e;
    int64_t idx;   /* position in the candidate list (ascending node index) */
} scored_t;

static int by_score_desc_idx_asc(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->e > b->e) return -1;
    if (a->e < b->e) return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

/*
 * R5 over n candidates whose scores are E[0..n) (candidate i has a smaller
 * node index than candidate i+1). kept[i] = 1 for the selected ones.
 * cum_before[i] (optional) = running mass of the candidates ordered before i,
 * divided by the total: the distance of |cum_before - p| tells how close a
 * candidate sits to the p boundary. Returns the number kept.
 */
int64_t orc_topp_select(int64_t n, const double *E, double p, uint8_t *kept, double *cum_before)
{
    if (n <= 0)
        return 0;
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (E[i] > m)
            m = E[i];
    scored_t *ord = (scored_t *)malloc((size_t)n * sizeof(scored_t));
    double Z = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        ord[i].e = E[i];
        ord[i].idx = i;
        Z += exp(E[i] - m);
        kept[i] = 0;
    }
    qsort(ord, (size_t)n, sizeof(scored_t), by_score_desc_idx_asc);
    double cum = 0.0;
    int done = 0;
    int64_t nk = 0;
    for (int64_t k = 0; k < n; ++k) {
        int64_t i = ord[k].idx;
        if (cum_before)
            cum_before[i] = cum / Z;
        if (!done) {
            kept[i] = 1;
            ++nk;
        }
        cum += exp(E[i] - m);
        if (p < 1.0 && cum >= p * Z)
            done = 1;
    }
    free(ord);
    return nk;
}

/*
 * Top-down routing of G queries (q: [G][d]) through the tree of one
 * (sequence, KV head) with n_1 = n1 leaves. p_level[l-1] is the fraction at
 * level l. Outputs, for every level l and head h, arrays of length n_l at
 * offset off_l = sum_{l'<l} n_{l'} inside per-head blocks of size tot:
 *   cand[h*tot + off_l + n]  = 1 if node n was a candidate of head h,
 *   kept[h*tot + off_l + n]  = 1 if it was selected,
 *   score[h*tot + off_l + n] = its estimate (if a candidate),
 *   cumb[h*tot + off_l + n]  = its cum_before (see orc_topp_select).
 * tot = sum_l n_l.
 */
void orc_route(const double *q, int G, int d, double s, int R, int c, int L, int64_t n1,
               double *const *mu, double *const *b, const double *p_level,
               uint8_t *cand, uint8_t *kept, double *score, double *cumb)
{
    int64_t nl[64];
    int64_t off[64];
    int64_t tot = 0;
    nl[1] = n1;
    for (int l = 2; l <= L; ++l)
        nl[l] = (nl[l - 1] + c - 1) / c;
    for (int l = 1; l <= L; ++l) {
        off[l] = tot;
        tot += nl[l];
    }
    memset(cand, 0, (size_t)(G * tot));
    memset(kept, 0, (size_t)(G * tot));
    if (n1 <= 0)
        return;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < G; ++h) {
        const double *qh = q + (int64_t)h * d;
        uint8_t *ch = cand + h * tot;
        uint8_t *kh = kept + h * tot;
        double *sh = score + h * tot;
        double *cbh = cumb + h * tot;
        /* every top-level node is a candidate */
        for (int64_t n = 0; n < nl[L]; ++n)
            ch[off[L] + n] = 1;
        for (int l = L; l >= 1; --l) {
            int64_t n_here = nl[l];
            int64_t *list = (int64_t *)malloc((size_t)(n_here > 0 ? n_here : 1) * sizeof(int64_t));
            int64_t nc = 0;
            for (int64_t n = 0; n < n_here; ++n)
                if (ch[off[l] + n])
                    list[nc++] = n;
            double *E = (double *)malloc((size_t)(nc > 0 ? nc : 1) * sizeof(double));
            double *cb = (double *)malloc((size_t)(nc > 0 ? nc : 1) * sizeof(double));
            uint8_t *kk = (uint8_t *)malloc((size_t)(nc > 0 ? nc : 1));
            for (int64_t i = 0; i < nc; ++i) {
                int64_t n = list[i];
                E[i] = orc_estimate(qh, mu[l - 1] + n * R * d, b[l - 1] + n * R, R, d, s);
                sh[off[l] + n] = E[i];
            }
            orc_topp_select(nc, E, p_level[l - 1], kk, cb);
            for (int64_t i = 0; i < nc; ++i) {
                int64_t n = list[i];
                cbh[off[l] + n] = cb[i];
                if (!kk[i])
                    continue;
                kh[off[l] + n] = 1;
                if (l > 1) {
                    /* expand: the existing children of a kept node */
                    for (int64_t j = n * c; j < n * c + c && j < nl[l - 1]; ++j)
                        ch[off[l - 1] + j] = 1;
                }
            }
            free(list);
            free(E);
            free(cb);
            free(kk);
        }
    }
}

/* R6: mark the attended tokens of one head. kept_leaf: [n1] 0/1. */
void orc_token_set(int64_t N, int c, int64_t n1, const uint8_t *kept_leaf, int tail_only,
                   uint8_t *tmask)
{
    memset(tmask, 0, (size_t)N);
    if (N <= 0)
        return;
    tmask[0] = 1;
    for (int64_t j = 0; j < n1; ++j)
        if (kept_leaf[j])
            for (int64_t t = j * c; t < j * c + c; ++t)
                tmask[t] = 1;
    int64_t cur = tail_only ? (N / c) * c : ((N - 1) / c) * c;
    for (int64_t t = cur; t < N; ++t)
        tmask[t] = 1;
}

/* Exact softmax attention of q over the marked tokens: out = sum softmax(s q.k_t) v_t. */
void orc_attend(const double *q, const double *K, const double *V, int64_t N, int d, double s,
                const uint8_t *tmask, double *out)
{
    double m = -INFINITY;
    for (int64_t t = 0; t < N; ++t)
        if (!tmask || tmask[t]) {
            double l = s * dot(q, K + t * d, d);
            if (l > m)
                m = l;
        }
    double den = 0.0;
    for (int k = 0; k < d; ++k)
        out[k] = 0.0;
    for (int64_t t = 0; t < N; ++t)
        if (!tmask || tmask[t]) {
            double w = exp(s * dot(q, K + t * d, d) - m);
            den += w;
            for (int k = 0; k < d; ++k)
                out[k] += w * V[t * d + k];
        }
    for (int k = 0; k < d; ++k)
        out[k] /= den;
}
