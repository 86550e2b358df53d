/*
 * CPU oracle for AdaCluster clustered sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
 * cpu_baseline leg may load this library.  The product path never calls it.
 * It shares no code, header or constant with the CUDA library.
 *
 * Source of every rule below: "AdaCluster: Adaptive Query-Key Clustering for
 * Sparse Attention in Video Generation" (Tan et al., arXiv 2604.18348):
 *   - §3.1 Query Clustering: normalise queries, then k-means on the unit vectors.
 *   - §3.2.1 Observation and Analysis: keys are clustered with Euclidean k-means;
 *     the bound q.c(k) - q.k <= ||q|| ||k - c(k)||.
 *   - §3.2.2 Multi-stage K-means Clustering and Algorithm 1 (MultiStageClustering).
 *   - §3.3 Overall Process and Algorithm 3 (AdaCluster): cluster Q, cluster K,
 *     dense attention when the flag F is set, else select clusters and attend.
 *   - §4.1 Setup: tau = 1.5 x the average token-to-centre distance of the first step.
 * Cluster selection follows the centroid-centroid reading: score each key cluster
 * by its centroid against the query-cluster centroid, weight by cluster size,
 * keep the smallest top-p prefix (§2.3 names centroid-based significance
 * estimation; it stands in for the select step of Algorithm 3).  The
 * alternative score is Quest's per-page upper bound (§3.2.3, eq. (1)) of the
 * representative query against each key cluster's per-dimension max/min, and
 * the alternative cut is Algorithm 3's argtopk.
 *
 * Arithmetic: every input is fp32 (bf16 inputs arrive widened, which is exact)
 * and is widened to double.  All sums and products are double, evaluated in the
 * plain loop order written here (compile with -ffp-contract=off so no fused
 * multiply-add changes a rounding).  Centroids are rounded to fp32 when stored,
 * because they are fp32 buffers at the library boundary.
 *
 * Parity pins (tests/test_oracle_pins.py): brute-force argmin on tiny inputs,
 * k-means objective monotonicity, k = 1 closed forms, Algorithm 1 closed-form
 * traces (tau = 0, tau = inf, N_max), selection invariants and a hand-derived
 * example, select-all attention = dense softmax attention, stable sort; the
 * Quest bound dominates every key of its page and is attained by a one-key page
 * or by the page's corner key, per-page max/min equal numpy's, and argtopk on a
 * hand example.
 * The score/weight reading of the selection rule is "parity unpinned" by the
 * paper itself (it is pinned only by invariants and a hand example).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EUCLID 0    /* keys: ||x - c||^2, centroid = mean              */
#define ORC_SPHERE 1    /* normalised queries: max x.mu, centroid = s/||s|| */

#define ORC_TAU_ABS 0
#define ORC_TAU_MEAN_X 1
#define ORC_TAU_MEDIAN_RADIUS_X 2

/* ------------------------------------------------------------------------ */
/* §3.1: q_hat = q / ||q||; a zero query stays zero.                        */
/* xs receives the working vectors (double) of the chosen mode:             */
/*   EUCLID: xs = x;  SPHERE: xs = x / ||x||.  norm receives ||x||.         */
void orc_prepare(int mode, int64_t n, int d, const float *x, double *xs, double *norm)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        const float *xi = x + i * d;
        double ss = 0.0;
        for (int t = 0; t < d; t++) ss = ss + (double)xi[t] * (double)xi[t];
        double nr = sqrt(ss);
        if (norm) norm[i] = nr;
        for (int t = 0; t < d; t++) {
            if (mode == ORC_SPHERE)
                xs[i * d + t] = (nr > 0.0) ? (double)xi[t] / nr : 0.0;
            else
                xs[i * d + t] = (double)xi[t];
        }
    }
}

/* Distance-like score of row xi against centroid c.
 * EUCLID: squared Euclidean distance sum_t (x_t - c_t)^2 (smaller is closer).
 * SPHERE: dot product sum_t x_t * c_t (larger is closer).                     */
static double orc_score(int mode, int d, const double *xi, const float *c)
{
    double acc = 0.0;
    if (mode == ORC_EUCLID) {
        for (int t = 0; t < d; t++) {
            double df = xi[t] - (double)c[t];
            acc = acc + df * df;
        }
    } else {
        for (int t = 0; t < d; t++) acc = acc + xi[t] * (double)c[t];
    }
    return acc;
}

/* Euclidean distance ||x - c||_2 (chordal distance on the sphere for SPHERE). */
static double orc_dist(int d, const double *xi, const float *c)
{
    double acc = 0.0;
    for (int t = 0; t < d; t++) {
        double df = xi[t] - (double)c[t];
        acc = acc + df * df;
    }
    return sqrt(acc);
}

/* Assignment step of k-means over the rows listed in `rows` (all rows when
 * rows == NULL).  Each row goes to the closest of the k centroids; ties go to
 * the lowest centroid index (strict comparison while scanning upward).
 * assign[r] and dist[r] are written per listed position r (0..nr-1), with
 * ids offset by id_base.  Returns the k-means objective: sum of squared
 * distances (EUCLID) or sum of (1 - x.mu) (SPHERE).                         */
double orc_assign(int mode, int64_t nr, const int32_t *rows, int d, const double *xs,
                  int k, const float *cent, int32_t id_base, int32_t *assign, double *dist)
{
    double obj = 0.0;
#pragma omp parallel for schedule(static) reduction(+ : obj)
    for (int64_t r = 0; r < nr; r++) {
        int64_t i = rows ? rows[r] : r;
        const double *xi = xs + i * d;
        int best = 0;
        double bs = orc_score(mode, d, xi, cent);
        for (int j = 1; j < k; j++) {
            double s = orc_score(mode, d, xi, cent + (int64_t)j * d);
            if (mode == ORC_EUCLID ? (s < bs) : (s > bs)) { bs = s; best = j; }
        }
        assign[r] = id_base + best;
        if (dist) dist[r] = orc_dist(d, xi, cent + (int64_t)best * d);
        obj += (mode == ORC_EUCLID) ? bs : (1.0 - bs);
    }
    return obj;
}

/* Update step.  EUCLID: c_j = mean of members.  SPHERE: mu_j = s_j / ||s_j||
 * with s_j the member sum (the spherical k-means update, which makes the
 * Euclidean and the angular assignment coincide on the unit sphere).
 * An empty cluster, or a zero member sum on the sphere, keeps its centroid.
 * count[j] receives the member count.  assign holds local ids 0..k-1.       */
void orc_update(int mode, int64_t nr, const int32_t *rows, int d, const double *xs,
                const int32_t *assign, int k, float *cent, int32_t *count)
{
    double *sum = (double *)calloc((size_t)k * d, sizeof(double));
    int64_t *cnt = (int64_t *)calloc((size_t)k, sizeof(int64_t));
    for (int64_t r = 0; r < nr; r++) {
        int64_t i = rows ? rows[r] : r;
        int j = assign[r];
        cnt[j] += 1;
        for (int t = 0; t < d; t++) sum[(int64_t)j * d + t] = sum[(int64_t)j * d + t] + xs[i * d + t];
    }
    for (int j = 0; j < k; j++) {
        if (count) count[j] = (int32_t)cnt[j];
        if (cnt[j] == 0) continue;
        double *s = sum + (int64_t)j * d;
        if (mode == ORC_EUCLID) {
            for (int t = 0; t < d; t++) cent[(int64_t)j * d + t] = (float)(s[t] / (double)cnt[j]);
        } else {
            double ss = 0.0;
            for (int t = 0; t < d; t++) ss = ss + s[t] * s[t];
            double nr2 = sqrt(ss);
            if (nr2 == 0.0) continue;
            for (int t = 0; t < d; t++) cent[(int64_t)j * d + t] = (float)(s[t] / nr2);
        }
    }
    free(sum);
    free(cnt);
}

/* Deterministic initial centroids: centroid j is the working vector of the
 * listed row floor(j * nr / k).  The paper leaves initialisation open. */
void orc_init(int64_t nr, const int32_t *rows, int d, const double *xs, int k, float *cent)
{
    for (int j = 0; j < k; j++) {
        int64_t r = ((int64_t)j * nr) / k;
        int64_t i = rows ? rows[r] : r;
        for (int t = 0; t < d; t++) cent[(int64_t)j * d + t] = (float)xs[i * d + t];
    }
}

/* Standard k-means loop (Lloyd): `iters` rounds of assign-then-update, then a
 * final assign so that the returned ids match the returned centroids.
 * cent holds the initial centroids on entry (init or warm start, §3.2.2
 * "Efficient initialization").  count is taken from the final assignment.
 * obj_trace (nullable, 2*iters+1 entries) records the objective after every
 * assign (even slots) and, recomputed, after every update (odd slots).      */
void orc_kmeans(int mode, int64_t nr, const int32_t *rows, int d, const double *xs,
                int k, int iters, float *cent, int32_t *assign, int32_t *count,
                double *dist, double *obj_trace)
{
    for (int it = 0; it < iters; it++) {
        double o = orc_assign(mode, nr, rows, d, xs, k, cent, 0, assign, NULL);
        if (obj_trace) obj_trace[2 * it] = o;
        orc_update(mode, nr, rows, d, xs, assign, k, cent, NULL);
        if (obj_trace) {
            /* objective of the old assignment under the new centroids */
            double o2 = 0.0;
            for (int64_t r = 0; r < nr; r++) {
                int64_t i = rows ? rows[r] : r;
                double s = orc_score(mode, d, xs + i * d, cent + (int64_t)assign[r] * d);
                o2 += (mode == ORC_EUCLID) ? s : (1.0 - s);
            }
            obj_trace[2 * it + 1] = o2;
        }
    }
    double o = orc_assign(mode, nr, rows, d, xs, k, cent, 0, assign, dist);
    if (obj_trace) obj_trace[2 * iters] = o;
    if (count) {
        for (int j = 0; j < k; j++) count[j] = 0;
        for (int64_t r = 0; r < nr; r++) count[assign[r]] += 1;
    }
}

static int orc_cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

/* Algorithm 1 (MultiStageClustering), §3.2.2, with the readings:
 *  - U starts as every token (the initialisation's "D" is read as K).
 *  - Stage t clusters U into m_t clusters: m_0 = m0, and for t >= 1
 *    m_t = min(|U|, ceil(m0 * |U| / N)) (the pages only ask for a moderate count).
 *  - The distance test after each stage runs over the tokens just clustered
 *    (the members of U); d_i = ||x_i - c(x_i)||_2 and x_i leaves U when d_i < tau.
 *  - |C| >= N_max is tested at the top of the loop, so the last stage may
 *    overshoot N_max; F is set only by that test.
 *  - Line 20: every token is assigned to the closest centre of C (global ids in
 *    creation order, ties to the lowest id).  C is not recomputed afterwards.
 *  - tau rules (computed once, from stage 0, "the first inference step" of §4.1):
 *      ABS: tau = tau_value;  MEAN_X: tau = tau_value * mean_i d_i over all tokens;
 *      MEDIAN_RADIUS_X: tau = tau_value * lower median over non-empty stage-0
 *      clusters of (mean member distance to the centre).
 * cap is the capacity of cent (rows); the caller sizes it >= nmax + m0.
 * Outputs: cent[0..nc), assign[N] (global ids), count[0..nc) from the final
 * assignment, dist[N] to the assigned centre, *nclusters, *dense_flag,
 * *nstages, *tau_out.  Returns 0, or -1 if cap would overflow.               */
int orc_multistage(int mode, int64_t n, int d, const double *xs, int m0, int iters,
                   int tau_rule, double tau_value, int nmax, int cap, float *cent,
                   int32_t *assign, int32_t *count, double *dist, int *nclusters,
                   int *dense_flag, int *nstages, double *tau_out)
{
    int32_t *U = (int32_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
    int32_t *loc = (int32_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
    double *dl = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    int64_t nu = n;
    for (int64_t i = 0; i < n; i++) U[i] = (int32_t)i;
    int nc = 0, t = 0, F = 0, rc = 0;
    double tau = (tau_rule == ORC_TAU_ABS) ? tau_value : 0.0;
    while (nu > 0) {
        if (nc >= nmax) { F = 1; break; }
        int mt;
        if (t == 0) mt = m0;
        else {
            int64_t num = (int64_t)m0 * nu;
            int64_t c = (num + n - 1) / n;
            mt = (int)(c < nu ? c : nu);
        }
        if (mt > nu) mt = (int)nu;
        if (nc + mt > cap) { rc = -1; break; }
        float *ct = cent + (int64_t)nc * d;
        orc_init(nu, U, d, xs, mt, ct);
        orc_kmeans(mode, nu, U, d, xs, mt, iters, ct, loc, NULL, dl, NULL);
        if (t == 0 && tau_rule == ORC_TAU_MEAN_X) {
            double s = 0.0;
            for (int64_t r = 0; r < nu; r++) s = s + dl[r];
            tau = tau_value * (s / (double)nu);
        } else if (t == 0 && tau_rule == ORC_TAU_MEDIAN_RADIUS_X) {
            double *rs = (double *)calloc((size_t)mt, sizeof(double));
            int64_t *rc2 = (int64_t *)calloc((size_t)mt, sizeof(int64_t));
            for (int64_t r = 0; r < nu; r++) { rs[loc[r]] = rs[loc[r]] + dl[r]; rc2[loc[r]] += 1; }
            int m = 0;
            for (int j = 0; j < mt; j++)
                if (rc2[j] > 0) rs[m++] = rs[j] / (double)rc2[j];
            qsort(rs, (size_t)m, sizeof(double), orc_cmp_double);
            tau = tau_value * rs[(m - 1) / 2];
            free(rs);
            free(rc2);
        }
        int64_t keep = 0;
        for (int64_t r = 0; r < nu; r++)
            if (!(dl[r] < tau)) U[keep++] = U[r];
        nu = keep;
        nc += mt;
        t += 1;
    }
    if (rc == 0) {
        orc_assign(mode, n, NULL, d, xs, nc, cent, 0, assign, dist);
        for (int j = 0; j < nc; j++) count[j] = 0;
        for (int64_t i = 0; i < n; i++) count[assign[i]] += 1;
    }
    *nclusters = nc;
    *dense_flag = F;
    *nstages = t;
    *tau_out = tau;
    free(U);
    free(loc);
    free(dl);
    return rc;
}

/* Mean ||q_i|| over the members of each query cluster (0 for empty ones). */
void orc_cluster_mean_norm(int64_t n, const double *norm, const int32_t *assign, int k, float *mean_norm)
{
    double *s = (double *)calloc((size_t)k, sizeof(double));
    int64_t *c = (int64_t *)calloc((size_t)k, sizeof(int64_t));
    for (int64_t i = 0; i < n; i++) { s[assign[i]] = s[assign[i]] + norm[i]; c[assign[i]] += 1; }
    for (int j = 0; j < k; j++) mean_norm[j] = c[j] ? (float)(s[j] / (double)c[j]) : 0.0f;
    free(s);
    free(c);
}

/* Quest bounds of the key clusters (§3.2.3, eq. (1)): for cluster b and
 * dimension t, kmax[b*d + t] is the largest k_i[t] over the members i of b and
 * kmin[b*d + t] the smallest.  Clusters without members get 0.              */
void orc_key_bounds(int64_t n, int d, const float *k, const int32_t *assign, int kk, float *kmax, float *kmin)
{
    char *seen = (char *)calloc((size_t)(kk > 0 ? kk : 1), 1);
    for (int64_t j = 0; j < (int64_t)kk * d; j++) { kmax[j] = 0.0f; kmin[j] = 0.0f; }
    for (int64_t i = 0; i < n; i++) {
        const int b = assign[i];
        const float *x = k + i * d;
        float *M = kmax + (int64_t)b * d, *m = kmin + (int64_t)b * d;
        if (!seen[b]) {
            for (int t = 0; t < d; t++) { M[t] = x[t]; m[t] = x[t]; }
            seen[b] = 1;
        } else {
            for (int t = 0; t < d; t++) {
                if (x[t] > M[t]) M[t] = x[t];
                if (x[t] < m[t]) m[t] = x[t];
            }
        }
    }
    free(seen);
}

/* Critical-cluster selection.  For each non-empty query cluster a and each
 * non-empty key cluster b, a score s_ab:
 *   score_mode 0 (centroid): s_ab = (rbar_a * (mu_a . c_b)) * (1/sqrt(d));
 *   score_mode 1 (Quest, §3.2.3 eq. (1)): with the representative query
 *     qbar = rbar_a * mu_a, s_ab = (sum_t max(qbar_t * M_bt, qbar_t * m_bt)) * (1/sqrt(d)),
 *     M_b / m_b the per-dimension maximum / minimum of the keys of b (an upper
 *     bound of qbar . k over every key k of b).
 * Then either
 *   top_k > 0 (Algorithm 3's argtopk): keep the top_k b of largest s_ab
 *     (ties: lower b first), or all of them if fewer are non-empty;
 *   else the top-p rule: w_ab = n_b * exp(s_ab - max_b s_ab), p_ab = w_ab / sum_b w_ab
 *     (sum in b order); visit b by p descending (ties: lower b first),
 *     accumulating p; keep b until the running sum reaches top_p; top_p >= 1
 *     keeps every non-empty b.
 * Empty query clusters select nothing.  The kept set is written in ascending b
 * to sel_idx[a * kk_stride ...], its size to sel_cnt[a].                      */
typedef struct { double p; int b; } orc_pb;
static int orc_cmp_pb(const void *x, const void *y)
{
    const orc_pb *a = (const orc_pb *)x, *b = (const orc_pb *)y;
    if (a->p > b->p) return -1;
    if (a->p < b->p) return 1;
    return (a->b > b->b) - (a->b < b->b);
}

/* s_ab of one (query cluster, key cluster) pair, as defined for orc_select2. */
static double orc_sel_score(int score_mode, int d, double scale, const float *mu, double rbar, const float *c,
                        const float *M, const float *mn)
{
    if (score_mode == 1) {
        double acc = 0.0;
        for (int t = 0; t < d; t++) {
            const double qb = rbar * (double)mu[t];
            const double hi = qb * (double)M[t], lo = qb * (double)mn[t];
            acc = acc + (hi > lo ? hi : lo);
        }
        return acc * scale;
    }
    double dot = 0.0;
    for (int t = 0; t < d; t++) dot = dot + (double)mu[t] * (double)c[t];
    return (rbar * dot) * scale;
}

/* Every s_ab into scores[a * kk + b] (for the pins). */
void orc_scores(int score_mode, int d, int kq, const float *q_cent, const float *q_mean_norm, int kk,
                const float *k_cent, const float *k_max, const float *k_min, double *scores)
{
    const double scale = 1.0 / sqrt((double)d);
    for (int a = 0; a < kq; a++)
        for (int b = 0; b < kk; b++)
            scores[(int64_t)a * kk + b] =
                orc_sel_score(score_mode, d, scale, q_cent + (int64_t)a * d, (double)q_mean_norm[a],
                          k_cent ? k_cent + (int64_t)b * d : 0, k_max ? k_max + (int64_t)b * d : 0,
                          k_min ? k_min + (int64_t)b * d : 0);
}

void orc_select2(int d, int kq, const float *q_cent, const float *q_mean_norm, const int32_t *q_count,
                 int kk, const float *k_cent, const int32_t *k_count, const float *k_max, const float *k_min,
                 int score_mode, int top_k, double top_p, int kk_stride, int32_t *sel_idx, int32_t *sel_cnt)
{
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic)
    for (int a = 0; a < kq; a++) {
        int32_t *out = sel_idx + (int64_t)a * kk_stride;
        sel_cnt[a] = 0;
        if (q_count[a] == 0) continue;
        double *s = (double *)malloc(sizeof(double) * (size_t)(kk > 0 ? kk : 1));
        orc_pb *pb = (orc_pb *)malloc(sizeof(orc_pb) * (size_t)(kk > 0 ? kk : 1));
        char *keep = (char *)calloc((size_t)(kk > 0 ? kk : 1), 1);
        const float *mu = q_cent + (int64_t)a * d;
        const double rbar = (double)q_mean_norm[a];
        double m = -INFINITY;
        for (int b = 0; b < kk; b++) {
            if (k_count[b] == 0) continue;
            s[b] = orc_sel_score(score_mode, d, scale, mu, rbar, k_cent + (int64_t)b * d,
                             score_mode == 1 ? k_max + (int64_t)b * d : 0, score_mode == 1 ? k_min + (int64_t)b * d : 0);
            if (s[b] > m) m = s[b];
        }
        int np = 0;
        if (top_k > 0) {
            for (int b = 0; b < kk; b++) {
                if (k_count[b] == 0) continue;
                pb[np].p = s[b];
                pb[np].b = b;
                np++;
            }
            qsort(pb, (size_t)np, sizeof(orc_pb), orc_cmp_pb);
            for (int r = 0; r < np && r < top_k; r++) keep[pb[r].b] = 1;
        } else {
            double W = 0.0;
            for (int b = 0; b < kk; b++) {
                if (k_count[b] == 0) continue;
                double w = (double)k_count[b] * exp(s[b] - m);
                s[b] = w;
                W = W + w;
            }
            for (int b = 0; b < kk; b++) {
                if (k_count[b] == 0) continue;
                pb[np].p = s[b] / W;
                pb[np].b = b;
                np++;
            }
            qsort(pb, (size_t)np, sizeof(orc_pb), orc_cmp_pb);
            double cum = 0.0;
            for (int r = 0; r < np; r++) {
                keep[pb[r].b] = 1;
                cum = cum + pb[r].p;
                if (top_p < 1.0 && cum >= top_p) break;
            }
        }
        int c = 0;
        for (int b = 0; b < kk; b++)
            if (keep[b]) out[c++] = b;
        sel_cnt[a] = c;
        free(s);
        free(pb);
        free(keep);
    }
}

/* The centroid score with the top-p rule (score_mode 0, top_k 0). */
void orc_select(int d, int kq, const float *q_cent, const float *q_mean_norm, const int32_t *q_count,
                int kk, const float *k_cent, const int32_t *k_count, double top_p,
                int kk_stride, int32_t *sel_idx, int32_t *sel_cnt)
{
    orc_select2(d, kq, q_cent, q_mean_norm, q_count, kk, k_cent, k_count, 0, 0, 0, 0, top_p, kk_stride, sel_idx,
                sel_cnt);
}

/* Stable counting sort of token ids by cluster id: perm lists the tokens of
 * cluster 0 in increasing token order, then cluster 1, ...; offsets[j] is the
 * first position of cluster j, offsets[k] = n.                              */
void orc_cluster_sort(int64_t n, const int32_t *assign, int k, int32_t *perm, int32_t *offsets)
{
    for (int j = 0; j <= k; j++) offsets[j] = 0;
    for (int64_t i = 0; i < n; i++) offsets[assign[i] + 1] += 1;
    for (int j = 0; j < k; j++) offsets[j + 1] += offsets[j];
    int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    for (int j = 0; j < k; j++) pos[j] = offsets[j];
    for (int64_t i = 0; i < n; i++) perm[pos[assign[i]]++] = (int32_t)i;
    free(pos);
}

/* Exact softmax attention for the listed query rows (Algorithm 3's sparse
 * attention, or its dense branch when dense != 0): row i attends to every key j whose cluster is in
 * the selected set of i's query cluster,
 *   o_i = sum_j exp(s_ij - m_i) v_j / sum_j exp(s_ij - m_i),  s_ij = q_i.k_j / sqrt(d).
 * A row whose selected set holds no key gets zeros.  out is [nrows, d].      */
void orc_attention_rows(int64_t n, int d, const float *q, const float *k, const float *v,
                        const int32_t *q_assign, const int32_t *k_assign, int kk,
                        const int32_t *sel_idx, const int32_t *sel_cnt, int kk_stride, int dense,
                        int64_t nrows, const int32_t *rows, double *out)
{
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; r++) {
        int64_t i = rows[r];
        char *allow = (char *)calloc((size_t)(kk > 0 ? kk : 1), 1);
        double *sc = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        double *o = out + r * d;
        if (!dense) {
            int a = q_assign[i];
            for (int c = 0; c < sel_cnt[a]; c++) allow[sel_idx[(int64_t)a * kk_stride + c]] = 1;
        }
        double m = -INFINITY;
        for (int64_t j = 0; j < n; j++) {
            if (!dense && !allow[k_assign[j]]) continue;
            double dot = 0.0;
            for (int t = 0; t < d; t++) dot = dot + (double)q[i * d + t] * (double)k[j * d + t];
            sc[j] = dot * scale;
            if (sc[j] > m) m = sc[j];
        }
        for (int t = 0; t < d; t++) o[t] = 0.0;
        double den = 0.0;
        for (int64_t j = 0; j < n; j++) {
            if (!dense && !allow[k_assign[j]]) continue;
            double e = exp(sc[j] - m);
            den = den + e;
            for (int t = 0; t < d; t++) o[t] = o[t] + e * (double)v[j * d + t];
        }
        if (den > 0.0)
            for (int t = 0; t < d; t++) o[t] = o[t] / den;
        free(allow);
        free(sc);
    }
}

/* Number of (query, key) pairs the sparse attention computes for one head:
 * sum over query clusters a of |a| * sum_{b selected by a} n_b. */
int64_t orc_pairs(int kq, const int32_t *q_count, const int32_t *k_count, const int32_t *sel_idx,
                  const int32_t *sel_cnt, int kk_stride)
{
    int64_t tot = 0;
    for (int a = 0; a < kq; a++) {
        int64_t keys = 0;
        for (int c = 0; c < sel_cnt[a]; c++) keys += k_count[sel_idx[(int64_t)a * kk_stride + c]];
        tot += (int64_t)q_count[a] * keys;
    }
    return tot;
}
