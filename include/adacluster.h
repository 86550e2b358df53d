/*
 * adacluster.h -- C ABI of libadacluster.so, a CUDA (sm_100a) implementation of
 * the AdaCluster clustered sparse attention hot path.
 *
 * Method: "AdaCluster: Adaptive Query-Key Clustering for Sparse Attention in
 * Video Generation" (Tan et al., arXiv 2604.18348), Algorithm 3 (§3.3):
 *   A_q, C_q    <- KMeans(Normalize(Q))                         (§3.1)
 *   A_k, C_k, F <- MultiStageClustering(K, tau, N_max)          (§3.2.2, Algorithm 1)
 *   F ? dense attention : attention over the selected key clusters only.
 * Cluster selection uses centroid-centroid scores weighted by key-cluster size
 * with a top-p cut (the centroid-based significance estimate of §2.3).
 *
 * Conventions shared by every call
 *  - Every function returns ac_status.  Argument errors are detected on the host
 *    and returned synchronously; nothing is launched in that case.
 *  - Work is enqueued asynchronously on the given CUDA stream (cudaStream_t
 *    passed as void*; NULL = legacy default stream).  Device-side errors (a
 *    bounded wait that timed out, a non-finite input, a capacity overflow) set a
 *    status word inside the context; ac_get_status() synchronises the stream and
 *    returns and clears it.
 *  - All tensor pointers are caller-owned DEVICE memory.  The library allocates
 *    device memory only in ac_create (a small status block); every other buffer,
 *    including the scratch workspace `ws`, is passed in.  Pointers must be
 *    16-byte aligned; tensors are dense row-major.
 *  - Layouts (H = heads, N = tokens, d = head dim in {64, 128}):
 *      q, k, v, out   [H, N, d]   element type = config dtype (fp32 or bf16)
 *      assign         [H, N]      int32 cluster id of each token
 *      cent           [H, cap, d] fp32 centroids
 *      count          [H, cap]    int32 members per cluster
 *      mean_norm      [H, kq_cap] fp32 mean ||q|| over a query cluster's members
 *      nclusters      [H]         int32 clusters in use (== kq/kk unless adaptive)
 *      dense_flag     [H]         uint8 1 = head takes dense attention (flag F)
 *      sel_idx        [H, kq_cap, kk_cap] int32 selected key-cluster ids, ascending
 *      sel_cnt        [H, kq_cap] int32 number of selected key clusters
 *    with cap = kq_cap for queries and kk_cap for keys (ac_capacities()).
 *  - Cluster ids are int32; ties in every argmin/argmax go to the lowest id.
 *  - Per-head counts that a call reads from device memory (nq, nk, ncl,
 *    sel_cnt) must lie in [0, capacity] (kq_cap, kk_cap, cap).  A value
 *    outside is clamped to that range so that no kernel indexes past a
 *    capacity-sized buffer, and AC_ERR_INVALID_ARG is recorded in the status
 *    word (ac_get_status).  Cluster ids outside [0, count) are skipped.
 *  - Concurrent calls on one context must not overlap on the GPU: the context's
 *    status word and the workspace are shared by the calls that use them.
 */
#ifndef ADACLUSTER_H
#define ADACLUSTER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AC_API __attribute__((visibility("default")))
#else
#define AC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AC_OK = 0,
    AC_ERR_INVALID_ARG = 1,  /* bad pointer, shape, or parameter              */
    AC_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not 64/128) */
    AC_ERR_CUDA = 3,         /* a CUDA runtime call failed                    */
    AC_ERR_WORKSPACE = 4,    /* workspace pointer NULL or too small           */
    AC_ERR_TIMEOUT = 5,      /* a bounded device wait expired                 */
    AC_ERR_NONFINITE = 6,    /* NaN or Inf in an input                        */
    AC_ERR_CAPACITY = 7      /* adaptive clustering outgrew its capacity      */
} ac_status;

typedef enum { AC_F32 = 0, AC_BF16 = 1 } ac_dtype;

/* How tau of Algorithm 1 is obtained.  ABS: tau = tau_value.  MEAN_X: tau =
 * tau_value x the mean token-to-centre distance of the first stage (§4.1 uses
 * 1.5).  MEDIAN_RADIUS_X: tau = tau_value x the lower median, over non-empty
 * first-stage clusters, of the mean member-to-centre distance.              */
typedef enum { AC_TAU_ABS = 0, AC_TAU_MEAN_X = 1, AC_TAU_MEDIAN_RADIUS_X = 2 } ac_tau_rule;

/* How key clusters are scored for selection (ac_select, ac_forward).
 * CENTROID: s_ab = mean_norm_a * (mu_a . c_b) / sqrt(d), the centroid-centroid
 *   estimate of §2.3 (the default).
 * QUEST: the page bound of §3.2.3 eq. (1) for the representative query
 *   qbar = mean_norm_a * mu_a against key cluster b,
 *   s_ab = sum_t max(qbar_t M_bt, qbar_t m_bt) / sqrt(d),
 *   with M_b / m_b the per-dimension max / min of the keys of b (ac_key_bounds);
 *   evaluated as TensorQuest's eq. (2), qbar+ . M_b + qbar- . m_b with
 *   qbar+ = max(qbar, 0) and qbar- = min(qbar, 0), which gives the same value. */
typedef enum { AC_SCORE_CENTROID = 0, AC_SCORE_QUEST = 1 } ac_score_mode;

/* ac_config.flags */
#define AC_FLAG_WARM_START 1u    /* ac_forward: seed k-means from q_cent_io/k_cent_io */
#define AC_FLAG_CHECK_FINITE 2u  /* scan inputs for NaN/Inf (AC_ERR_NONFINITE)        */
#define AC_FLAG_PROFILE 4u       /* ac_forward records per-stage CUDA events (no sync);
                                    read them with ac_profile_read                     */
#define AC_FLAG_NO_GRAPH 8u      /* ac_forward: never replay its cached CUDA graphs    */

typedef struct {
    int heads, n, d;        /* H, N, d (d in {64, 128}); batch is folded into heads   */
    ac_dtype dtype;         /* element type of q, k, v and out                         */
    int kq, kk;             /* cluster counts, or the first-stage count m0 if adaptive */
    int iters;              /* k-means iterations (assign + update) per stage          */
    int adaptive_q;         /* 1 = Algorithm 1 on normalised queries                   */
    int adaptive_k;         /* 1 = Algorithm 1 on keys                                 */
    ac_tau_rule tau_rule;
    double tau_value;
    int nmax_q, nmax_k;     /* Algorithm 1's N_max for queries / keys                  */
    double top_p;           /* (0, 1]; >= 1 keeps every non-empty key cluster          */
    unsigned flags;
    ac_score_mode score_mode;  /* selection score (zero-initialised: CENTROID)          */
    int top_k;              /* > 0: keep the top_k best-scored key clusters (Algorithm 3's
                               argtopk) instead of the top-p prefix                   */
    int text_keys;          /* > 0: the last text_keys keys of every head (the text
                               tokens) take no part in key clustering and form one
                               more key group, id = the head's key cluster count,
                               that no score ranks and every query cluster selects
                               (a dense strip).  Not from the pages, which give text
                               tokens no special treatment; 0 = off.  < n.         */
    int per_query;          /* 1: selection per query row, as Algorithm 3 writes it
                               (S has one row per query token; argtopk along each
                               row): each query attends to the keys of its own
                               top_k key clusters.  Requires top_k > 0 and bf16
                               (else AC_ERR_UNSUPPORTED); 0 = per query cluster.   */
} ac_config;

/* Per-call statistics filled by ac_forward when `stats` is non-NULL (the call
 * then synchronises the stream before returning). */
typedef struct {
    double ms_cluster_q, ms_cluster_k, ms_select, ms_sort, ms_attn, ms_total;
    int64_t pairs;          /* (query, key) pairs the attention computed, all heads   */
    int dense_heads;        /* heads that took dense attention                        */
    int max_stages_q, max_stages_k;
    /* Rounds (assignment + update) the fixed-count k-means ran, max over heads;
     * 0 for adaptive clustering.  A head stops before ac_config.iters rounds once
     * an assignment pass reproduces the previous one (the result is the same as
     * running all rounds: the update would give back the same centres).       */
    int kmeans_rounds_q, kmeans_rounds_k;
    /* Pairs the attention kernel computed.  Equal to `pairs` with per-cluster
     * selection; with per_query, `pairs` counts each row's own set and this the
     * union per query cluster (rows mask the rest).                          */
    int64_t pairs_computed;
} ac_stats;

/* Averages over the ac_forward calls recorded with AC_FLAG_PROFILE since the
 * last ac_profile_read (at most the last 256 calls). */
typedef struct {
    int calls;
    double ms_cluster_q, ms_cluster_k, ms_select;
    double ms_prep;          /* cluster sort, gather and work list of the attention */
    double ms_attn_kernel;   /* the block-sparse attention kernel alone             */
    double ms_total;
    long long launches;      /* kernels this library launched since the last read   */
} ac_profile;

typedef struct ac_ctx ac_ctx;

/* Create a context for one problem shape.  Validates the configuration and
 * allocates the context's small device status block.  *out = NULL on error.  */
AC_API ac_status ac_create(const ac_config *cfg, ac_ctx **out);
AC_API void ac_destroy(ac_ctx *ctx);

/* Capacities of the cluster dimension: kq/kk, or N_max + m0 in adaptive mode
 * (Algorithm 1 tests |C| >= N_max before a stage, so the last stage may add up
 * to m0 clusters beyond N_max). */
AC_API ac_status ac_capacities(const ac_ctx *ctx, int *kq_cap, int *kk_cap);

/* Bytes of scratch workspace that every call below needs (one size for all). */
AC_API ac_status ac_workspace_size(const ac_ctx *ctx, size_t *bytes);

/* Query clustering (§3.1, Algorithm 3): q_hat = q/||q|| (zero stays
 * zero), then spherical k-means: assign each q_hat to the centroid of largest
 * q_hat.mu (equivalently the closest unit centroid), update mu_j = s_j/||s_j||
 * with s_j the member sum (empty clusters keep their centroid); `iters`
 * rounds, then a final assignment.  With adaptive_q, Algorithm 1 runs on q_hat
 * with the chordal distance.  Initial centroids: init_cent [H, kq, d] if non-NULL,
 * else q_hat of tokens floor(j*N/kq).  Outputs assign, cent, count, mean_norm,
 * nclusters, dense_flag (none of them may be NULL).                       */
AC_API ac_status ac_cluster_q(ac_ctx *ctx, const void *q, const float *init_cent, int32_t *assign,
                       float *cent, int32_t *count, float *mean_norm, int32_t *nclusters,
                       uint8_t *dense_flag, void *ws, size_t ws_bytes, void *stream);

/* Key clustering (§3.2.1; Algorithm 1 of §3.2.2 when adaptive_k): Euclidean
 * k-means, assign by smallest ||k - c||^2, update c_j = member mean.  Same
 * initialisation, iteration and output rules as ac_cluster_q.              */
AC_API ac_status ac_cluster_k(ac_ctx *ctx, const void *k, const float *init_cent, int32_t *assign,
                       float *cent, int32_t *count, int32_t *nclusters, uint8_t *dense_flag,
                       void *ws, size_t ws_bytes, void *stream);

/* Critical-cluster selection.  For each non-empty query cluster a of a head
 * whose dense_flag is 0, every non-empty key cluster b gets the score s_ab of
 * config.score_mode (see ac_score_mode).  Then
 *   top_k > 0: the top_k key clusters of largest s_ab are kept (ties: lower b);
 *   else: p_ab = count_b exp(s_ab - max_b s_ab) / sum_b (...), and key clusters
 *     are taken in decreasing p (ties: lower b) until the taken mass reaches top_p.
 * sel_idx lists the kept clusters in ascending id.  Empty query clusters and
 * dense heads get sel_cnt = 0.  nq/nk/dense_flag may be NULL (then kq/kk and 0
 * are used).  k_max/k_min [H, kk_cap, d] (from ac_key_bounds) are read only,
 * and required only, with AC_SCORE_QUEST.                                    */
AC_API ac_status ac_select(ac_ctx *ctx, const float *q_cent, const float *q_mean_norm,
                    const int32_t *q_count, const float *k_cent, const int32_t *k_count,
                    const float *k_max, const float *k_min,
                    const int32_t *nq, const int32_t *nk, const uint8_t *dense_flag,
                    int32_t *sel_idx, int32_t *sel_cnt, void *ws, size_t ws_bytes, void *stream);

/* Per-query selection (config.per_query = 1; §3.3, Algorithm 3: the score
 * matrix S has one row per query token and Index <- argtopk(S, topk) runs along
 * each row).  For every query row i of every head whose dense_flag is 0 (NULL:
 * none is), each non-empty key cluster b gets
 *   CENTROID: s_ib = (q_i . c_b) / sqrt(d)
 *   QUEST:    s_ib = sum_t max(q_it M_bt, q_it m_bt) / sqrt(d)   (k_max, k_min)
 * (the query is its own representative), and the top_k of largest s_ib (ties:
 * lower b) are kept; with text_keys, the text group (id = the head's key cluster
 * count) is always kept.  row_bits [H, N, W] (W = ceil(kk_cap / 32) words,
 * bit b of word b / 32) receives each row's set; rows of dense heads get none.
 * k_cent [H, kk_cap, d] (CENTROID), k_count [H, kk_cap], nk [H] (NULL: kk).
 * Scores are double, in the order of a plain loop over the d elements, so the
 * sets are exact.  AC_ERR_UNSUPPORTED unless config.per_query.              */
AC_API ac_status ac_select_rows(ac_ctx *ctx, const void *q, const float *k_cent, const int32_t *k_count,
                                const float *k_max, const float *k_min, const int32_t *nk,
                                const uint8_t *dense_flag, uint32_t *row_bits, void *ws, size_t ws_bytes,
                                void *stream);

/* Sparse attention with per-query selection: query row i attends to the keys
 * of the clusters in its own set row_bits[h, i] (from ac_select_rows):
 *   out_i = sum_{j: assign_k(j) in S_i} softmax_j(q_i.k_j / sqrt(d)) v_j.
 * The kernel runs, per query cluster, over the union of its rows' sets and
 * masks each row to its own clusters.  Everything else as ac_sparse_attn.
 * AC_ERR_UNSUPPORTED unless config.per_query.                              */
AC_API ac_status ac_sparse_attn_rows(ac_ctx *ctx, const void *q, const void *k, const void *v,
                                     const int32_t *q_assign, const int32_t *k_assign, const uint32_t *row_bits,
                                     const int32_t *nq, const int32_t *nk, const uint8_t *dense_flag, void *out,
                                     float *lse, void *ws, size_t ws_bytes, void *stream);

/* Quest page bounds of the key clusters (§3.2.3 eq. (1)): k_max / k_min
 * [H, kk_cap, d] receive, per cluster and dimension, the largest / smallest
 * key value over the cluster's members (0 for clusters without members).
 * k [H, N, d] in the configured dtype, k_assign [H, N]; nk may be NULL (then kk).
 * The values are exact (a max / min of the inputs, widened to fp32).         */
AC_API ac_status ac_key_bounds(ac_ctx *ctx, const void *k, const int32_t *k_assign, const int32_t *nk,
                               float *k_max, float *k_min, void *ws, size_t ws_bytes, void *stream);

/* Stable counting sort of token ids by cluster id (per head): perm [H, N]
 * lists tokens of cluster 0 in increasing token order, then cluster 1, ...;
 * offsets [H, cap + 1] holds each cluster's first position and offsets[cap]
 * = N (clusters >= nclusters are empty).  ncl may be NULL (then cap).       */
AC_API ac_status ac_cluster_sort(ac_ctx *ctx, const int32_t *assign, int cap, const int32_t *ncl,
                          int32_t *perm, int32_t *offsets, void *ws, size_t ws_bytes, void *stream);

/* Allocation-free cluster sort.  The paper has no counterpart: this is a
 * convenience for callers that cannot allocate device memory where they need
 * the sort.  Examples are an engine plugin limited to memory reserved before
 * execution, or a host loop whose memory budget is fixed at start-up.
 * Same result as ac_cluster_sort (assign [heads, n], ncl [heads] or NULL,
 * perm [heads, n], offsets [heads, cap + 1]), but no context, no workspace,
 * and no cudaMalloc/cudaFree or other allocating call.
 *  - Scratch is a 16 MiB array in the library's own device memory; every GPU
 *    that loads the library holds it until the process exits.  A problem
 *    needs 256 + 16*heads + 4*heads*n + 4*heads*cap + 4*heads*ceil(n/1024)*cap
 *    bytes (each term rounded up to 256); larger problems, or cap > 8192,
 *    return AC_ERR_UNSUPPORTED without launching anything.
 *  - The first call on each device looks up that device's address of the
 *    array (cudaGetSymbolAddress, with the device current); make that first
 *    call before any stream capture.
 *  - The device address of the array is looked up again whenever the
 *    device's current context changes (after cudaDeviceReset, for example).
 *  - All calls share the one array, which keeps the last call's contents;
 *    calls that overlap on the GPU (different streams without ordering) race,
 *    so order them.
 *  - ncl[h] must lie in [0, cap]; a larger (or negative) count is clamped to
 *    cap (or 0).  There is no context, so this is not reported.
 *  - ids outside [0, ncl[h]) are skipped: the sort covers only the valid ids
 *    (offsets[cap] = their number) and the perm slots past them are left
 *    unwritten.
 *  - A pending launch error of earlier work on the calling thread is cleared
 *    on entry (cudaGetLastError), so the return value describes this call.
 * Returns AC_ERR_INVALID_ARG for NULL pointers or non-positive sizes.         */
AC_API ac_status ac_cluster_sort_static(const int32_t *assign, int heads, int n, int cap, const int32_t *ncl,
                                        int32_t *perm, int32_t *offsets, void *stream);

/* Exact softmax attention over the selected key clusters (Algorithm 3's gather
 * and attention; its dense branch for heads with dense_flag = 1):
 *   out_i = sum_{j: assign_k(j) in S(assign_q(i))} softmax_j(q_i.k_j / sqrt(d)) v_j.
 * Tokens are gathered into cluster order internally; rows are written back in
 * token order.  A query whose selected set is empty gets zeros.  lse [H, N]
 * (natural-log log-sum-exp of the scaled scores) is written when non-NULL.
 * nq/nk/dense_flag may be NULL.  Computes in bf16 (fp32 accumulation) for bf16
 * inputs and in tf32 (fp32 accumulation) for fp32 inputs.                   */
AC_API ac_status ac_sparse_attn(ac_ctx *ctx, const void *q, const void *k, const void *v,
                         const int32_t *q_assign, const int32_t *k_assign, const int32_t *sel_idx,
                         const int32_t *sel_cnt, const int32_t *nq, const int32_t *nk,
                         const uint8_t *dense_flag, void *out, float *lse, void *ws,
                         size_t ws_bytes, void *stream);

/* The whole of Algorithm 3 for every head: ac_cluster_q, ac_cluster_k,
 * (ac_key_bounds with AC_SCORE_QUEST), ac_select, ac_sparse_attn (with
 * per_query: ac_select_rows, ac_sparse_attn_rows).  q_cent_io / k_cent_io ([H, cap, d], nullable):
 * with AC_FLAG_WARM_START they seed k-means (§3.2.2 "Efficient
 * initialization"); when non-NULL they receive the final centroids.
 * Adaptive clustering reads one int per head back to the host per stage; the
 * fixed-count path never synchronises unless `stats` is non-NULL.
 * Graph replay: a fixed-count call without stats, AC_FLAG_PROFILE or
 * AC_FLAG_NO_GRAPH, on a stream that is not being captured, whose q, k, v,
 * q_cent_io, k_cent_io, out and workspace repeat those of an earlier call, is
 * captured into a CUDA graph (the call's ~250 launches) on that second call
 * and replayed on every later one; the replay reads the buffers' current
 * contents.  Four buffer sets are remembered per context (ac_destroy releases
 * their graphs).  If capture fails the call runs launch by launch and the
 * context stops capturing.                                                */
AC_API ac_status ac_forward(ac_ctx *ctx, const void *q, const void *k, const void *v, float *q_cent_io,
                     float *k_cent_io, void *out, ac_stats *stats, void *ws, size_t ws_bytes,
                     void *stream);

/* Multi-step driver over denoising steps (AdaCluster, §3.2.2 "Efficient
 * initialization" and §4.1): the token distribution drifts little from one
 * step to the next, so the clustering of step 0 sets each head's cluster
 * counts (Algorithm 1 when the config is adaptive, else kq / kk) and its
 * dense flag F, and every later step keeps those counts and flags and seeds
 * k-means with the previous step's centres, which then needs fewer rounds
 * (ac_stats.kmeans_rounds_*).
 *   state: caller-owned device buffer of ac_step_state_size bytes, 16-byte
 *          aligned, holding the per-head counts, flags and the q / k centres.
 *          Step 0 writes all of it; step > 0 reads it and updates the centres.
 *          Its contents are opaque; step > 0 requires a state written by an
 *          earlier step of the same context configuration.
 *   step:  0 for the first denoising step, > 0 afterwards.
 * Everything else as ac_forward (no q_cent_io / k_cent_io: the centres live in
 * the state).  Errors: AC_ERR_INVALID_ARG for NULL or misaligned buffers or
 * step < 0; workspace errors as ac_forward. */
AC_API ac_status ac_step_state_size(const ac_ctx *ctx, size_t *bytes);
/* Device pointers to the parts of a step state (for inspection): parts[0] =
 * per-head query cluster counts (int32 [H]), [1] key counts, [2] query dense
 * flags (uint8 [H]), [3] key (combined) dense flags, [4] query centres (fp32
 * [H, kq_cap, d]), [5] key centres (fp32 [H, kk_cap, d]).  No device access. */
AC_API ac_status ac_step_state_parts(const ac_ctx *ctx, void *state, void **parts);
AC_API ac_status ac_forward_step(ac_ctx *ctx, int step, const void *q, const void *k, const void *v,
                                 void *state, void *out, ac_stats *stats, void *ws, size_t ws_bytes,
                                 void *stream);

/* Wait for the recorded events, fill *out (averages per call) and reset the
 * record.  Events are recorded on the stream each ac_forward call used. */
AC_API ac_status ac_profile_read(ac_ctx *ctx, ac_profile *out);

/* Diagnostic of the failure path: one warp waits, through the bounded wait
 * every kernel of this library uses, on a barrier phase that nothing
 * completes.  The wait gives up after `seconds` (0 < seconds <= 10) and
 * records AC_ERR_TIMEOUT, which the next ac_get_status returns; the context
 * stays usable.  No fault, no hang.  AC_ERR_INVALID_ARG for a bad `seconds`. */
AC_API ac_status ac_selftest_wait(ac_ctx *ctx, double seconds, void *stream);

/* Synchronise `stream`, return the first device-side error recorded since the
 * last call (AC_OK if none) and clear it. */
AC_API ac_status ac_get_status(ac_ctx *ctx, void *stream);

AC_API const char *ac_status_string(ac_status s);

#ifdef __cplusplus
}
#endif
#endif /* ADACLUSTER_H */
