// Internal launch interface between the C ABI (ac_api.cu) and the kernels.
#pragma once
#include "ac_common.cuh"

namespace ac {

enum { MODE_EUCLID = 0, MODE_SPHERE = 1 };
enum { DT_F32 = 0, DT_BF16 = 1 };
constexpr int SORT_TILE = 1024;  // positions per rank/histogram tile (one CTA of 4 warps)

// Working value of element t of a row: x (EUCLID) or x/||x|| (SPHERE), in
// double (nrm = ||x|| in double; a zero row stays zero).
template <typename T>
__device__ __forceinline__ double work_val(const T *xi, int t, int mode, double nrm) {
    double v = (double)to_f(xi[t]);
    if (mode == MODE_SPHERE) return nrm > 0.0 ? ddiv(v, nrm) : 0.0;
    return v;
}

// Host-side count of kernels this library has launched (profiling).
void note_launch();
long long launches_total();

// ---- ac_kmeans.cu
void k_row_norm(const void *x, int dtype, int H, int N, int D, double *norm, int check, int *status,
                cudaStream_t st);
void k_init_cent(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const double *norm,
                 const HeadSeg *seg, int kmax, int mode, float *cent, int cap, cudaStream_t st);
void k_assign(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const HeadSeg *seg,
              int nrows_max, const float *cent, int cap, float *cn2, float *cmax, const double *norm, int mode,
              int32_t *assign, int32_t *amb_list, int32_t *amb_count, cudaStream_t st);
void k_assign_exact(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const HeadSeg *seg,
                    const float *cent, int cap, const double *norm, int mode, const int32_t *amb_list,
                    const int32_t *amb_count, const int2 *amb_cand, int32_t *assign, cudaStream_t st);
void k_dist(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const HeadSeg *seg,
            int nrows_max, const float *cent, int cap, const double *norm, int mode, const int32_t *assign,
            double *dist, cudaStream_t st);
// order (optional, from k_sort): the clusters are taken largest first
void k_update(const void *x, int dtype, int H, int N, int D, const HeadSeg *seg, int kmax, const int32_t *perm,
              const int32_t *off, int cap, const double *norm, int mode, float *cent, cudaStream_t st,
              const int32_t *order = nullptr);
void k_mean_norm(int H, int N, const HeadSeg *seg, const int32_t *perm, const int32_t *off, int cap,
                 const double *norm, float *mean_norm, cudaStream_t st);
// Early stop of fixed-count k-means (ac_kmeans.cu): kst [H, 4] = {stopped,
// rows changed in the pass, rounds run, -}; a stopped head's seg gets 0 rows.
void k_conv_check(int H, int N, const HeadSeg *seg, const int32_t *assign, int32_t *prev, int32_t *kst, int first,
                  cudaStream_t st);
void k_conv_decide(int H, HeadSeg *seg, int32_t *kst, int it, cudaStream_t st);

// ---- ac_assign_tc.cu (bf16 inputs): tcgen05 screen; the exact pass follows
// cnp [H, kpad] (nullable: the per-tile kernel): the per-column score shift
// of the persistent kernel, which runs one CTA per SM (num_sms).
int k_assign_tc(const void *xc, int H, int N, int D, const int32_t *rows, const HeadSeg *seg, int nrows_max,
                const float *cent, int cap, int kpad, void *chi, void *clo, float *cn2, float *cmax,
                const double *norm, int mode, int32_t *assign, int32_t *amb_list, int32_t *amb_count, int2 *amb_cand,
                int *status, void *encode_fn, float *cnp, int num_sms, cudaStream_t st);

// ---- ac_sort.cu
// Stable counting sort of positions 0..seg.nrows-1 by id (< seg.k): perm gets
// rows[pos] (or pos), off [H, cap+1] the cluster offsets, cnt [H, cap] the sizes;
// order [H, cap] (optional) the non-empty clusters by size class, largest first, then -1.
void k_sort(const int32_t *ids, const int32_t *rows, const HeadSeg *seg, int H, int N, int nrows_max, int cap,
            int32_t *rank, int32_t *hist, int32_t *cnt, int32_t *off, int32_t *perm, int *status, cudaStream_t st,
            int32_t *order = nullptr);
size_t sort_hist_elems(int H, int N, int cap);
void k_gather_rows(const void *src, void *dst, const int32_t *perm, int H, int N, int row_bytes, cudaStream_t st);

// ---- ac_multistage.cu
struct MsState;  // device-side Algorithm 1 state, see ac_multistage.cu

// ---- ac_select.cu
void k_select(int H, int D, const float *q_cent, const float *q_mean_norm, const int32_t *q_count, int kq_cap,
              const float *k_cent, const int32_t *k_count, const float *k_max, const float *k_min, int kk_cap,
              const int32_t *nq, const int32_t *nk, int kq_fixed, int kk_fixed, const uint8_t *dense, int score_mode,
              int top_k, double top_p, int32_t *sel_idx, int32_t *sel_cnt, int *status, cudaStream_t st,
              int text_group = 0,
              float *k_cent_t = nullptr,   // [H, D, kk_cap] scratch: transposed centroids (or Quest maxima)
              float *k_min_t = nullptr);   // [H, D, kk_cap] scratch: transposed Quest minima
// Per-cluster, per-dimension max / min of x over the members listed by a
// cluster sort (perm, off [H, cap + 1]); 0 for empty clusters.
void k_cluster_bounds(const void *x, int dtype, int H, int N, int D, const int32_t *perm, const int32_t *off,
                      int cap, float *xmax, float *xmin, cudaStream_t st);

// ---- ac_attn.cu
struct AttnItem {
    int h, a, q_start, q_len;  // a < 0: dense head (all keys)
};
// n_items[0] = item count; n_items[1] = 0 (the bf16 attention kernel's work counter)
void k_build_items(int H, int N, int rows_per_item, int kq_cap, int kk_cap, const int32_t *qoff, const int32_t *nq,
                   const uint8_t *dense, int kq_fixed, const int32_t *koff, const int32_t *sel_idx,
                   const int32_t *sel_cnt, AttnItem *items, int32_t *n_items, int64_t *pairs, int32_t *scratch,
                   int *status, cudaStream_t st);
size_t items_scratch_elems(int H, int kq_cap);
int attn_max_items(int H, int N, int kq_cap);
// Key runs of every (head, query cluster) (ac_attn.cu): the selected key
// clusters in ascending order, neighbours merged into one range of rows of the
// gathered K/V (empty clusters between them are absorbed).  runs [H, kq_cap,
// kk_cap]; info [H, kq_cap] = {runs, chunks of `chunk_rows` rows as KeyStream
// packs them}.  Cluster ids outside [0, kk_cap) are skipped.
void k_key_runs(int H, int kq_cap, int kk_cap, const int32_t *koff, const int32_t *sel_idx, const int32_t *sel_cnt,
                int chunk_rows, int2 *runs, int2 *info, cudaStream_t st);
// Valid-row counts of every chunk of ATTN3_CHUNK (128) keys (4 bits per 8-row
// group, two 32-bit words per chunk) of every (head, query cluster) key
// stream: masks [H, kq_cap, max_chunks, 2].
int attn_max_chunks(int N, int kk_cap, int chunk);
void k_chunk_masks(int H, int kq_cap, int kk_cap, int max_chunks, const int2 *runs, const int2 *info,
                   uint32_t *masks, cudaStream_t st);
// bf16: two 128-row query tiles per CTA, 128-key chunks (ac_attn3.cu); items of up to 256 rows
constexpr int ATTN3_CHUNK = 128;
int k_attention3(int D, int H, int N, const void *qg, const void *kg, const void *vg, const int32_t *qperm,
                 int kk_cap, int kq_cap, const int2 *runs, const int2 *run_info, const uint32_t *masks,
                 int max_chunks, const AttnItem *items, const int32_t *n_items, int max_items, void *out, float *lse,
                 int *status, int num_sms, void *encode_fn, cudaStream_t st, const uint16_t *rowmask = nullptr);
int k_attention(int dtype, int D, int H, int N, const void *qg, const void *kg, const void *vg,
                const int32_t *qperm, int kk_cap, int kq_cap, const int2 *runs, const int2 *run_info,
                const AttnItem *items, const int32_t *n_items, int max_items, void *out, float *lse, int *status,
                int num_sms, void *encode_fn, cudaStream_t st);

// ---- ac_perquery.cu: per-query selection (argtopk along each row of S)
// Rows of scores per batch (all heads) that fit the scratch of about 1 GiB.
size_t pq_score_batch_rows(int H, int N, int kk_cap);
// bits [H, N, W]: each query row's top_k key clusters (W = ceil(kk_cap / 32));
// head_pairs [H]: sum over rows of the selected clusters' sizes.
int k_select_rows(const void *q, int dtype, int H, int N, int D, const float *k_cent, const float *k_max,
                  const float *k_min, const int32_t *k_count, int kk_cap, const int32_t *nk, int kk_fixed,
                  int text_group, const uint8_t *dense, int score_mode, int top_k, uint32_t *bits, int W,
                  double *scores, int batch, unsigned long long *head_pairs, cudaStream_t st);
// Per query cluster: the union of its rows' sets as ascending sel_idx / sel_cnt.
void k_select_union(int H, int N, const uint32_t *bits, int W, const int32_t *qperm, const int32_t *qoff, int kq_cap,
                    const int32_t *nq, int kq_fixed, const uint8_t *dense, int kk_cap, int32_t *sel_idx,
                    int32_t *sel_cnt, cudaStream_t st);
// One key run per selected non-empty cluster (not merged).
void k_key_runs_single(int H, int kq_cap, int kk_cap, const int32_t *koff, const int32_t *sel_idx,
                       const int32_t *sel_cnt, int chunk_rows, int2 *runs, int2 *info, cudaStream_t st);
// rowmask [H, max_chunks, N]: per row (cluster order) and chunk, the 8-key groups the row keeps.
// Returns -1 (nothing launched) when its group table would not fit in shared memory.
int k_rowmask(int H, int N, int kq_cap, int kk_cap, int max_chunks, const int32_t *koff, const int2 *runs,
              const int2 *info, const int32_t *qperm, const int32_t *qoff, const uint32_t *bits, int W,
              uint16_t *rowmask, cudaStream_t st);

// The key rows of one work item as a stream of pieces: the rows of each run in
// turn (all rows [0, dense_rows) of a dense head).  piece(room) hands out the
// current run's next min(room, left) rows; their slot in the chunk is that
// count rounded up to 8 rows.  A chunk takes pieces until its `cap` rows are
// full or the stream ends, so every chunk but the last is exactly full.  The
// work-list builder and the roles of the attention kernel that need the
// pieces step through the same sequence.
struct KeyStream {
    const int2 *run;
    int nrun, ri, cur, end;
    int2 nxt;
    __device__ __forceinline__ void init(const int2 *runs, int n, int dense_rows) {
        run = runs;
        nrun = runs ? n : 1;
        ri = -1;
        cur = end = 0;
        nxt = runs ? (n > 0 ? runs[0] : make_int2(0, 0)) : make_int2(0, dense_rows);
    }
    __device__ __forceinline__ bool piece(int room, int &start, int &valid, int &slot) {
        while (cur >= end) {
            if (++ri >= nrun) return false;
            cur = nxt.x;
            end = nxt.y;
            if (run && ri + 1 < nrun) nxt = run[ri + 1];  // one run ahead
        }
        start = cur;
        valid = min(room, end - cur);
        slot = (valid + 7) & ~7;
        cur += valid;
        return true;
    }
};

}  // namespace ac
