// C ABI of libadacluster.so: argument checks, workspace layout and the host
// orchestration of AdaCluster's Algorithm 3 ("AdaCluster: Adaptive Query-Key
// Clustering for Sparse Attention in Video Generation", §3.3).  All compute
// runs in the kernels of this directory; this file only launches them.
#include <algorithm>
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "adacluster.h"
#include "ac_kernels.cuh"
#include "ac_multistage.cuh"

using namespace ac;

void ac_or_flags(int H, const uint8_t *a, uint8_t *b, cudaStream_t st);
void wait_selftest_launch(uint64_t limit_ns, int *status, cudaStream_t st);

static std::atomic<long long> g_launches{0};
namespace ac {
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
void note_launches(long long n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
long long launches_total() { return g_launches.load(std::memory_order_relaxed); }
}  // namespace ac

constexpr int PROF_RING = 256;
constexpr int PROF_EV = 6;

struct ac_ctx {
    ac_config cfg;
    int kq_cap, kk_cap, cap_max;
    int elt;
    int *d_status;     // [8] device status words
    int32_t *d_info;   // [8] device -> host control summary
    int32_t *h_info;   // [8] pinned host mirror
    int num_sms;
    void *encode_fn;
    cudaEvent_t ev[8];
    cudaEvent_t *prof;     // [PROF_RING][PROF_EV]
    long long prof_n;      // calls recorded since the last read
    long long launch_base;
    // ac_forward's captured launch sequences, by the call's buffers
    struct GraphSlot {
        const void *key[7];
        size_t ws_bytes;
        cudaGraphExec_t exec;  // null: seen once, not captured yet
        long long launches;
        bool used;
    } graphs[4];
    int graph_next;
    bool graph_off;  // a capture failed: run launch by launch from then on
    cudaStream_t cap_stream;  // captures calls made on the legacy default stream, which cannot capture
};

// ------------------------------------------------------------ workspace
namespace {
struct Bump {
    size_t off = 0;
    size_t take(size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~(size_t)255;
        return o;
    }
};

struct Ws {
    // clustering scratch
    size_t norm, U0, U1, passign, dist, rank, hist, cnt, off, perm, amb, ambc, cn2, cmax, seg, ms;
    // the k-means rounds' clusters largest first (update launch order)
    size_t uorder;
    // ac_forward internals
    size_t qa, ka, qc, kc, qcount, kcount, qmn, nq, nk, dq, dk, sel, selc;
    // attention
    size_t qperm, kperm, qoff, koff, qg, kg, vg, items, nitems, pairs, cnt2, segq, segk;
    // tensor-core screen: split centroids and per-stage gathered rows
    size_t chi, clo, cnp, xu, amb_cand, items_scr, runs, run_info, masks, kbmax, kbmin;
    // early stop of k-means: previous assignment, per-head records (q, k, Algorithm 1
    // stages), a copy of a stage's pass descriptors
    size_t aprev, kst, seg2;
    // selection: the key centroids (or Quest maxima) transposed per head, the Quest minima transposed
    size_t kct, kmt;
    // Algorithm 1's single-cluster stages on chip: working vectors [H, wrows, d] (double)
    size_t wc;
    int wrows;
    // Algorithm 1's final reassignment over the distinct centres: [H, cap, d], ids [H, cap], descriptors
    size_t cu, cmap, segu;
    // per-query selection: row bit sets [H, N, W], score batch [H, pq_batch, kk_cap] (double),
    // row masks [H, max_chunks, N] (uint16), per-head pairs [H]
    size_t rbits, pqs, rowmask, hpairs;
    int W, pq_batch;
    int kpad;
    size_t total;
};

Ws layout(const ac_ctx *c) {
    const ac_config &g = c->cfg;
    const size_t H = g.heads, N = g.n, D = g.d;
    const size_t HN = H * N;
    const size_t capm = c->cap_max;
    Bump b;
    Ws w;
    w.norm = b.take(HN * 8);
    w.U0 = b.take(HN * 4);
    w.U1 = b.take(HN * 4);
    w.passign = b.take(HN * 4);
    w.dist = b.take(HN * 8);
    w.rank = b.take(HN * 4);
    w.hist = b.take(sort_hist_elems((int)H, (int)N, (int)capm) * 4);
    w.cnt = b.take(H * capm * 4);
    w.off = b.take(H * (capm + 1) * 4);
    w.uorder = b.take(H * capm * 4);
    w.perm = b.take(HN * 4);
    w.amb = b.take(HN * 4);
    w.ambc = b.take(H * 4);
    w.cn2 = b.take(H * capm * 4);
    w.cmax = b.take(H * 4);
    w.seg = b.take(H * sizeof(HeadSeg));
    w.ms = b.take(H * sizeof(MsHead));
    w.qa = b.take(HN * 4);
    w.ka = b.take(HN * 4);
    w.qc = b.take(H * c->kq_cap * D * 4);
    w.kc = b.take(H * c->kk_cap * D * 4);
    w.qcount = b.take(H * c->kq_cap * 4);
    w.kcount = b.take(H * c->kk_cap * 4);
    w.qmn = b.take(H * c->kq_cap * 4);
    w.nq = b.take(H * 4);
    w.nk = b.take(H * 4);
    w.dq = b.take(H);
    w.dk = b.take(H);
    w.sel = b.take(H * (size_t)c->kq_cap * c->kk_cap * 4);
    w.selc = b.take(H * c->kq_cap * 4);
    w.qperm = b.take(HN * 4);
    w.kperm = b.take(HN * 4);
    w.qoff = b.take(H * (c->kq_cap + 1) * 4);
    w.koff = b.take(H * (c->kk_cap + 1) * 4);
    w.qg = b.take(HN * D * c->elt);
    w.kg = b.take(HN * D * c->elt);
    w.vg = b.take(HN * D * c->elt);
    w.items = b.take((size_t)attn_max_items((int)H, (int)N, c->kq_cap) * sizeof(AttnItem));
    w.nitems = b.take(16);
    w.pairs = b.take(16);
    w.cnt2 = b.take(H * capm * 4);
    w.segq = b.take(H * sizeof(HeadSeg));
    w.segk = b.take(H * sizeof(HeadSeg));
    w.kpad = (int)((capm + 127) / 128 * 128);
    w.chi = b.take(H * (size_t)w.kpad * D * 2);
    w.clo = b.take(H * (size_t)w.kpad * D * 2);
    w.cnp = b.take(H * (size_t)w.kpad * 4);
    w.xu = b.take(HN * D * c->elt);
    w.amb_cand = b.take(HN * 8);
    w.items_scr = b.take(items_scratch_elems((int)H, c->kq_cap) * 4 + 16);
    w.runs = b.take(H * (size_t)c->kq_cap * c->kk_cap * 8);
    w.run_info = b.take(H * (size_t)c->kq_cap * 8);
    w.masks = b.take(H * (size_t)c->kq_cap * attn_max_chunks(c->cfg.n, c->kk_cap, ATTN3_CHUNK) * (ATTN3_CHUNK / 64) * 4);
    const bool quest = c->cfg.score_mode == AC_SCORE_QUEST;
    w.kbmax = b.take(quest ? H * (size_t)c->kk_cap * D * 4 : 0);
    w.kbmin = b.take(quest ? H * (size_t)c->kk_cap * D * 4 : 0);
    w.aprev = b.take(HN * 4);
    w.kst = b.take(3 * H * 4 * 4);
    w.seg2 = b.take(H * sizeof(HeadSeg));
    w.kct = b.take(H * (size_t)c->kk_cap * D * 4);
    w.kmt = b.take(quest ? H * (size_t)c->kk_cap * D * 4 : 0);
    // a stage with m_t = ceil(m0 |U| / N) = 1 has |U| <= N / m0
    w.wrows = 0;
    if (g.adaptive_q) w.wrows = (int)(N / g.kq + 1);
    if (g.adaptive_k) w.wrows = std::max(w.wrows, (int)(N / g.kk + 1));
    w.wc = b.take(H * (size_t)w.wrows * D * 8);
    const bool adaptive = g.adaptive_q || g.adaptive_k;
    w.cu = b.take(adaptive ? H * capm * D * 4 : 0);
    w.cmap = b.take(adaptive ? H * capm * 4 : 0);
    w.segu = b.take(adaptive ? H * sizeof(HeadSeg) : 0);
    const bool pq = g.per_query != 0;
    w.W = (c->kk_cap + 31) / 32;
    w.pq_batch = pq ? (int)pq_score_batch_rows((int)H, (int)N, c->kk_cap) : 0;
    w.rbits = b.take(pq ? HN * w.W * 4 : 0);
    w.pqs = b.take(pq ? H * (size_t)w.pq_batch * c->kk_cap * 8 : 0);
    w.rowmask = b.take(pq ? H * (size_t)attn_max_chunks(c->cfg.n, c->kk_cap, ATTN3_CHUNK) * N * 2 : 0);
    w.hpairs = b.take(pq ? H * 8 : 0);
    w.total = b.off;
    return w;
}

template <typename P> P *at(void *ws, size_t off) { return reinterpret_cast<P *>(static_cast<char *>(ws) + off); }

#define AC_CUDA(call)                                                                    \
    do {                                                                                 \
        cudaError_t e_ = (call);                                                         \
        if (e_ != cudaSuccess) {                                                         \
            fprintf(stderr, "adacluster: %s failed: %s\n", #call, cudaGetErrorString(e_)); \
            return AC_ERR_CUDA;                                                          \
        }                                                                                \
    } while (0)

ac_status launch_check() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        fprintf(stderr, "adacluster: kernel launch failed: %s\n", cudaGetErrorString(e));
        return AC_ERR_CUDA;
    }
    return AC_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ac_status check_ws(const ac_ctx *c, void *ws, size_t ws_bytes) {
    if (!ws) return AC_ERR_WORKSPACE;
    if (ws_bytes < layout(c).total) return AC_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return AC_ERR_WORKSPACE;
    return AC_OK;
}

// One assignment step: tensor-core screen for bf16 inputs (rows of the pass
// contiguous in xc), fp32 screen otherwise; the exact pass resolves near-ties.
ac_status assign_step(ac_ctx *c, const Ws &w, void *ws, const void *x, const void *xc, const int32_t *rows,
                      const HeadSeg *seg, int nrows_max, const float *cent, int cap, int mode, int32_t *assign,
                      cudaStream_t st) {
    const ac_config &g = c->cfg;
    const int H = g.heads, N = g.n, D = g.d;
    float *cn2 = at<float>(ws, w.cn2), *cmax = at<float>(ws, w.cmax);
    int32_t *amb = at<int32_t>(ws, w.amb), *ambc = at<int32_t>(ws, w.ambc);
    const double *norm = at<double>(ws, w.norm);
    if (g.dtype == AC_BF16) {
        AC_CUDA(cudaMemsetAsync(ambc, 0, sizeof(int32_t) * H, st));
        if (k_assign_tc(xc, H, N, D, rows, seg, nrows_max, cent, cap, w.kpad, at<void>(ws, w.chi),
                        at<void>(ws, w.clo), cn2, cmax, norm, mode, assign, amb, ambc, at<int2>(ws, w.amb_cand),
                        c->d_status, c->encode_fn, at<float>(ws, w.cnp), c->num_sms, st) != 0)
            return AC_ERR_CUDA;
        k_assign_exact(x, DT_BF16, H, N, D, rows, seg, cent, cap, norm, mode, amb, ambc, at<int2>(ws, w.amb_cand),
                       assign, st);
    } else {
        k_assign(x, DT_F32, H, N, D, rows, seg, nrows_max, cent, cap, cn2, cmax, norm, mode, assign, amb, ambc, st);
    }
    return AC_OK;
}

#define AC_TRY(expr)                   \
    do {                               \
        ac_status s_ = (expr);         \
        if (s_ != AC_OK) return s_;    \
    } while (0)

// ------------------------------------------------------ clustering driver
// One k-means run per head (fixed count) or Algorithm 1 (adaptive), all heads
// batched in every launch.
// Clustering of every head (fixed-count k-means, or Algorithm 1 when the
// config is adaptive).  ncl_fixed / flag_fixed (device, [H], nullable): per-head
// counts and dense flags kept from an earlier call; they select the fixed-count
// path with those counts.  kst (device, [H, 4]): the fixed-count path's
// convergence record (see k_conv_decide).
ac_status run_cluster(ac_ctx *c, int mode, const void *x, const float *init, int32_t *assign, float *cent,
                      int32_t *count, float *mean_norm, int32_t *ncl, uint8_t *flag, void *ws, cudaStream_t st,
                      int *max_stages, const int32_t *ncl_fixed = nullptr, const uint8_t *flag_fixed = nullptr) {
    const ac_config &g = c->cfg;
    const int H = g.heads, N = g.n, D = g.d;
    const int dt = g.dtype == AC_BF16 ? DT_BF16 : DT_F32;
    const bool q = (mode == MODE_SPHERE);
    const int cap = q ? c->kq_cap : c->kk_cap;
    const int k = q ? g.kq : g.kk;
    const bool adaptive = (q ? g.adaptive_q : g.adaptive_k) && !ncl_fixed;
    const int nmax = q ? g.nmax_q : g.nmax_k;
    // keys: the text strip (the last text_keys rows) is not clustered
    const int text = q ? 0 : g.text_keys;
    const int Nc = N - text;
    Ws w = layout(c);
    double *norm = at<double>(ws, w.norm);
    HeadSeg *seg = at<HeadSeg>(ws, w.seg);
    int32_t *perm = at<int32_t>(ws, w.perm), *off = at<int32_t>(ws, w.off);
    int32_t *rank = at<int32_t>(ws, w.rank), *hist = at<int32_t>(ws, w.hist);
    int32_t *cnt = at<int32_t>(ws, w.cnt);
    int32_t *uorder = at<int32_t>(ws, w.uorder);
    float *cn2 = at<float>(ws, w.cn2), *cmax = at<float>(ws, w.cmax);
    int32_t *amb = at<int32_t>(ws, w.amb), *ambc = at<int32_t>(ws, w.ambc);
    int *status = c->d_status;

    k_row_norm(x, dt, H, N, D, norm, (g.flags & AC_FLAG_CHECK_FINITE) ? 1 : 0, status, st);
    if (!adaptive) {
        // per-head counts (kept from an earlier call) or the configured count
        const int kmax = ncl_fixed ? cap : k;
        auto set_seg = [&]() {
            if (ncl_fixed) k_seg_from_counts(H, Nc, ncl_fixed, k, cap, seg, status, st, text > 0 ? 1 : 0);
            else k_seg_uniform(H, Nc, k, seg, ncl, flag, st);
        };
        set_seg();
        if (ncl_fixed) {
            AC_CUDA(cudaMemcpyAsync(ncl, ncl_fixed, sizeof(int32_t) * H, cudaMemcpyDeviceToDevice, st));
            AC_CUDA(cudaMemcpyAsync(flag, flag_fixed, H, cudaMemcpyDeviceToDevice, st));
        }
        if (init && init != cent)
            AC_CUDA(cudaMemcpyAsync(cent, init, sizeof(float) * H * cap * D, cudaMemcpyDeviceToDevice, st));
        else if (!init)
            k_init_cent(x, dt, H, N, D, nullptr, norm, seg, kmax, mode, cent, cap, st);
        // Lloyd rounds; a head stops (its seg gets 0 rows) once an assignment
        // pass repeats the previous one, which leaves every result unchanged
        int32_t *kst = at<int32_t>(ws, w.kst) + (q ? 0 : 4 * H);
        int32_t *prev = at<int32_t>(ws, w.aprev);
        for (int it = 0; it < g.iters; it++) {
            AC_TRY(assign_step(c, w, ws, x, x, nullptr, seg, N, cent, cap, mode, assign, st));
            k_conv_check(H, N, seg, assign, prev, kst, it == 0 ? 1 : 0, st);
            k_conv_decide(H, seg, kst, it, st);
            k_sort(assign, nullptr, seg, H, N, N, cap, rank, hist, cnt, off, perm, status, st, uorder);
            k_update(x, dt, H, N, D, seg, kmax, perm, off, cap, norm, mode, cent, st, uorder);
        }
        // the last pass for the heads still running; then all heads again
        AC_TRY(assign_step(c, w, ws, x, x, nullptr, seg, N, cent, cap, mode, assign, st));
        if (g.iters > 0) set_seg();
        k_sort(assign, nullptr, seg, H, N, N, cap, rank, hist, count, off, perm, status, st);
        if (mean_norm) k_mean_norm(H, N, seg, perm, off, cap, norm, mean_norm, st);
        if (text > 0) k_text_group(H, N, Nc, seg, assign, count, cap, ncl, st);
        if (max_stages) *max_stages = 1;
        return launch_check();
    }
    // ---- Algorithm 1
    int32_t *U = at<int32_t>(ws, w.U0), *Un = at<int32_t>(ws, w.U1);
    int32_t *pa = at<int32_t>(ws, w.passign);
    double *dist = at<double>(ws, w.dist);
    MsHead *ms = at<MsHead>(ws, w.ms);
    k_ms_init(H, N, Nc, ms, U, Un, st);
    bool on_chip = false;
    for (int t = 0;; t++) {
        k_ms_control(H, Nc, k, nmax, cap - (text > 0 ? 1 : 0), ms, seg, c->d_info, status, st);
        AC_CUDA(cudaMemcpyAsync(c->h_info, c->d_info, 8 * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
        AC_CUDA(cudaStreamSynchronize(st));
        if (c->h_info[4]) return AC_ERR_CAPACITY;
        // heads whose last stage removed nothing skip their repeats: copy the centres
        if (c->h_info[7] > 0) k_ms_repeat(H, D, ms, cent, cap, st);
        if (c->h_info[0] == 0) break;
        const int mnu = c->h_info[1], mmt = c->h_info[2];
        // From the first stage after tau is fixed on, once every active head
        // has m_t = 1, all their remaining stages are single-cluster stages:
        // one kernel runs them all on chip (one CTA per head), without a host
        // round trip per stage.  The next control pass finds every head done.
        if (t >= 1 && mmt == 1 && !on_chip && w.wrows > 0) {
            k_ms_single(x, dt, H, N, D, Nc, k, nmax, cap - (text > 0 ? 1 : 0), g.iters, norm, mode, U, Un,
                        at<double>(ws, w.wc), w.wrows, ms, cent, cap, status, st);
            on_chip = true;
            continue;
        }
        // A stage whose every active head has one cluster (mmt = 1) is
        // complete after one round: all its rows are assigned to cluster 0, so
        // the first update already gives the centre every later round repeats
        // bit for bit.  Running one round instead of iters skips the repeats'
        // launches (most stages of a long Algorithm-1 run are such stages).
        const int iters_t = mmt == 1 ? (g.iters < 1 ? g.iters : 1) : g.iters;
        k_init_cent(x, dt, H, N, D, U, norm, seg, mmt, mode, cent, cap, st);
        void *xu = at<void>(ws, w.xu);
        if (dt == DT_BF16) k_gather_rows(x, xu, U, H, N, D * c->elt, st);
        // the stage's k-means stops per head like the fixed-count one (a
        // repeated assignment is a fixed point); the stage's pass descriptors
        // are kept and put back for the steps after it
        HeadSeg *seg_keep = at<HeadSeg>(ws, w.seg2);
        int32_t *kst = at<int32_t>(ws, w.kst) + 8 * H;
        int32_t *prev = at<int32_t>(ws, w.aprev);
        if (iters_t > 0) AC_CUDA(cudaMemcpyAsync(seg_keep, seg, sizeof(HeadSeg) * H, cudaMemcpyDeviceToDevice, st));
        for (int it = 0; it < iters_t; it++) {
            AC_TRY(assign_step(c, w, ws, x, xu, U, seg, mnu, cent, cap, mode, pa, st));
            k_conv_check(H, N, seg, pa, prev, kst, it == 0 ? 1 : 0, st);
            k_conv_decide(H, seg, kst, it, st);
            k_sort(pa, U, seg, H, N, mnu, cap, rank, hist, cnt, off, perm, status, st, uorder);
            k_update(x, dt, H, N, D, seg, mmt, perm, off, cap, norm, mode, cent, st, uorder);
        }
        AC_TRY(assign_step(c, w, ws, x, xu, U, seg, mnu, cent, cap, mode, pa, st));
        if (iters_t > 0) AC_CUDA(cudaMemcpyAsync(seg, seg_keep, sizeof(HeadSeg) * H, cudaMemcpyDeviceToDevice, st));
        k_dist(x, dt, H, N, D, U, seg, mnu, cent, cap, norm, mode, pa, dist, st);
        if (t == 0) {
            if (g.tau_rule == AC_TAU_MEDIAN_RADIUS_X)
                k_sort(pa, U, seg, H, N, mnu, cap, rank, hist, cnt, off, perm, status, st);
            k_ms_tau(H, N, (int)g.tau_rule, (double)g.tau_value, seg, dist, perm, off, cap, mmt, ms, st);
        }
        k_ms_remove(H, N, seg, dist, U, Un, ms, st);
        int32_t *tmp = U;
        U = Un;
        Un = tmp;
        AC_CUDA(cudaGetLastError());
    }
    k_ms_final(H, Nc, ms, seg, ncl, flag, c->d_info, st);
    if (max_stages) {
        // stages run by the host loop and on chip: max over heads (info[6])
        AC_CUDA(cudaMemcpyAsync(c->h_info, c->d_info, 8 * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
        AC_CUDA(cudaStreamSynchronize(st));
        *max_stages = c->h_info[6];
    }
    // Final reassignment of every token to the closest centre of C (ties to the
    // lowest id).  Stages that repeat leave identical centres in C; the pass runs
    // over the distinct ones (the first of identical centres, in id order) and
    // maps the ids back, which is the same assignment at a fraction of the work.
    {
        float *cu = at<float>(ws, w.cu);
        int32_t *cmap = at<int32_t>(ws, w.cmap);
        HeadSeg *segu = at<HeadSeg>(ws, w.segu);
        k_dedup_cent(H, D, seg, cent, cap, cu, cmap, segu, st);
        AC_TRY(assign_step(c, w, ws, x, x, nullptr, segu, N, cu, cap, mode, assign, st));
        k_map_ids(H, N, seg, cmap, cap, assign, st);
    }
    k_sort(assign, nullptr, seg, H, N, N, cap, rank, hist, count, off, perm, status, st);
    if (mean_norm) k_mean_norm(H, N, seg, perm, off, cap, norm, mean_norm, st);
    if (text > 0) k_text_group(H, N, Nc, seg, assign, count, cap, ncl, st);
    return launch_check();
}

// row_bits (device, [H, N, W], nullable): per-query selection.  Each query row
// attends only to the key clusters of its own bit set; the work list takes the
// union of the sets of each query cluster (sel / selc are then ignored).
ac_status do_sparse_attn(ac_ctx *c, const void *q, const void *k, const void *v, const int32_t *qa,
                         const int32_t *ka, const int32_t *sel, const int32_t *selc, const int32_t *nq,
                         const int32_t *nk, const uint8_t *dense, void *out, float *lse, void *ws, cudaStream_t st,
                         int64_t *pairs_dev, cudaEvent_t *ev_kernel = nullptr, const uint32_t *row_bits = nullptr) {
    const ac_config &g = c->cfg;
    const int H = g.heads, N = g.n, D = g.d;
    Ws w = layout(c);
    HeadSeg *sq = at<HeadSeg>(ws, w.segq), *sk = at<HeadSeg>(ws, w.segk);
    int32_t *rank = at<int32_t>(ws, w.rank), *hist = at<int32_t>(ws, w.hist), *cnt = at<int32_t>(ws, w.cnt2);
    int32_t *qperm = at<int32_t>(ws, w.qperm), *kperm = at<int32_t>(ws, w.kperm);
    int32_t *qoff = at<int32_t>(ws, w.qoff), *koff = at<int32_t>(ws, w.koff);
    void *qg = at<void>(ws, w.qg), *kg = at<void>(ws, w.kg), *vg = at<void>(ws, w.vg);
    AttnItem *items = at<AttnItem>(ws, w.items);
    int32_t *nitems = at<int32_t>(ws, w.nitems);
    k_seg_from_counts(H, N, nq, g.kq, c->kq_cap, sq, c->d_status, st);
    k_seg_from_counts(H, N, nk, g.kk + (g.text_keys > 0 ? 1 : 0), c->kk_cap, sk, c->d_status, st);
    k_sort(qa, nullptr, sq, H, N, N, c->kq_cap, rank, hist, cnt, qoff, qperm, c->d_status, st);
    k_sort(ka, nullptr, sk, H, N, N, c->kk_cap, rank, hist, cnt, koff, kperm, c->d_status, st);
    const int rb = D * c->elt;
    k_gather_rows(q, qg, qperm, H, N, rb, st);
    k_gather_rows(k, kg, kperm, H, N, rb, st);
    k_gather_rows(v, vg, kperm, H, N, rb, st);
    const bool two_tiles = (g.dtype == AC_BF16);  // bf16: two query tiles per CTA (items of 256 rows)
    if (row_bits) {
        // the union of each query cluster's row sets is the cluster's key stream
        sel = at<int32_t>(ws, w.sel);
        selc = at<int32_t>(ws, w.selc);
        k_select_union(H, N, row_bits, w.W, qperm, qoff, c->kq_cap, nq, g.kq, dense, c->kk_cap,
                       const_cast<int32_t *>(sel), const_cast<int32_t *>(selc), st);
    }
    k_build_items(H, N, two_tiles ? 256 : 128, c->kq_cap, c->kk_cap, qoff, nq, dense, g.kq, koff, sel, selc, items,
                  nitems, pairs_dev, at<int32_t>(ws, w.items_scr), c->d_status, st);
    int2 *runs = at<int2>(ws, w.runs), *run_info = at<int2>(ws, w.run_info);
    if (row_bits) k_key_runs_single(H, c->kq_cap, c->kk_cap, koff, sel, selc, ATTN3_CHUNK, runs, run_info, st);
    else k_key_runs(H, c->kq_cap, c->kk_cap, koff, sel, selc, ATTN3_CHUNK, runs, run_info, st);
    const int max_chunks = attn_max_chunks(N, c->kk_cap, ATTN3_CHUNK);
    uint32_t *masks = at<uint32_t>(ws, w.masks);
    if (two_tiles) k_chunk_masks(H, c->kq_cap, c->kk_cap, max_chunks, runs, run_info, masks, st);
    uint16_t *rowmask = nullptr;
    if (row_bits) {
        rowmask = at<uint16_t>(ws, w.rowmask);
        if (k_rowmask(H, N, c->kq_cap, c->kk_cap, max_chunks, koff, runs, run_info, qperm, qoff, row_bits, w.W,
                      rowmask, st) != 0)
            return AC_ERR_UNSUPPORTED;
    }
    if (ev_kernel) cudaEventRecord(ev_kernel[0], st);
    int rc;
    if (two_tiles)
        rc = k_attention3(D, H, N, qg, kg, vg, qperm, c->kk_cap, c->kq_cap, runs, run_info, masks, max_chunks, items,
                          nitems, attn_max_items(H, N, c->kq_cap), out, lse, c->d_status, c->num_sms, c->encode_fn,
                          st, rowmask);
    else
        rc = k_attention(DT_F32, D, H, N, qg, kg, vg, qperm, c->kk_cap, c->kq_cap, runs, run_info, items, nitems,
                         attn_max_items(H, N, c->kq_cap), out, lse, c->d_status, c->num_sms, c->encode_fn, st);
    if (rc != 0) return AC_ERR_CUDA;
    if (ev_kernel) cudaEventRecord(ev_kernel[1], st);
    return launch_check();
}

ac_status validate(const ac_config *g) {
    if (!g) return AC_ERR_INVALID_ARG;
    if (g->heads < 1 || g->n < 1 || g->iters < 0) return AC_ERR_INVALID_ARG;
    if (g->d != 64 && g->d != 128) return AC_ERR_UNSUPPORTED;
    if (g->dtype != AC_F32 && g->dtype != AC_BF16) return AC_ERR_INVALID_ARG;
    if (g->kq < 1 || g->kk < 1 || g->kq > g->n || g->kk > g->n) return AC_ERR_INVALID_ARG;
    if (!(g->top_p > 0.0)) return AC_ERR_INVALID_ARG;
    if (g->score_mode != AC_SCORE_CENTROID && g->score_mode != AC_SCORE_QUEST) return AC_ERR_INVALID_ARG;
    if (g->top_k < 0) return AC_ERR_INVALID_ARG;
    if (g->text_keys < 0 || g->text_keys >= g->n || (g->text_keys > 0 && g->kk > g->n - g->text_keys))
        return AC_ERR_INVALID_ARG;
    if ((long long)g->heads * g->n > 0x7fffffffLL / 2) return AC_ERR_UNSUPPORTED;
    if (g->per_query != 0 && g->per_query != 1) return AC_ERR_INVALID_ARG;
    // per-query selection: argtopk (Algorithm 3's form) on the bf16 path
    if (g->per_query && (g->top_k <= 0 || g->dtype != AC_BF16)) return AC_ERR_UNSUPPORTED;
    if (g->adaptive_q && g->nmax_q < 1) return AC_ERR_INVALID_ARG;
    if (g->adaptive_k && g->nmax_k < 1) return AC_ERR_INVALID_ARG;
    if ((g->adaptive_q || g->adaptive_k) &&
        (g->tau_rule < AC_TAU_ABS || g->tau_rule > AC_TAU_MEDIAN_RADIUS_X || !(g->tau_value >= 0.0)))
        return AC_ERR_INVALID_ARG;
    return AC_OK;
}
}  // namespace

namespace {
// Sort the keys by cluster (into the workspace's key permutation and offsets)
// and take each cluster's per-dimension max / min.
void key_bounds(ac_ctx *c, const void *k, const int32_t *ka, const int32_t *nk, float *kmax, float *kmin, void *ws,
                cudaStream_t st) {
    const ac_config &g = c->cfg;
    Ws w = layout(c);
    HeadSeg *sk = at<HeadSeg>(ws, w.segk);
    int32_t *kperm = at<int32_t>(ws, w.kperm), *koff = at<int32_t>(ws, w.koff);
    k_seg_from_counts(g.heads, g.n, nk, g.kk + (g.text_keys > 0 ? 1 : 0), c->kk_cap, sk, c->d_status, st);
    k_sort(ka, nullptr, sk, g.heads, g.n, g.n, c->kk_cap, at<int32_t>(ws, w.rank), at<int32_t>(ws, w.hist),
           at<int32_t>(ws, w.cnt2), koff, kperm, c->d_status, st);
    k_cluster_bounds(k, g.dtype == AC_BF16 ? DT_BF16 : DT_F32, g.heads, g.n, g.d, kperm, koff, c->kk_cap, kmax, kmin,
                     st);
}
}  // namespace

// ------------------------------------------------------------------ ABI
extern "C" {

const char *ac_status_string(ac_status s) {
    switch (s) {
    case AC_OK: return "ok";
    case AC_ERR_INVALID_ARG: return "invalid argument";
    case AC_ERR_UNSUPPORTED: return "unsupported configuration";
    case AC_ERR_CUDA: return "CUDA error";
    case AC_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case AC_ERR_TIMEOUT: return "device wait timed out";
    case AC_ERR_NONFINITE: return "non-finite input";
    case AC_ERR_CAPACITY: return "adaptive clustering exceeded its capacity";
    }
    return "unknown status";
}

ac_status ac_create(const ac_config *cfg, ac_ctx **out) {
    if (!out) return AC_ERR_INVALID_ARG;
    *out = nullptr;
    ac_status v = validate(cfg);
    if (v != AC_OK) return v;
    ac_ctx *c = (ac_ctx *)calloc(1, sizeof(ac_ctx));
    if (!c) return AC_ERR_INVALID_ARG;
    c->cfg = *cfg;
    c->kq_cap = cfg->adaptive_q ? cfg->nmax_q + cfg->kq : cfg->kq;
    c->kk_cap = (cfg->adaptive_k ? cfg->nmax_k + cfg->kk : cfg->kk) + (cfg->text_keys > 0 ? 1 : 0);
    c->cap_max = c->kq_cap > c->kk_cap ? c->kq_cap : c->kk_cap;
    c->elt = cfg->dtype == AC_BF16 ? 2 : 4;
    if (c->cap_max > 8192) {
        free(c);
        return AC_ERR_UNSUPPORTED;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaMalloc(&c->d_status, 8 * sizeof(int)) != cudaSuccess) {
        free(c);
        return AC_ERR_CUDA;
    }
    if (cudaMalloc(&c->d_info, 8 * sizeof(int32_t)) != cudaSuccess ||
        cudaMallocHost(&c->h_info, 8 * sizeof(int32_t)) != cudaSuccess ||
        cudaMemset(c->d_status, 0, 8 * sizeof(int)) != cudaSuccess) {
        ac_destroy(c);
        return AC_ERR_CUDA;
    }
    for (int i = 0; i < 8; i++)
        if (cudaEventCreate(&c->ev[i]) != cudaSuccess) {
            ac_destroy(c);
            return AC_ERR_CUDA;
        }
    c->prof = (cudaEvent_t *)calloc((size_t)PROF_RING * PROF_EV, sizeof(cudaEvent_t));
    if (!c->prof) {
        ac_destroy(c);
        return AC_ERR_INVALID_ARG;
    }
    for (int i = 0; i < PROF_RING * PROF_EV; i++)
        if (cudaEventCreate(&c->prof[i]) != cudaSuccess) {
            ac_destroy(c);
            return AC_ERR_CUDA;
        }
    c->launch_base = launches_total();
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &c->encode_fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || !c->encode_fn) {
        ac_destroy(c);
        return AC_ERR_CUDA;
    }
    *out = c;
    return AC_OK;
}

void ac_destroy(ac_ctx *c) {
    if (!c) return;
    for (auto &gs : c->graphs)
        if (gs.exec) cudaGraphExecDestroy(gs.exec);
    if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
    if (c->d_status) cudaFree(c->d_status);
    if (c->d_info) cudaFree(c->d_info);
    if (c->h_info) cudaFreeHost(c->h_info);
    for (int i = 0; i < 8; i++)
        if (c->ev[i]) cudaEventDestroy(c->ev[i]);
    if (c->prof) {
        for (int i = 0; i < PROF_RING * PROF_EV; i++)
            if (c->prof[i]) cudaEventDestroy(c->prof[i]);
        free(c->prof);
    }
    free(c);
}

ac_status ac_profile_read(ac_ctx *c, ac_profile *out) {
    if (!c || !out) return AC_ERR_INVALID_ARG;
    memset(out, 0, sizeof(*out));
    long long n = c->prof_n < PROF_RING ? c->prof_n : PROF_RING;
    long long first = c->prof_n - n;
    double acc[6] = {0, 0, 0, 0, 0, 0};
    for (long long i = first; i < c->prof_n; i++) {
        cudaEvent_t *e = c->prof + (size_t)(i % PROF_RING) * PROF_EV;
        AC_CUDA(cudaEventSynchronize(e[5]));
        float ms;
        const int a[6][2] = {{0, 1}, {1, 2}, {2, 3}, {3, 4}, {4, 5}, {0, 5}};
        for (int j = 0; j < 6; j++) {
            AC_CUDA(cudaEventElapsedTime(&ms, e[a[j][0]], e[a[j][1]]));
            acc[j] += ms;
        }
    }
    out->calls = (int)n;
    if (n > 0) {
        out->ms_cluster_q = acc[0] / n;
        out->ms_cluster_k = acc[1] / n;
        out->ms_select = acc[2] / n;
        out->ms_prep = acc[3] / n;
        out->ms_attn_kernel = acc[4] / n;
        out->ms_total = acc[5] / n;
    }
    long long now = launches_total();
    out->launches = now - c->launch_base;
    c->launch_base = now;
    c->prof_n = 0;
    return AC_OK;
}

ac_status ac_capacities(const ac_ctx *c, int *kq_cap, int *kk_cap) {
    if (!c) return AC_ERR_INVALID_ARG;
    if (kq_cap) *kq_cap = c->kq_cap;
    if (kk_cap) *kk_cap = c->kk_cap;
    return AC_OK;
}

}  // extern "C"

namespace {

// Where ac_forward's stages read their inputs and leave their outputs.
struct Fwd {
    const float *q_init = nullptr, *k_init = nullptr;  // warm-start centres (nullable)
    float *q_cent = nullptr, *k_cent = nullptr;        // centre outputs (nullable: workspace)
    const int32_t *nq_fixed = nullptr, *nk_fixed = nullptr;  // per-head counts kept from step 0
    const uint8_t *dq_fixed = nullptr, *dk_fixed = nullptr;  // per-head dense flags kept from step 0
};

// Caller-owned state of the multi-step driver: {nq [H], nk [H], dq [H], dk [H],
// q centres [H, kq_cap, d], k centres [H, kk_cap, d]}, 256-byte aligned parts.
struct StepState {
    int32_t *nq, *nk;
    uint8_t *dq, *dk;
    float *q_cent, *k_cent;
    size_t total;
};
StepState step_state(const ac_ctx *c, void *base) {
    const size_t H = c->cfg.heads, D = c->cfg.d;
    Bump b;
    const size_t onq = b.take(H * 4), onk = b.take(H * 4), odq = b.take(H), odk = b.take(H);
    const size_t oqc = b.take(H * (size_t)c->kq_cap * D * 4), okc = b.take(H * (size_t)c->kk_cap * D * 4);
    StepState ss;
    ss.total = b.off;
    char *p = static_cast<char *>(base);
    ss.nq = base ? reinterpret_cast<int32_t *>(p + onq) : nullptr;
    ss.nk = base ? reinterpret_cast<int32_t *>(p + onk) : nullptr;
    ss.dq = base ? reinterpret_cast<uint8_t *>(p + odq) : nullptr;
    ss.dk = base ? reinterpret_cast<uint8_t *>(p + odk) : nullptr;
    ss.q_cent = base ? reinterpret_cast<float *>(p + oqc) : nullptr;
    ss.k_cent = base ? reinterpret_cast<float *>(p + okc) : nullptr;
    return ss;
}

// Max over heads of the rounds the fixed-count k-means ran (kst [H, 4]); 0 if
// nothing was recorded.
int max_rounds(const int32_t *kst_dev, int H) {
    int32_t *h = (int32_t *)malloc(sizeof(int32_t) * 4 * H);
    if (!h) return 0;
    int m = 0;
    if (cudaMemcpy(h, kst_dev, sizeof(int32_t) * 4 * H, cudaMemcpyDeviceToHost) == cudaSuccess)
        for (int i = 0; i < H; i++) m = h[4 * i + 2] > m ? h[4 * i + 2] : m;
    free(h);
    return m;
}

// Algorithm 3 for every head: both clusterings, the selection and the sparse
// attention, on one stream.
ac_status forward_impl(ac_ctx *c, const void *q, const void *k, const void *v, const Fwd &f, void *out,
                       ac_stats *stats, void *ws, cudaStream_t st) {
    const ac_config &g = c->cfg;
    Ws w = layout(c);
    float *qc = f.q_cent ? f.q_cent : at<float>(ws, w.qc);
    float *kc = f.k_cent ? f.k_cent : at<float>(ws, w.kc);
    int32_t *qa = at<int32_t>(ws, w.qa), *ka = at<int32_t>(ws, w.ka);
    int32_t *qn = at<int32_t>(ws, w.qcount), *kn = at<int32_t>(ws, w.kcount);
    float *qmn = at<float>(ws, w.qmn);
    int32_t *nq = at<int32_t>(ws, w.nq), *nk = at<int32_t>(ws, w.nk);
    uint8_t *dq = at<uint8_t>(ws, w.dq), *dk = at<uint8_t>(ws, w.dk);
    int32_t *sel = at<int32_t>(ws, w.sel), *selc = at<int32_t>(ws, w.selc);
    int32_t *kst = at<int32_t>(ws, w.kst);
    int sq = 1, sk = 1;
    cudaEvent_t *pe = nullptr;
    if (g.flags & AC_FLAG_PROFILE) {
        pe = c->prof + (size_t)(c->prof_n % PROF_RING) * PROF_EV;
        c->prof_n++;
        AC_CUDA(cudaEventRecord(pe[0], st));
    }
    if (stats) {
        AC_CUDA(cudaMemsetAsync(kst, 0, sizeof(int32_t) * 8 * g.heads, st));
        AC_CUDA(cudaEventRecord(c->ev[0], st));
    }
    ac_status s = run_cluster(c, MODE_SPHERE, q, f.q_init, qa, qc, qn, qmn, nq, dq, ws, st, stats ? &sq : nullptr,
                              f.nq_fixed, f.dq_fixed);
    if (s != AC_OK) return s;
    if (pe) AC_CUDA(cudaEventRecord(pe[1], st));
    if (stats) AC_CUDA(cudaEventRecord(c->ev[1], st));
    s = run_cluster(c, MODE_EUCLID, k, f.k_init, ka, kc, kn, nullptr, nk, dk, ws, st, stats ? &sk : nullptr,
                    f.nk_fixed, f.dk_fixed);
    if (s != AC_OK) return s;
    if (pe) AC_CUDA(cudaEventRecord(pe[2], st));
    if (stats) AC_CUDA(cudaEventRecord(c->ev[2], st));
    // a head is dense when either clustering set its flag F
    uint8_t *dense = dk;
    if (g.adaptive_q || f.dq_fixed) ac_or_flags(g.heads, dq, dk, st);
    float *kbmax = nullptr, *kbmin = nullptr;
    if (g.score_mode == AC_SCORE_QUEST) {
        kbmax = at<float>(ws, w.kbmax);
        kbmin = at<float>(ws, w.kbmin);
        key_bounds(c, k, ka, nk, kbmax, kbmin, ws, st);
    }
    const int tg = g.text_keys > 0 ? 1 : 0;
    uint32_t *rbits = nullptr;
    if (g.per_query) {
        // Algorithm 3's argtopk along each row of S: every query row's own set
        rbits = at<uint32_t>(ws, w.rbits);
        k_select_rows(q, DT_BF16, g.heads, g.n, g.d, kc, kbmax, kbmin, kn, c->kk_cap, nk, g.kk + tg, tg, dense,
                      (int)g.score_mode, g.top_k, rbits, w.W, at<double>(ws, w.pqs), w.pq_batch,
                      at<unsigned long long>(ws, w.hpairs), st);
    } else {
        k_select(g.heads, g.d, qc, qmn, qn, c->kq_cap, kc, kn, kbmax, kbmin, c->kk_cap, nq, nk, g.kq, g.kk + tg, dense,
                 (int)g.score_mode, g.top_k, g.top_p, sel, selc, c->d_status, st, tg, at<float>(ws, w.kct),
                 g.score_mode == AC_SCORE_QUEST ? at<float>(ws, w.kmt) : nullptr);
    }
    if (pe) AC_CUDA(cudaEventRecord(pe[3], st));
    if (stats) AC_CUDA(cudaEventRecord(c->ev[3], st));
    s = do_sparse_attn(c, q, k, v, qa, ka, sel, selc, nq, nk, dense, out, nullptr, ws, st, at<int64_t>(ws, w.pairs),
                       pe ? pe + 4 : nullptr, rbits);
    if (s != AC_OK) return s;
    if (stats) {
        AC_CUDA(cudaEventRecord(c->ev[4], st));
        AC_CUDA(cudaEventSynchronize(c->ev[4]));
        float ms[4];
        cudaEventElapsedTime(&ms[0], c->ev[0], c->ev[1]);
        cudaEventElapsedTime(&ms[1], c->ev[1], c->ev[2]);
        cudaEventElapsedTime(&ms[2], c->ev[2], c->ev[3]);
        cudaEventElapsedTime(&ms[3], c->ev[3], c->ev[4]);
        memset(stats, 0, sizeof(*stats));
        stats->ms_cluster_q = ms[0];
        stats->ms_cluster_k = ms[1];
        stats->ms_select = ms[2];
        stats->ms_attn = ms[3];
        stats->ms_total = ms[0] + ms[1] + ms[2] + ms[3];
        int64_t pairs = 0;
        AC_CUDA(cudaMemcpy(&pairs, at<int64_t>(ws, w.pairs), sizeof(pairs), cudaMemcpyDeviceToHost));
        stats->pairs = pairs;
        stats->pairs_computed = pairs;
        uint8_t *hd = (uint8_t *)malloc(g.heads);
        unsigned long long *hp = (unsigned long long *)malloc(sizeof(unsigned long long) * g.heads);
        if (hd && hp) {
            AC_CUDA(cudaMemcpy(hd, dense, g.heads, cudaMemcpyDeviceToHost));
            for (int h = 0; h < g.heads; h++) stats->dense_heads += hd[h] ? 1 : 0;
            if (g.per_query) {
                // the pairs the method attends: each row's own set (dense heads: N^2)
                AC_CUDA(cudaMemcpy(hp, at<unsigned long long>(ws, w.hpairs), sizeof(unsigned long long) * g.heads,
                                   cudaMemcpyDeviceToHost));
                int64_t own = 0;
                for (int h = 0; h < g.heads; h++)
                    own += hd[h] ? (int64_t)g.n * (int64_t)g.n : (int64_t)hp[h];
                stats->pairs = own;
            }
        }
        free(hd);
        free(hp);
        stats->max_stages_q = sq;
        stats->max_stages_k = sk;
        stats->kmeans_rounds_q = max_rounds(kst, g.heads);
        stats->kmeans_rounds_k = max_rounds(kst + 4 * g.heads, g.heads);
    }
    return launch_check();
}

}  // namespace

extern "C" {

ac_status ac_workspace_size(const ac_ctx *c, size_t *bytes) {
    if (!c || !bytes) return AC_ERR_INVALID_ARG;
    *bytes = layout(c).total;
    return AC_OK;
}

ac_status ac_cluster_q(ac_ctx *c, const void *q, const float *init_cent, int32_t *assign, float *cent,
                       int32_t *count, float *mean_norm, int32_t *nclusters, uint8_t *dense_flag, void *ws,
                       size_t ws_bytes, void *stream) {
    if (!c || !q || !assign || !cent || !count || !mean_norm || !nclusters || !dense_flag) return AC_ERR_INVALID_ARG;
    if (!aligned16(q) || (init_cent && c->cfg.adaptive_q)) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    return run_cluster(c, MODE_SPHERE, q, init_cent, assign, cent, count, mean_norm, nclusters, dense_flag, ws,
                       (cudaStream_t)stream, nullptr);
}

ac_status ac_cluster_k(ac_ctx *c, const void *k, const float *init_cent, int32_t *assign, float *cent,
                       int32_t *count, int32_t *nclusters, uint8_t *dense_flag, void *ws, size_t ws_bytes,
                       void *stream) {
    if (!c || !k || !assign || !cent || !count || !nclusters || !dense_flag) return AC_ERR_INVALID_ARG;
    if (!aligned16(k) || (init_cent && c->cfg.adaptive_k)) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    return run_cluster(c, MODE_EUCLID, k, init_cent, assign, cent, count, nullptr, nclusters, dense_flag, ws,
                       (cudaStream_t)stream, nullptr);
}

ac_status ac_select(ac_ctx *c, const float *q_cent, const float *q_mean_norm, const int32_t *q_count,
                    const float *k_cent, const int32_t *k_count, const float *k_max, const float *k_min,
                    const int32_t *nq, const int32_t *nk, const uint8_t *dense_flag, int32_t *sel_idx,
                    int32_t *sel_cnt, void *ws, size_t ws_bytes, void *stream) {
    if (!c || !q_cent || !q_mean_norm || !q_count || !k_cent || !k_count || !sel_idx || !sel_cnt)
        return AC_ERR_INVALID_ARG;
    const ac_config &g = c->cfg;
    if (g.score_mode == AC_SCORE_QUEST && (!k_max || !k_min)) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    k_select(g.heads, g.d, q_cent, q_mean_norm, q_count, c->kq_cap, k_cent, k_count, k_max, k_min, c->kk_cap, nq, nk,
             g.kq, g.kk + (g.text_keys > 0 ? 1 : 0), dense_flag, (int)g.score_mode, g.top_k, g.top_p, sel_idx, sel_cnt,
             c->d_status, (cudaStream_t)stream, g.text_keys > 0 ? 1 : 0, at<float>(ws, layout(c).kct),
             g.score_mode == AC_SCORE_QUEST ? at<float>(ws, layout(c).kmt) : nullptr);
    return launch_check();
}


ac_status ac_select_rows(ac_ctx *c, const void *q, const float *k_cent, const int32_t *k_count, const float *k_max,
                         const float *k_min, const int32_t *nk, const uint8_t *dense_flag, uint32_t *row_bits,
                         void *ws, size_t ws_bytes, void *stream) {
    if (!c || !q || !k_count || !row_bits) return AC_ERR_INVALID_ARG;
    const ac_config &g = c->cfg;
    if (!g.per_query) return AC_ERR_UNSUPPORTED;
    if (g.score_mode == AC_SCORE_QUEST ? (!k_max || !k_min) : !k_cent) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    Ws w = layout(c);
    const int tg = g.text_keys > 0 ? 1 : 0;
    k_select_rows(q, DT_BF16, g.heads, g.n, g.d, k_cent, k_max, k_min, k_count, c->kk_cap, nk, g.kk + tg, tg,
                  dense_flag, (int)g.score_mode, g.top_k, row_bits, w.W, at<double>(ws, w.pqs), w.pq_batch,
                  at<unsigned long long>(ws, w.hpairs), (cudaStream_t)stream);
    return launch_check();
}

ac_status ac_sparse_attn_rows(ac_ctx *c, const void *q, const void *k, const void *v, const int32_t *q_assign,
                              const int32_t *k_assign, const uint32_t *row_bits, const int32_t *nq, const int32_t *nk,
                              const uint8_t *dense_flag, void *out, float *lse, void *ws, size_t ws_bytes,
                              void *stream) {
    if (!c || !q || !k || !v || !q_assign || !k_assign || !row_bits || !out) return AC_ERR_INVALID_ARG;
    if (!c->cfg.per_query) return AC_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    Ws w = layout(c);
    return do_sparse_attn(c, q, k, v, q_assign, k_assign, nullptr, nullptr, nq, nk, dense_flag, out, lse, ws,
                          (cudaStream_t)stream, at<int64_t>(ws, w.pairs), nullptr, row_bits);
}

ac_status ac_key_bounds(ac_ctx *c, const void *k, const int32_t *k_assign, const int32_t *nk, float *k_max,
                        float *k_min, void *ws, size_t ws_bytes, void *stream) {
    if (!c || !k || !k_assign || !k_max || !k_min) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    key_bounds(c, k, k_assign, nk, k_max, k_min, ws, (cudaStream_t)stream);
    return launch_check();
}

ac_status ac_cluster_sort(ac_ctx *c, const int32_t *assign, int cap, const int32_t *ncl, int32_t *perm,
                          int32_t *offsets, void *ws, size_t ws_bytes, void *stream) {
    if (!c || !assign || !perm || !offsets || cap < 1 || cap > c->cap_max) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    const ac_config &g = c->cfg;
    Ws w = layout(c);
    cudaStream_t st = (cudaStream_t)stream;
    HeadSeg *seg = at<HeadSeg>(ws, w.seg);
    k_seg_from_counts(g.heads, g.n, ncl, cap, cap, seg, c->d_status, st);
    k_sort(assign, nullptr, seg, g.heads, g.n, g.n, cap, at<int32_t>(ws, w.rank), at<int32_t>(ws, w.hist),
           at<int32_t>(ws, w.cnt), offsets, perm, c->d_status, st);
    return launch_check();
}

ac_status ac_sparse_attn(ac_ctx *c, const void *q, const void *k, const void *v, const int32_t *q_assign,
                         const int32_t *k_assign, const int32_t *sel_idx, const int32_t *sel_cnt,
                         const int32_t *nq, const int32_t *nk, const uint8_t *dense_flag, void *out, float *lse,
                         void *ws, size_t ws_bytes, void *stream) {
    if (!c || !q || !k || !v || !q_assign || !k_assign || !sel_idx || !sel_cnt || !out) return AC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    Ws w = layout(c);
    return do_sparse_attn(c, q, k, v, q_assign, k_assign, sel_idx, sel_cnt, nq, nk, dense_flag, out, lse, ws,
                          (cudaStream_t)stream, at<int64_t>(ws, w.pairs));
}

ac_status ac_forward(ac_ctx *c, const void *q, const void *k, const void *v, float *q_cent_io, float *k_cent_io,
                     void *out, ac_stats *stats, void *ws, size_t ws_bytes, void *stream) {
    if (!c || !q || !k || !v || !out) return AC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return AC_ERR_INVALID_ARG;
    const ac_config &g = c->cfg;
    const bool warm = (g.flags & AC_FLAG_WARM_START) != 0;
    if (warm && ((q_cent_io && g.adaptive_q) || (k_cent_io && g.adaptive_k))) return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    Fwd f;
    f.q_init = (warm && q_cent_io) ? q_cent_io : nullptr;
    f.k_init = (warm && k_cent_io) ? k_cent_io : nullptr;
    f.q_cent = q_cent_io;
    f.k_cent = k_cent_io;
    const cudaStream_t st = (cudaStream_t)stream;
    const bool graphable = !stats && !(g.flags & (AC_FLAG_PROFILE | AC_FLAG_NO_GRAPH)) && !g.adaptive_q &&
                           !g.adaptive_k && !c->graph_off;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (!graphable || cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
        return forward_impl(c, q, k, v, f, out, stats, ws, st);
    // a call on the same buffers as a captured one replays it; buffers seen
    // once before are captured now; new buffers are only noted (a call that
    // never repeats its buffers pays no capture)
    const void *key[7] = {q, k, v, q_cent_io, k_cent_io, out, ws};
    ac_ctx::GraphSlot *hit = nullptr;
    for (auto &gs : c->graphs)
        if (gs.used && gs.ws_bytes == ws_bytes && memcmp(gs.key, key, sizeof(key)) == 0) hit = &gs;
    if (hit && hit->exec) {
        AC_CUDA(cudaGraphLaunch(hit->exec, st));
        note_launches(hit->launches);
        return AC_OK;
    }
    if (!hit) {
        auto &slot = c->graphs[c->graph_next];
        c->graph_next = (c->graph_next + 1) % 4;
        if (slot.exec) cudaGraphExecDestroy(slot.exec);
        memcpy(slot.key, key, sizeof(key));
        slot.ws_bytes = ws_bytes;
        slot.exec = nullptr;
        slot.used = true;
        return forward_impl(c, q, k, v, f, out, stats, ws, st);
    }
    // capture this call's launches (nothing runs during capture), then launch the
    // graph on the caller's stream, which orders it like the launches it holds.
    // The legacy default stream cannot capture: the context's own stream does.
    cudaStream_t cap = st;
    if (st == nullptr || st == cudaStreamLegacy) {
        if (!c->cap_stream && cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
            cudaGetLastError();
            c->cap_stream = nullptr;
            c->graph_off = true;
            return forward_impl(c, q, k, v, f, out, stats, ws, st);
        }
        cap = c->cap_stream;
    }
    const long long l0 = launches_total();
    if (cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        cudaGetLastError();
        c->graph_off = true;
        return forward_impl(c, q, k, v, f, out, stats, ws, st);
    }
    const ac_status s2 = forward_impl(c, q, k, v, f, out, stats, ws, cap);
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(cap, &graph);
    const long long nl = launches_total() - l0;
    cudaGraphExec_t exec = nullptr;
    if (s2 == AC_OK && e == cudaSuccess && graph && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess)
        exec = nullptr;
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    if (s2 != AC_OK) return s2;  // the argument errors a plain call returns, before any launch
    if (!exec) {
        c->graph_off = true;
        return forward_impl(c, q, k, v, f, out, stats, ws, st);
    }
    hit->exec = exec;
    hit->launches = nl;
    AC_CUDA(cudaGraphLaunch(exec, st));
    return AC_OK;
}

ac_status ac_step_state_size(const ac_ctx *c, size_t *bytes) {
    if (!c || !bytes) return AC_ERR_INVALID_ARG;
    *bytes = step_state(c, nullptr).total;
    return AC_OK;
}

ac_status ac_step_state_parts(const ac_ctx *c, void *state, void **parts) {
    if (!c || !state || !parts) return AC_ERR_INVALID_ARG;
    const StepState ss = step_state(c, state);
    parts[0] = ss.nq;
    parts[1] = ss.nk;
    parts[2] = ss.dq;
    parts[3] = ss.dk;
    parts[4] = ss.q_cent;
    parts[5] = ss.k_cent;
    return AC_OK;
}

ac_status ac_forward_step(ac_ctx *c, int step, const void *q, const void *k, const void *v, void *state, void *out,
                          ac_stats *stats, void *ws, size_t ws_bytes, void *stream) {
    if (!c || !q || !k || !v || !out || !state || step < 0) return AC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
        return AC_ERR_INVALID_ARG;
    ac_status s = check_ws(c, ws, ws_bytes);
    if (s != AC_OK) return s;
    const StepState ss = step_state(c, state);
    cudaStream_t st = (cudaStream_t)stream;
    Fwd f;
    f.q_cent = ss.q_cent;
    f.k_cent = ss.k_cent;
    if (step > 0) {
        // the counts and dense flags of step 0, k-means seeded with the
        // previous step's centres (updated in place)
        f.q_init = ss.q_cent;
        f.k_init = ss.k_cent;
        f.nq_fixed = ss.nq;
        f.nk_fixed = ss.nk;
        f.dq_fixed = ss.dq;
        f.dk_fixed = ss.dk;
    }
    s = forward_impl(c, q, k, v, f, out, stats, ws, st);
    if (s != AC_OK || step > 0) return s;
    // step 0: keep the counts and flags Algorithm 1 (or the fixed config) chose
    Ws w = layout(c);
    AC_CUDA(cudaMemcpyAsync(ss.nq, at<int32_t>(ws, w.nq), sizeof(int32_t) * c->cfg.heads, cudaMemcpyDeviceToDevice, st));
    AC_CUDA(cudaMemcpyAsync(ss.nk, at<int32_t>(ws, w.nk), sizeof(int32_t) * c->cfg.heads, cudaMemcpyDeviceToDevice, st));
    AC_CUDA(cudaMemcpyAsync(ss.dq, at<uint8_t>(ws, w.dq), c->cfg.heads, cudaMemcpyDeviceToDevice, st));
    AC_CUDA(cudaMemcpyAsync(ss.dk, at<uint8_t>(ws, w.dk), c->cfg.heads, cudaMemcpyDeviceToDevice, st));
    return launch_check();
}

ac_status ac_selftest_wait(ac_ctx *c, double seconds, void *stream) {
    if (!c || !(seconds > 0.0) || seconds > 10.0) return AC_ERR_INVALID_ARG;
    wait_selftest_launch((uint64_t)(seconds * 1e9), c->d_status, (cudaStream_t)stream);
    return launch_check();
}

ac_status ac_get_status(ac_ctx *c, void *stream) {
    if (!c) return AC_ERR_INVALID_ARG;
    AC_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    int h[8];
    AC_CUDA(cudaMemcpy(h, c->d_status, sizeof(h), cudaMemcpyDeviceToHost));
    AC_CUDA(cudaMemset(c->d_status, 0, sizeof(h)));
    return (ac_status)h[0];
}

}  // extern "C"

// One warp waits, through the kernels' bounded wait, on an mbarrier phase that
// nothing completes; the wait gives up after limit_ns and records ST_TIMEOUT.
__global__ void wait_selftest_kernel(uint64_t limit_ns, int *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ac::mbar_init(&bar, 1);
        abort_flag = 0;
        ac::fence_mbar_init();
    }
    __syncthreads();
    const bool done = ac::mbar_wait_warp(&bar, 0, &abort_flag, status, limit_ns);
    if (done && threadIdx.x == 0) ac::set_status(status, ac::ST_OK);  // unreachable: nothing arrives
}

__global__ void or_flags_kernel(int H, const uint8_t *a, uint8_t *b) {
    int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < H) b[h] = (uint8_t)(a[h] | b[h]);
}
void wait_selftest_launch(uint64_t limit_ns, int *status, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, status);
    note_launch();
}
void ac_or_flags(int H, const uint8_t *a, uint8_t *b, cudaStream_t st) {
    or_flags_kernel<<<(H + 127) / 128, 128, 0, st>>>(H, a, b); note_launch();
}
