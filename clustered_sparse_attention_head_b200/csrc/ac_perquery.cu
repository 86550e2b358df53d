// Per-query selection (AdaCluster §3.3, Algorithm 3: the score matrix S has one
// row per query token, Index <- argtopk(S, topk) along each row), and the
// tables that let the block-sparse attention kernel honour each row's own set.
//
//  1. pq_scores_c_kernel (CENTROID scores, 16-byte aligned operands) and
//     pq_scores_kernel (QUEST scores, or unaligned operands): s_ib for every
//     query row i and key cluster b, in double with the oracle's summation
//     order (elements in order): CENTROID s = (q_i . c_b) / sqrt(d); QUEST
//     s = sum_t max(q_t M_bt, q_t m_bt) / sqrt(d) (the query is its own
//     representative).  A bf16 or fp32 element times an fp32 centroid element
//     has at most 48 significant bits, so its double product is exact and one
//     fused multiply-add per element rounds exactly where a multiply then an
//     add does.
//  2. pq_topk_kernel: one warp per row keeps the top_k non-empty clusters of
//     largest s (ties to the lower id) as a bit set [H, N, W] (W = kk_cap / 32
//     words), by a warp quickselect up to 512 clusters; the text-key group, if
//     any, is always set.  It also sums the row's pairs (sum of the selected
//     clusters' sizes).
//  3. pq_union_kernel: per query cluster, the union of its rows' sets, as the
//     ascending sel_idx / sel_cnt lists the work list and key runs take.
//  4. key_runs_single_kernel: one key run per selected non-empty cluster (not
//     merged), so every 8-key group of a chunk belongs to one cluster.
//  5. pq_rowmask_kernel: per row and chunk a 16-bit mask, bit g = the row's
//     set holds the cluster of 8-key group g ([H, max_chunks, N] by the
//     row's position in cluster order); the attention kernel masks the groups
//     whose bit is clear.
#include "ac_kernels.cuh"

namespace ac {

// Score tiles of 64 rows x 64 clusters per 256-thread CTA, each thread 4 x 4;
// operands staged in shared memory as doubles, element-major (so a thread's
// four rows or four clusters of one element are two 16-byte loads), rows of
// PQ_LD doubles
constexpr int PQ_ROWS = 64, PQ_COLS = 64, PQ_LD = 66;

template <typename T, int D>
__global__ void __launch_bounds__(256) pq_scores_kernel(const T *__restrict__ q, int N, int r0, int nb,
                                                        const float *__restrict__ k_cent,
                                                        const float *__restrict__ k_max,
                                                        const float *__restrict__ k_min, int kk_cap,
                                                        const int32_t *__restrict__ nk, int kk_fixed, int text_group,
                                                        int score_mode, double *__restrict__ scores) {
    extern __shared__ double pqs[];
    double *qs = pqs;                 // [D][PQ_LD]: element t of row r at qs[t * PQ_LD + r]
    double *cs = qs + D * PQ_LD;      // [D][PQ_LD]: centroid (or M) element t of cluster c
    double *ms = cs + D * PQ_LD;      // [D][PQ_LD]: m (Quest only)
    const int h = blockIdx.z, tid = threadIdx.x;
    const int nkh = (nk ? min(max(nk[h], 0), kk_cap) : kk_fixed) - text_group;
    const int b0 = blockIdx.y * PQ_COLS, i0 = blockIdx.x * PQ_ROWS;
    if (b0 >= nkh) return;
    for (int e = tid; e < PQ_ROWS * D; e += 256) {
        const int r = e / D, t = e - r * D;
        const int i = r0 + i0 + r;
        qs[t * PQ_LD + r] = (i0 + r < nb && i < N) ? (double)to_f(q[((size_t)h * N + i) * D + t]) : 0.0;
    }
    for (int e = tid; e < PQ_COLS * D; e += 256) {
        const int c = e / D, t = e - c * D;
        const int b = b0 + c;
        const size_t o = ((size_t)h * kk_cap + b) * D + t;
        if (score_mode == 1) {
            cs[t * PQ_LD + c] = b < nkh ? (double)k_max[o] : 0.0;
            ms[t * PQ_LD + c] = b < nkh ? (double)k_min[o] : 0.0;
        } else {
            cs[t * PQ_LD + c] = b < nkh ? (double)k_cent[o] : 0.0;
        }
    }
    __syncthreads();
    const int tx = tid & 15, ty = tid >> 4;  // clusters 4 tx .. 4 tx + 3, rows 4 ty .. 4 ty + 3
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = 0.0;
    if (score_mode == 1) {
        for (int t = 0; t < D; t++) {
            const double2 qa = *reinterpret_cast<const double2 *>(qs + t * PQ_LD + 4 * ty);
            const double2 qb = *reinterpret_cast<const double2 *>(qs + t * PQ_LD + 4 * ty + 2);
            const double2 ca = *reinterpret_cast<const double2 *>(cs + t * PQ_LD + 4 * tx);
            const double2 cb = *reinterpret_cast<const double2 *>(cs + t * PQ_LD + 4 * tx + 2);
            const double2 ma = *reinterpret_cast<const double2 *>(ms + t * PQ_LD + 4 * tx);
            const double2 mb = *reinterpret_cast<const double2 *>(ms + t * PQ_LD + 4 * tx + 2);
            const double qv[4] = {qa.x, qa.y, qb.x, qb.y}, cv[4] = {ca.x, ca.y, cb.x, cb.y},
                         mv[4] = {ma.x, ma.y, mb.x, mb.y};
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const double hi = dmul(qv[i], cv[j]);
                    const double lo = dmul(qv[i], mv[j]);
                    acc[i][j] = dadd(acc[i][j], hi > lo ? hi : lo);
                }
        }
    } else {
        for (int t = 0; t < D; t++) {
            const double2 qa = *reinterpret_cast<const double2 *>(qs + t * PQ_LD + 4 * ty);
            const double2 qb = *reinterpret_cast<const double2 *>(qs + t * PQ_LD + 4 * ty + 2);
            const double2 ca = *reinterpret_cast<const double2 *>(cs + t * PQ_LD + 4 * tx);
            const double2 cb = *reinterpret_cast<const double2 *>(cs + t * PQ_LD + 4 * tx + 2);
            const double qv[4] = {qa.x, qa.y, qb.x, qb.y}, cv[4] = {ca.x, ca.y, cb.x, cb.y};
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) acc[i][j] = __fma_rn(qv[i], cv[j], acc[i][j]);
        }
    }
    const double scale = 1.0 / sqrt((double)D);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int r = i0 + 4 * ty + i;
        if (r >= nb || r0 + r >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int b = b0 + 4 * tx + j;
            if (b < nkh) scores[((size_t)h * nb + r) * kk_cap + b] = dmul(acc[i][j], scale);
        }
    }
}

// Centroid scores, the same sums as pq_scores_kernel (elements in order, one
// fused multiply-add each), tiled for the FP64 pipe: a CTA computes 128 rows x
// 128 clusters, each thread 8 rows x 8 clusters, with the element axis staged
// in chunks of 32 through two shared-memory stages (the next chunk's global
// loads are in flight while the FMAs run on the current one).  Shared memory
// delivers 128 bytes per cycle whatever the broadcast, so the thread tile sets
// the ratio of shared-memory wavefronts to FMAs: (8 + 8) doubles read per 64
// FMAs.  One CTA per SM (232 registers a thread).  Needs q and the centroids
// 16-byte aligned (checked on the host; pq_scores_kernel otherwise).
constexpr int PQC_ROWS = 128, PQC_COLS = 128, PQC_KC = 32;
constexpr size_t PQC_SMEM = (size_t)2 * PQC_KC * (PQC_ROWS + PQC_COLS) * sizeof(double);

template <typename T> struct PqcRow;  // one thread's 16 consecutive query elements
template <> struct PqcRow<__nv_bfloat16> {
    uint4 a, b;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
        a = __ldg(reinterpret_cast<const uint4 *>(p));
        b = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ float get(int u) const {
        const uint4 &x = u < 8 ? a : b;
        const int v = u & 7;
        const uint32_t w = v < 2 ? x.x : (v < 4 ? x.y : (v < 6 ? x.z : x.w));
        return __uint_as_float((v & 1) ? (w & 0xFFFF0000u) : (w << 16));
    }
};
template <> struct PqcRow<float> {
    float4 x[4];
    __device__ __forceinline__ void load(const float *p) {
#pragma unroll
        for (int i = 0; i < 4; i++) x[i] = __ldg(reinterpret_cast<const float4 *>(p) + i);
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < 4; i++) x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __device__ __forceinline__ float get(int u) const {
        const float4 &v = x[u >> 2];
        const int c = u & 3;
        return c == 0 ? v.x : (c == 1 ? v.y : (c == 2 ? v.z : v.w));
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(256, 1) pq_scores_c_kernel(const T *__restrict__ q, int N, int r0, int nb,
                                                            const float *__restrict__ k_cent, int kk_cap,
                                                            const int32_t *__restrict__ nk, int kk_fixed,
                                                            int text_group, double *__restrict__ scores) {
    extern __shared__ double pqc[];
    // stage s: qs = pqc + s * KC * (ROWS + COLS), [KC][ROWS]; cs follows, [KC][COLS]
    const int h = blockIdx.z, tid = threadIdx.x;
    const int nkh = (nk ? min(max(nk[h], 0), kk_cap) : kk_fixed) - text_group;
    const int b0 = blockIdx.y * PQC_COLS, i0 = blockIdx.x * PQC_ROWS;
    if (b0 >= nkh) return;
    // staging roles: query row lr and centroid lc, 16 elements each from 16 lj
    const int lr = tid & 127, lj = tid >> 7;
    const int lc = tid & 127;
    const bool row_ok = i0 + lr < nb && r0 + i0 + lr < N;
    const bool cl_ok = b0 + lc < nkh;
    const T *qrow = q + ((size_t)h * N + (row_ok ? r0 + i0 + lr : 0)) * D + 16 * lj;
    const float *crow = k_cent + ((size_t)h * kk_cap + (cl_ok ? b0 + lc : 0)) * D + 16 * lj;
    PqcRow<T> qr;
    PqcRow<float> cr;
    auto fetch = [&](int t0) {
        if (row_ok) qr.load(qrow + t0); else qr.zero();
        if (cl_ok) cr.load(crow + t0); else cr.zero();
    };
    auto stash = [&](int s) {
        double *qs = pqc + (size_t)s * PQC_KC * (PQC_ROWS + PQC_COLS);
        double *cs = qs + PQC_KC * PQC_ROWS;
#pragma unroll
        for (int u = 0; u < 16; u++) qs[(16 * lj + u) * PQC_ROWS + lr] = (double)qr.get(u);
#pragma unroll
        for (int u = 0; u < 16; u++) cs[(16 * lj + u) * PQC_COLS + lc] = (double)cr.get(u);
    };
    // compute roles: warp w = row groups 4 (w >> 1) .. + 3, cluster groups 8 (w & 1) .. + 7;
    // thread: rows 8 ty .. 8 ty + 7, clusters tx + 16 j (j < 8: eight threads of
    // a quarter warp read eight consecutive doubles, no bank conflict)
    const int w = tid >> 5, l = tid & 31;
    const int ty = 4 * (w >> 1) + (l >> 3), tx = 8 * (w & 1) + (l & 7);
    double acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 8; j++) acc[i][j] = 0.0;
    fetch(0);
    stash(0);
    __syncthreads();
    constexpr int NCH = D / PQC_KC;
#pragma unroll 1
    for (int c = 0; c < NCH; c++) {
        if (c + 1 < NCH) fetch((c + 1) * PQC_KC);
        const double *qs = pqc + (size_t)(c & 1) * PQC_KC * (PQC_ROWS + PQC_COLS);
        const double *cs = qs + PQC_KC * PQC_ROWS;
#pragma unroll 4
        for (int t = 0; t < PQC_KC; t++) {
            double qv[8], cv[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const double2 x = *reinterpret_cast<const double2 *>(qs + t * PQC_ROWS + 8 * ty + 2 * i);
                qv[2 * i] = x.x;
                qv[2 * i + 1] = x.y;
            }
#pragma unroll
            for (int j = 0; j < 8; j++) cv[j] = cs[t * PQC_COLS + tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 8; i++)
#pragma unroll
                for (int j = 0; j < 8; j++) acc[i][j] = __fma_rn(qv[i], cv[j], acc[i][j]);
        }
        if (c + 1 < NCH) stash((c + 1) & 1);
        __syncthreads();
    }
    const double scale = 1.0 / sqrt((double)D);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int r = i0 + 8 * ty + i;
        if (r >= nb || r0 + r >= N) continue;
        double *srow = scores + ((size_t)h * nb + r) * kk_cap;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int b = b0 + tx + 16 * j;
            if (b < nkh) srow[b] = dmul(acc[i][j], scale);
        }
    }
}

// One warp per query row keeps the top_k non-empty clusters of largest score,
// ties to the lower id.  Up to 512 clusters: lane l holds clusters l + 32 i
// (i < 16) in registers and the warp runs a quickselect for the row's top_k-th
// cluster e* in the selection order (larger score, then lower id): a pivot is
// drawn from the clusters still in question, every lane counts its candidates
// at or before it, and the warp-wide count places e* before, at or after the
// pivot.  The row keeps e* and every cluster before it; bit word i of the set
// is a ballot of lane bits i.  Rotating the pivot's lane and register with the
// round keeps rows whose scores follow the cluster order from splitting
// unevenly (about ten rounds for 500 clusters).  More clusters: top_k rounds of a
// warp-wide argmax over the row's scores staged in shared memory, clusters
// already taken skipped.  Up to four warps per block, fewer when kk_cap is
// large; each warp takes rows in turn and adds its rows' pairs to the head's
// total once.
// PQ_REG_CLUSTERS: most key clusters a row holds in its lanes' registers (16 per lane)
constexpr int PQ_WARPS = 4, PQ_REG_CLUSTERS = 512;
// bytes of a warp's score region
__host__ __device__ constexpr size_t pq_topk_region(int kk_cap) { return (size_t)kk_cap * 8; }
// blocks per head of the top-k launch
__host__ __device__ constexpr int pq_topk_blocks(int H) { return 8192 / H > 64 ? 8192 / H : 64; }
__global__ void __launch_bounds__(PQ_WARPS * 32, 4) pq_topk_kernel(const double *__restrict__ scores, int N, int r0,
                                                               int nb, const int32_t *__restrict__ k_count, int kk_cap,
                                                               const int32_t *__restrict__ nk, int kk_fixed,
                                                               int text_group, const uint8_t *__restrict__ dense,
                                                               int top_k, int W, uint32_t *__restrict__ bits,
                                                               unsigned long long *__restrict__ head_pairs) {
    extern __shared__ unsigned char pqt[];
    const unsigned full = 0xffffffffu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const size_t region = pq_topk_region(kk_cap);
    double *sc = reinterpret_cast<double *>(pqt + (size_t)warp * region);  // [warps][region]
    uint32_t *bw = reinterpret_cast<uint32_t *>(pqt + (size_t)nw * region) + (size_t)warp * W;  // [warps][W]
    const int h = blockIdx.y;
    const int nkh_all = nk ? min(max(nk[h], 0), kk_cap) : kk_fixed;
    const int nkh = nkh_all - text_group;
    const int32_t *kc = k_count + (size_t)h * kk_cap;
    const bool dn = dense && dense[h];
    const bool regs = nkh <= PQ_REG_CLUSTERS;
    // register path: the lane's clusters that hold keys
    uint32_t km = 0u;
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const int b = lane + 32 * i;
        if (regs && b < nkh && kc[b] > 0) km |= 1u << i;
    }
    const unsigned long long text_pairs = text_group ? (unsigned long long)kc[nkh] : 0ull;
    unsigned long long pairs = 0ull;  // lane 0: this warp's rows
    for (int r = blockIdx.x * nw + warp; r < nb && r0 + r < N; r += gridDim.x * nw) {
        uint32_t *out = bits + ((size_t)h * N + r0 + r) * W;
        const double *srow = scores + ((size_t)h * nb + r) * kk_cap;
        if (dn) {
            for (int w = lane; w < W; w += 32) out[w] = 0u;
        } else if (regs) {
            double v[16];
            uint32_t vm = 0u;  // bit i: cluster lane + 32 i holds keys and its score is a number
#pragma unroll
            for (int i = 0; i < 16; i++) {
                v[i] = 0.0;
                if ((km >> i) & 1u) {
                    const double sv = srow[lane + 32 * i];
                    v[i] = sv;
                    if (sv == sv) vm |= 1u << i;
                }
            }
            const int tot = (int)__reduce_add_sync(full, (unsigned)__popc(vm));
            uint32_t sel = vm;
            if (tot > top_k) {
                // C: candidates for e*; S: clusters known to be before e*, base of them
                uint32_t C = vm, S = 0u;
                int base = 0;
                sel = 0u;
                for (int it = 0; it < PQ_REG_CLUSTERS; it++) {  // each round drops at least the pivot from C
                    const uint32_t lanes = __ballot_sync(full, C != 0u);
                    const int rot = (it * 13 + r * 7) & 31;
                    const uint32_t rl = rot ? ((lanes >> rot) | (lanes << (32 - rot))) : lanes;
                    const int lead = (__ffs(rl) - 1 + rot) & 31;
                    const int es = (it * 5 + r) & 15;
                    const uint32_t rc = ((C | (C << 16)) >> es) & 0xFFFFu;
                    const int e = (__ffs(rc) - 1 + es) & 15;
                    double pv = 0.0;
#pragma unroll
                    for (int i = 0; i < 16; i++) pv = i == e ? v[i] : pv;
                    pv = __shfl_sync(full, pv, lead);
                    const int pid = __shfl_sync(full, lane + 32 * e, lead);
                    uint32_t le = 0u;  // candidates at or before the pivot
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const bool bf = v[i] > pv || (v[i] == pv && lane + 32 * i <= pid);
                        le |= (uint32_t)bf << i;
                    }
                    le &= C;
                    const int cnt = (int)__reduce_add_sync(full, (unsigned)__popc(le));
                    if (base + cnt == top_k) {
                        sel = S | le;
                        break;
                    }
                    if (base + cnt > top_k) {
                        C = le;
                        if (lane == lead) C &= ~(1u << e);
                    } else {
                        S |= le;
                        base += cnt;
                        C &= ~le;
                    }
                }
            }
            unsigned rp = 0u;
            uint32_t myw = 0u;
#pragma unroll
            for (int i = 0; i < 16; i++) {
                if ((sel >> i) & 1u) rp += (unsigned)kc[lane + 32 * i];
                const uint32_t wd = __ballot_sync(full, (sel >> i) & 1u);
                if (lane == i) myw = wd;
            }
            rp = __reduce_add_sync(full, rp);
            for (int w = lane; w < W; w += 32) {
                uint32_t x = w < 16 ? myw : 0u;
                if (text_group && w == (nkh >> 5)) x |= 1u << (nkh & 31);  // the text-key group, always kept
                out[w] = x;
            }
            if (lane == 0) pairs += (unsigned long long)rp + text_pairs;
        } else {
            for (int w = lane; w < W; w += 32) bw[w] = 0u;
            // empty clusters and (below) taken ones hold NaN, which no comparison accepts
            const double qnan = __longlong_as_double(0x7ff8000000000000ll);
            for (int b = lane; b < nkh; b += 32) sc[b] = kc[b] > 0 ? srow[b] : qnan;
            __syncwarp();
            for (int round = 0; round < top_k; round++) {
                double best = -INFINITY;
                int bb = 0x7fffffff;
                for (int b = lane; b < nkh; b += 32) {
                    const double x = sc[b];
                    if (x > best || (x == best && b < bb)) {
                        best = x;
                        bb = b;
                    }
                }
                for (int o = 16; o > 0; o >>= 1) {
                    const double ob = __shfl_xor_sync(full, best, o);
                    const int oj = __shfl_xor_sync(full, bb, o);
                    if (ob > best || (ob == best && oj < bb)) {
                        best = ob;
                        bb = oj;
                    }
                }
                if (bb == 0x7fffffff) break;  // no non-empty cluster left
                if (lane == 0) {
                    sc[bb] = qnan;
                    bw[bb >> 5] |= 1u << (bb & 31);
                    pairs += (unsigned long long)kc[bb];
                }
                __syncwarp();
            }
            if (text_group && lane == 0) {
                const int tg = nkh;  // the text-key group's id
                bw[tg >> 5] |= 1u << (tg & 31);
                pairs += text_pairs;
            }
            __syncwarp();
            for (int w = lane; w < W; w += 32) out[w] = bw[w];
            __syncwarp();  // the next row's staging after every lane's reads
        }
    }
    if (lane == 0 && pairs) atomicAdd(head_pairs + h, pairs);
}

// Union of the rows' sets of query cluster a (members listed by the query
// cluster sort), as an ascending list.  One CTA per (cluster, head).
__global__ void pq_union_kernel(int N, const uint32_t *__restrict__ bits, int W, const int32_t *__restrict__ qperm,
                                const int32_t *__restrict__ qoff, int kq_cap, const int32_t *__restrict__ nq,
                                int kq_fixed, const uint8_t *__restrict__ dense, int kk_cap,
                                int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_cnt) {
    extern __shared__ uint32_t uw[];  // [W]
    __shared__ int wsum[32];
    const int h = blockIdx.y, a = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int nqh = nq ? min(max(nq[h], 0), kq_cap) : kq_fixed;
    const int32_t *o = qoff + (size_t)h * (kq_cap + 1);
    if (a >= nqh || (dense && dense[h]) || o[a + 1] <= o[a]) {
        if (tid == 0) sel_cnt[(size_t)h * kq_cap + a] = 0;
        return;
    }
    for (int w = tid; w < W; w += nt) {
        uint32_t x = 0u;
        for (int p = o[a]; p < o[a + 1]; p++) x |= bits[((size_t)h * N + qperm[(size_t)h * N + p]) * W + w];
        uw[w] = x;
    }
    __syncthreads();
    // ascending list of the set bits (block-wide exclusive scan of the word counts)
    int base = 0;
    int32_t *out = sel_idx + ((size_t)h * kq_cap + a) * kk_cap;
    for (int w0 = 0; w0 < W; w0 += nt) {
        const int w = w0 + tid;
        const int c = w < W ? __popc(uw[w]) : 0;
        int x = c;
        const int lane = tid & 31, wi = tid >> 5;
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) wsum[wi] = x;
        __syncthreads();
        int before = base + x - c;
        for (int u = 0; u < wi; u++) before += wsum[u];
        if (w < W) {
            uint32_t m = uw[w];
            while (m) {
                const int b = w * 32 + __ffs(m) - 1;
                m &= m - 1u;
                if (b < kk_cap) out[before++] = b;
            }
        }
        __syncthreads();
        for (int u = 0; u < nt / 32; u++) base += wsum[u];
        __syncthreads();
    }
    if (tid == 0) sel_cnt[(size_t)h * kq_cap + a] = min(base, kk_cap);
}

// One key run per selected non-empty cluster, ascending (the runs are not
// merged); info = {runs, chunks of chunk_rows rows}.  One thread per (head,
// query cluster) walks its list.
__global__ void key_runs_single_kernel(int H, int kq_cap, int kk_cap, const int32_t *__restrict__ koff,
                                       const int32_t *__restrict__ sel_idx, const int32_t *__restrict__ sel_cnt,
                                       int chunk_rows, int2 *__restrict__ runs, int2 *__restrict__ info) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= H * kq_cap) return;
    const int h = g / kq_cap, a = g - h * kq_cap;
    const int32_t *ko = koff + (size_t)h * (kk_cap + 1);
    const int32_t *sl = sel_idx + ((size_t)h * kq_cap + a) * kk_cap;
    const int n = min(max(sel_cnt[(size_t)h * kq_cap + a], 0), kk_cap);
    int2 *out = runs + ((size_t)h * kq_cap + a) * kk_cap;
    int nr = 0;
    unsigned long long slot_rows = 0ull;
    for (int c = 0; c < n; c++) {
        const int b = sl[c];
        if (b < 0 || b >= kk_cap) continue;
        const int r0 = ko[b], r1 = ko[b + 1];
        if (r1 <= r0) continue;
        out[nr++] = make_int2(r0, r1);
        slot_rows += (unsigned long long)((r1 - r0 + 7) & ~7);
    }
    info[(size_t)h * kq_cap + a] =
        make_int2(nr, (int)((slot_rows + (unsigned long long)chunk_rows - 1) / (unsigned long long)chunk_rows));
}

// Per row of query cluster a and chunk j of its key stream: bit g set when
// the row's own set holds the cluster of 8-key group g.  The groups' clusters
// come from the runs' slot layout (every run's rows from its slot start, its
// last group padded), as the key stream packs them.  One run per selected
// cluster, so at most kk_cap runs (their slot starts take kk_cap rounded up to
// even ints of shared memory, so that the group table behind them is 8-byte
// aligned).
__host__ __device__ constexpr int pq_run_slots(int kk_cap) { return (kk_cap + 1) & ~1; }
__global__ void pq_rowmask_kernel(int N, int kq_cap, int kk_cap, int max_chunks, const int32_t *__restrict__ koff,
                                  const int2 *__restrict__ runs, const int2 *__restrict__ info,
                                  const int32_t *__restrict__ qperm, const int32_t *__restrict__ qoff,
                                  const uint32_t *__restrict__ bits, int W, int rows_pass,
                                  uint16_t *__restrict__ rowmask) {
    extern __shared__ int pqr[];
    int *s_start = pqr;                  // [nr] slot start of each run
    int *gcl = pqr + pq_run_slots(kk_cap);  // [nch * 16] cluster of each group (-1: padding)
    __shared__ int wsum[32];
    const int h = blockIdx.y, a = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const size_t qa = (size_t)h * kq_cap + a;
    const int2 inf = info[qa];
    const int nr = min(inf.x, kk_cap), nch = min(inf.y, max_chunks);
    const int32_t *o = qoff + (size_t)h * (kq_cap + 1);
    if (nch <= 0 || o[a + 1] <= o[a]) return;
    const int2 *rr = runs + qa * kk_cap;
    const int32_t *ko = koff + (size_t)h * (kk_cap + 1);
    int carry = 0;
    for (int b0 = 0; b0 < nr; b0 += nt) {
        const int r = b0 + tid;
        int len = 0;
        if (r < nr) {
            const int2 v = rr[r];
            len = (v.y - v.x + 7) & ~7;
        }
        int x = len;
        const int lane = tid & 31, w = tid >> 5;
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) wsum[w] = x;
        __syncthreads();
        int before = carry + x - len;
        for (int u = 0; u < w; u++) before += wsum[u];
        if (r < nr) s_start[r] = before;
        __syncthreads();
        for (int u = 0; u < nt / 32; u++) carry += wsum[u];
        __syncthreads();
    }
    for (int gi = tid; gi < nch * 16; gi += nt) {
        const int pos = gi * 8;
        int lo = 0, hi = nr - 1, r = -1;
        while (lo <= hi) {
            const int mid = (lo + hi) >> 1;
            if (s_start[mid] <= pos) { r = mid; lo = mid + 1; }
            else hi = mid - 1;
        }
        int cl = -1;
        if (r >= 0) {
            const int2 v = rr[r];
            const int key = v.x + (pos - s_start[r]);
            if (key < v.y) {
                // the cluster whose rows hold `key`: last b with koff[b] <= key
                int l2 = 0, h2 = kk_cap - 1, b = 0;
                while (l2 <= h2) {
                    const int mid = (l2 + h2) >> 1;
                    if (ko[mid] <= key) { b = mid; l2 = mid + 1; }
                    else h2 = mid - 1;
                }
                cl = b;
            }
        }
        gcl[gi] = cl;
    }
    __syncthreads();
    // compress each chunk's 16 groups, in place, into (cluster << 16 | groups)
    // entries, one per run of groups of one cluster (usually one or two; the
    // first two always written, zero entries select nothing)
    int *nent = gcl + max_chunks * 16;  // [nch]
    for (int j = tid; j < nch; j += nt) {
        int ne = 0, cur = -1;
        uint32_t gm = 0u;
        for (int g = 0; g < 16; g++) {
            const int cl = gcl[j * 16 + g];
            if (cl != cur) {
                if (cur >= 0) gcl[j * 16 + ne++] = (int)(((uint32_t)cur << 16) | gm);
                cur = cl;
                gm = 0u;
            }
            if (cl >= 0) gm |= 1u << g;
        }
        if (cur >= 0) gcl[j * 16 + ne++] = (int)(((uint32_t)cur << 16) | gm);
        nent[j] = ne;
        for (int e = ne; e < 2; e++) gcl[j * 16 + e] = 0;
    }
    // rows in passes of rows_pass: their bit sets copied row by row (coalesced)
    // into shared memory at an odd stride, so that the per-chunk tests read
    // 32 different rows' words without bank conflicts
    uint32_t *sb = reinterpret_cast<uint32_t *>(nent + max_chunks);  // [rows_pass][W + 1]
    const int ld = W + 1;
    for (int p0 = o[a]; p0 < o[a + 1]; p0 += rows_pass) {
        const int np = min(rows_pass, o[a + 1] - p0);
        __syncthreads();  // the previous pass's reads of sb (and, first, the entry table)
        for (int g = tid; g < np * W; g += nt) {
            const int rr = g / W, w = g - rr * W;
            sb[rr * ld + w] = bits[((size_t)h * N + qperm[(size_t)h * N + p0 + rr]) * W + w];
        }
        __syncthreads();
        for (int rr = tid; rr < np; rr += nt) {
            const uint32_t *rb = sb + rr * ld;
            uint16_t *dst = rowmask + (size_t)h * max_chunks * N + p0 + rr;
            // entry v keeps its groups when the row's set holds cluster v >> 16
            auto take = [&](uint32_t v) { return ((rb[v >> 21] >> ((v >> 16) & 31u)) & 1u) ? (v & 0xFFFFu) : 0u; };
            for (int j = 0; j < nch; j++, dst += N) {
                const int ne = nent[j];
                const int2 v2 = *reinterpret_cast<const int2 *>(gcl + j * 16);
                uint32_t m = take((uint32_t)v2.x) | take((uint32_t)v2.y);
                for (int e = 2; e < ne; e++) m |= take((uint32_t)gcl[j * 16 + e]);
                *dst = (uint16_t)m;
            }
        }
    }
}

// ------------------------------------------------------------------ launchers
size_t pq_score_batch_rows(int H, int N, int kk_cap) {
    // scores of a batch of rows for all heads in about 1 GiB
    size_t per_row = (size_t)H * kk_cap * sizeof(double);
    size_t b = ((size_t)1 << 30) / (per_row ? per_row : 1);
    b = b < 1024 ? 1024 : b;
    return b < (size_t)N ? b : (size_t)N;
}

int k_select_rows(const void *q, int dtype, int H, int N, int D, const float *k_cent, const float *k_max,
                  const float *k_min, const int32_t *k_count, int kk_cap, const int32_t *nk, int kk_fixed,
                  int text_group, const uint8_t *dense, int score_mode, int top_k, uint32_t *bits, int W,
                  double *scores, int batch, unsigned long long *head_pairs, cudaStream_t st) {
    const int nkmax = nk ? kk_cap : kk_fixed;
    const size_t smem_s = (size_t)(score_mode == 1 ? 3 : 2) * D * PQ_LD * sizeof(double);
    const size_t per_warp = pq_topk_region(kk_cap) + (size_t)W * sizeof(uint32_t);
    int nwarps = (int)((size_t)(200 * 1024) / per_warp);
    nwarps = nwarps < 1 ? 1 : (nwarps > PQ_WARPS ? PQ_WARPS : nwarps);
    const size_t smem_t = (size_t)nwarps * per_warp;
    cudaMemsetAsync(head_pairs, 0, sizeof(unsigned long long) * H, st);
    // centroid scores from 16-byte aligned operands: the chunked kernel
    const bool tiled = score_mode == 0 && ((uintptr_t)q & 15u) == 0 && ((uintptr_t)k_cent & 15u) == 0;
    for (int r0 = 0; r0 < N; r0 += batch) {
        const int nb = N - r0 < batch ? N - r0 : batch;
        dim3 g1((nb + PQ_ROWS - 1) / PQ_ROWS, (nkmax + PQ_COLS - 1) / PQ_COLS, H);
#define AC_PQS(T, DD)                                                                                              \
    do {                                                                                                           \
        if (smem_s > 48 * 1024)                                                                                    \
            cudaFuncSetAttribute(pq_scores_kernel<T, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s); \
        pq_scores_kernel<T, DD><<<g1, 256, smem_s, st>>>(static_cast<const T *>(q), N, r0, nb, k_cent, k_max, k_min, \
                                                         kk_cap, nk, kk_fixed, text_group, score_mode, scores);     \
    } while (0)
#define AC_PQC(T, DD)                                                                                              \
    do {                                                                                                           \
        cudaFuncSetAttribute(pq_scores_c_kernel<T, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PQC_SMEM); \
        pq_scores_c_kernel<T, DD><<<gc, 256, PQC_SMEM, st>>>(static_cast<const T *>(q), N, r0, nb, k_cent, kk_cap,  \
                                                           nk, kk_fixed, text_group, scores);                      \
    } while (0)
        if (tiled) {
            dim3 gc((nb + PQC_ROWS - 1) / PQC_ROWS, (nkmax + PQC_COLS - 1) / PQC_COLS, H);
            if (dtype == DT_BF16) {
                if (D == 64) AC_PQC(__nv_bfloat16, 64);
                else AC_PQC(__nv_bfloat16, 128);
            } else {
                if (D == 64) AC_PQC(float, 64);
                else AC_PQC(float, 128);
            }
        } else if (dtype == DT_BF16) {
            if (D == 64) AC_PQS(__nv_bfloat16, 64);
            else AC_PQS(__nv_bfloat16, 128);
        } else {
            if (D == 64) AC_PQS(float, 64);
            else AC_PQS(float, 128);
        }
#undef AC_PQS
#undef AC_PQC
        note_launch();
        if (smem_t > 48 * 1024)
            cudaFuncSetAttribute(pq_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_t);
        const int need = (nb + nwarps - 1) / nwarps;
        dim3 g2(need < pq_topk_blocks(H) ? need : pq_topk_blocks(H), H);
        pq_topk_kernel<<<g2, nwarps * 32, smem_t, st>>>(scores, N, r0, nb, k_count, kk_cap, nk, kk_fixed,
                                                          text_group, dense, top_k, W, bits, head_pairs);
        note_launch();
    }
    return 0;
}

void k_select_union(int H, int N, const uint32_t *bits, int W, const int32_t *qperm, const int32_t *qoff, int kq_cap,
                    const int32_t *nq, int kq_fixed, const uint8_t *dense, int kk_cap, int32_t *sel_idx,
                    int32_t *sel_cnt, cudaStream_t st) {
    const size_t smem = (size_t)W * sizeof(uint32_t);
    if (smem > 48 * 1024) cudaFuncSetAttribute(pq_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    pq_union_kernel<<<dim3(kq_cap, H), 256, smem, st>>>(N, bits, W, qperm, qoff, kq_cap, nq, kq_fixed, dense, kk_cap,
                                                        sel_idx, sel_cnt);
    note_launch();
}

void k_key_runs_single(int H, int kq_cap, int kk_cap, const int32_t *koff, const int32_t *sel_idx,
                       const int32_t *sel_cnt, int chunk_rows, int2 *runs, int2 *info, cudaStream_t st) {
    const int n = H * kq_cap;
    key_runs_single_kernel<<<(n + 127) / 128, 128, 0, st>>>(H, kq_cap, kk_cap, koff, sel_idx, sel_cnt, chunk_rows,
                                                            runs, info);
    note_launch();
}

int k_rowmask(int H, int N, int kq_cap, int kk_cap, int max_chunks, const int32_t *koff, const int2 *runs,
              const int2 *info, const int32_t *qperm, const int32_t *qoff, const uint32_t *bits, int W,
              uint16_t *rowmask, cudaStream_t st) {
    const size_t base = (size_t)(pq_run_slots(kk_cap) + (size_t)max_chunks * 17) * sizeof(int);
    const size_t limit = 227 * 1024, per_row = (size_t)(W + 1) * sizeof(uint32_t);
    // rows per pass: the block's 256 threads, fewer when the bit sets are long
    const int rows_pass = base + 32 * per_row > limit ? 0 : (int)std::min<size_t>(256, (limit - base) / per_row / 32 * 32);
    if (rows_pass < 32) return -1;  // the group table of the longest key stream does not fit
    const size_t smem = base + (size_t)rows_pass * per_row;
    cudaFuncSetAttribute(pq_rowmask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    pq_rowmask_kernel<<<dim3(kq_cap, H), 256, smem, st>>>(N, kq_cap, kk_cap, max_chunks, koff, runs, info, qperm,
                                                          qoff, bits, W, rows_pass, rowmask);
    note_launch();
    return 0;
}

}  // namespace ac
