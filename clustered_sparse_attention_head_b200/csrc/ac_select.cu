// Critical-cluster selection (AdaCluster, Algorithm 3's select step): for a query
// cluster a, key cluster b is scored either by its centroid against a's
// centroid (the centroid-based significance estimate of §2.3) or by Quest's
// page bound (§3.2.3 eq. (1), in TensorQuest's form of eq. (2)).  Then either
// the top_k best-scored clusters are kept (Algorithm 3's argtopk), or, with
// scores weighted by b's size, the smallest set holding a top_p share of the
// estimated attention mass.
//
// One CTA per (query cluster, head).  Scores, weights and the running mass are
// double, evaluated in the order of a plain sequential loop (scores per b
// along d; the normaliser and the running mass by one thread in b order and
// in visiting order), so the kept set matches a CPU evaluation of the same
// loop except where two masses differ in the last bits of exp().
#include "ac_kernels.cuh"

namespace ac {

// Key centroids transposed per head, [kk_cap, D] -> [D, kk_cap], so that the
// selection's per-thread dot products read consecutive addresses across a warp.
__global__ void transpose_cent_kernel(const float *__restrict__ src, int rows, int D, float *__restrict__ dst) {
    __shared__ float tile[32][33];
    const int h = blockIdx.z;
    const float *s = src + (size_t)h * rows * D;
    float *d = dst + (size_t)h * rows * D;
    const int r0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < D) tile[i][threadIdx.x] = s[(size_t)r * D + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < rows && c < D) d[(size_t)c * rows + r] = tile[threadIdx.x][i];
    }
}

__global__ void select_kernel(int D, const float *__restrict__ q_cent, const float *__restrict__ q_mean_norm,
                              const int32_t *__restrict__ q_count, int kq_cap, const float *__restrict__ k_cent,
                              const int32_t *__restrict__ k_count, const float *__restrict__ k_max,
                              const float *__restrict__ k_min, int kk_cap, const int32_t *__restrict__ nq,
                              const int32_t *__restrict__ nk, int kq_fixed, int kk_fixed,
                              const uint8_t *__restrict__ dense, int score_mode, int top_k, double top_p, int n2,
                              int text_group, const float *__restrict__ k_cent_t, const float *__restrict__ k_min_t,
                              int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_cnt, int *status) {
    extern __shared__ __align__(16) unsigned char smraw[];
    double *sp = reinterpret_cast<double *>(smraw);          // [n2] p (sort key)
    int *sb = reinterpret_cast<int *>(sp + n2);             // [n2] b
    double *sw = reinterpret_cast<double *>(sb + n2);        // [kk_cap] weights
    int *skn = reinterpret_cast<int *>(sw + kk_cap);          // [kk_cap] key cluster sizes
    unsigned char *keep = reinterpret_cast<unsigned char *>(skn + kk_cap);  // [kk_cap]
    __shared__ double mu[128];
    __shared__ double qpos[128], qneg[128];
    __shared__ double red[32];
    __shared__ int ired[33];
    __shared__ double sW;

    const int h = blockIdx.y, a = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    // counts from caller memory are clamped to the capacities (ST_INVALID if not within)
    const int nqh = nq ? clamp_count(nq[h], kq_cap, a == 0 && tid == 0 ? status : nullptr) : kq_fixed;
    // with a text-key group, the last key id is that group: never scored, always kept
    const int nkh =
        nk ? clamp_count(nk[h] - text_group, kk_cap - text_group, a == 0 && tid == 0 ? status : nullptr)
           : kk_fixed - text_group;
    int32_t *out = sel_idx + ((size_t)h * kq_cap + a) * kk_cap;
    if (a >= kq_cap) return;
    if (a >= nqh || (dense && dense[h]) || q_count[(size_t)h * kq_cap + a] == 0) {
        if (tid == 0) sel_cnt[(size_t)h * kq_cap + a] = 0;
        return;
    }
    const float *kc = k_cent + (size_t)h * kk_cap * D;
    const float *kct = k_cent_t ? k_cent_t + (size_t)h * kk_cap * D : nullptr;  // [D, kk_cap]
    const int *kn = skn;
    for (int b = tid; b < kk_cap; b += nt) skn[b] = k_count[(size_t)h * kk_cap + b];
    const double rbar = (double)q_mean_norm[(size_t)h * kq_cap + a];
    for (int t = tid; t < D; t += nt) {
        mu[t] = (double)q_cent[((size_t)h * kq_cap + a) * D + t];
        // TensorQuest split of the representative query qbar = rbar * mu
        const double qb = dmul(rbar, mu[t]);
        qpos[t] = qb > 0.0 ? qb : 0.0;
        qneg[t] = qb < 0.0 ? qb : 0.0;
    }
    const double scale = 1.0 / sqrt((double)D);
    const float *kmx = k_max ? k_max + (size_t)h * kk_cap * D : nullptr;
    const float *kmn = k_min ? k_min + (size_t)h * kk_cap * D : nullptr;
    __syncthreads();

    // scores and their maximum over non-empty key clusters
    double m = -INFINITY;
    for (int b = tid; b < nkh; b += nt) {
        double s = -INFINITY;
        if (kn[b] > 0) {
            if (score_mode == 1) {
                // qbar+ . M_b + qbar- . m_b, summed per dimension: each term
                // equals max(qbar_t M_bt, qbar_t m_bt) of eq. (1) exactly
                double acc = 0.0;
                if (kct && k_min_t) {
                    // transposed bounds: a warp reads consecutive clusters
                    const float *Mt = kct, *mt = k_min_t + (size_t)h * kk_cap * D;
                    for (int t = 0; t < D; t++)
                        acc = dadd(acc, dadd(dmul(qpos[t], (double)Mt[(size_t)t * kk_cap + b]),
                                             dmul(qneg[t], (double)mt[(size_t)t * kk_cap + b])));
                } else {
                    const float *M = kmx + (size_t)b * D, *mn = kmn + (size_t)b * D;
                    for (int t = 0; t < D; t++)
                        acc = dadd(acc, dadd(dmul(qpos[t], (double)M[t]), dmul(qneg[t], (double)mn[t])));
                }
                s = dmul(acc, scale);
            } else {
                double dot = 0.0;
                if (kct) {
                    for (int t = 0; t < D; t++) dot = dadd(dot, dmul(mu[t], (double)kct[(size_t)t * kk_cap + b]));
                } else {
                    const float *c = kc + (size_t)b * D;
                    for (int t = 0; t < D; t++) dot = dadd(dot, dmul(mu[t], (double)c[t]));
                }
                s = dmul(dmul(rbar, dot), scale);
            }
            m = fmax(m, s);
        }
        sw[b] = s;
    }
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
        double mm = -INFINITY;
        for (int w = 0; w < nt / 32; w++) mm = fmax(mm, red[w]);
        red[0] = mm;
    }
    __syncthreads();
    m = red[0];
    if (top_k > 0) {
        // argtopk: sort by the score itself
        for (int i = tid; i < n2; i += nt) {
            const bool live = i < nkh && kn[i] > 0;
            sp[i] = live ? sw[i] : -INFINITY;
            sb[i] = live ? i : 0x7fffffff;
        }
    } else {
        for (int b = tid; b < nkh; b += nt) {
            if (kn[b] > 0) sw[b] = dmul((double)kn[b], exp(dsub(sw[b], m)));
        }
        __syncthreads();
        if (tid == 0) {
            double W = 0.0;
            for (int b = 0; b < nkh; b++)
                if (kn[b] > 0) W = dadd(W, sw[b]);
            sW = W;
        }
        __syncthreads();
        const double W = sW;
        for (int i = tid; i < n2; i += nt) {
            if (i < nkh && kn[i] > 0) {
                sp[i] = ddiv(sw[i], W);
                sb[i] = i;
            } else {
                sp[i] = -1.0;
                sb[i] = 0x7fffffff;
            }
        }
    }
    for (int b = tid; b < kk_cap; b += nt) keep[b] = 0;
    __syncthreads();
    // bitonic sort: p descending, then b ascending
    for (int k = 2; k <= n2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < n2; i += nt) {
                int l = i ^ j;
                if (l > i) {
                    double pi = sp[i], pl = sp[l];
                    int bi = sb[i], bl = sb[l];
                    bool i_first = (pi > pl) || (pi == pl && bi < bl);
                    bool up = ((i & k) == 0);
                    if (up ? !i_first : i_first) {
                        sp[i] = pl; sp[l] = pi;
                        sb[i] = bl; sb[l] = bi;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (tid == 0) {
        double cum = 0.0;
        for (int r = 0; r < n2; r++) {
            if (sb[r] == 0x7fffffff) break;
            if (top_k > 0 && r >= top_k) break;
            keep[sb[r]] = 1;
            if (top_k > 0) continue;
            cum = dadd(cum, sp[r]);
            if (top_p < 1.0 && cum >= top_p) break;
        }
    }
    __syncthreads();
    // compact kept ids in ascending order
    if (tid == 0) ired[32] = 0;
    __syncthreads();
    for (int b0 = 0; b0 < nkh; b0 += nt) {
        int b = b0 + tid;
        int f = (b < nkh) ? keep[b] : 0;
        unsigned bal = __ballot_sync(0xffffffffu, f);
        int lane = tid & 31, w = tid >> 5;
        if (lane == 0) ired[w] = __popc(bal);
        __syncthreads();
        int before = ired[32];
        for (int u = 0; u < w; u++) before += ired[u];
        if (f) out[before + __popc(bal & ((1u << lane) - 1u))] = b;
        __syncthreads();
        if (tid == 0) {
            int tot = 0;
            for (int u = 0; u < nt / 32; u++) tot += ired[u];
            ired[32] += tot;
        }
        __syncthreads();
    }
    if (tid == 0) {
        int n = ired[32];
        if (text_group) out[n++] = nkh;
        sel_cnt[(size_t)h * kq_cap + a] = n;
    }
}

void k_select(int H, int D, const float *q_cent, const float *q_mean_norm, const int32_t *q_count, int kq_cap,
              const float *k_cent, const int32_t *k_count, const float *k_max, const float *k_min, int kk_cap,
              const int32_t *nq, const int32_t *nk, int kq_fixed, int kk_fixed, const uint8_t *dense, int score_mode,
              int top_k, double top_p, int32_t *sel_idx, int32_t *sel_cnt, int *status, cudaStream_t st,
              int text_group, float *k_cent_t, float *k_min_t) {
    int n2 = 1;
    while (n2 < kk_cap) n2 <<= 1;
    size_t smem = (size_t)n2 * (sizeof(double) + sizeof(int)) + (size_t)kk_cap * (sizeof(double) + sizeof(int) + 1);
    const dim3 tg((kk_cap + 31) / 32, (D + 31) / 32, H), tb(32, 8);
    if (k_cent_t && score_mode == 0) {
        transpose_cent_kernel<<<tg, tb, 0, st>>>(k_cent, kk_cap, D, k_cent_t);
        note_launch();
        k_min_t = nullptr;
    } else if (k_cent_t && k_min_t && score_mode == 1) {
        // the Quest bounds, transposed the same way (k_cent_t holds M^T)
        transpose_cent_kernel<<<tg, tb, 0, st>>>(k_max, kk_cap, D, k_cent_t);
        transpose_cent_kernel<<<tg, tb, 0, st>>>(k_min, kk_cap, D, k_min_t);
        note_launch();
        note_launch();
    } else {
        k_cent_t = nullptr;
        k_min_t = nullptr;
    }
    // opt in whenever dynamic plus static shared memory may pass 48 KB (the
    // attribute belongs to the current device, so it is set on every call)
    if (smem > 32 * 1024) cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 g(kq_cap, H);
    select_kernel<<<g, 256, smem, st>>>(D, q_cent, q_mean_norm, q_count, kq_cap, k_cent, k_count, k_max, k_min,
                                        kk_cap, nq, nk, kq_fixed, kk_fixed, dense, score_mode, top_k, top_p, n2,
                                        text_group, k_cent_t, k_min_t, sel_idx, sel_cnt, status);
    note_launch();
}

// Quest page bounds: one CTA per (cluster, head), one thread per dimension,
// walking the cluster's members in the cluster-sorted order (coalesced rows).
template <typename T>
__global__ void cluster_bounds_kernel(const T *__restrict__ x, int N, int D, const int32_t *__restrict__ perm,
                                      const int32_t *__restrict__ off, int cap, float *__restrict__ xmax,
                                      float *__restrict__ xmin) {
    const int h = blockIdx.y, b = blockIdx.x;
    const int32_t *o = off + (size_t)h * (cap + 1);
    const int i0 = o[b], i1 = o[b + 1];
    for (int t = threadIdx.x; t < D; t += blockDim.x) {
        float mx = 0.f, mn = 0.f;
        for (int i = i0; i < i1; i++) {
            const float v = to_f(x[((size_t)h * N + perm[(size_t)h * N + i]) * D + t]);
            mx = i == i0 ? v : fmaxf(mx, v);
            mn = i == i0 ? v : fminf(mn, v);
        }
        xmax[((size_t)h * cap + b) * D + t] = mx;
        xmin[((size_t)h * cap + b) * D + t] = mn;
    }
}

void k_cluster_bounds(const void *x, int dtype, int H, int N, int D, const int32_t *perm, const int32_t *off,
                      int cap, float *xmax, float *xmin, cudaStream_t st) {
    dim3 g(cap, H);
    if (dtype == DT_BF16)
        cluster_bounds_kernel<__nv_bfloat16><<<g, D, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), N, D, perm, off,
                                                             cap, xmax, xmin);
    else
        cluster_bounds_kernel<float><<<g, D, 0, st>>>(static_cast<const float *>(x), N, D, perm, off, cap, xmax, xmin);
    note_launch();
}

}  // namespace ac
