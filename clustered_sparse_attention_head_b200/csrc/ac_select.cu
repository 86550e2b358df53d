// Critical-cluster selection (AdaCluster, Algorithm 3 lines 6-7, with the
// centroid-based significance estimate of §2.3): for a query cluster a, key
// cluster b is scored by its centroid against a's centroid, weighted by b's
// size, and the smallest set of key clusters holding a top_p share of the
// estimated attention mass is kept.
//
// One CTA per (query cluster, head).  Scores, weights and the running mass are
// double, evaluated in the order of a plain sequential loop (scores per b
// along d; the normaliser and the running mass by one thread in b order and
// in visiting order), so the kept set matches a CPU evaluation of the same
// loop except where two masses differ in the last bits of exp().
#include "ac_kernels.cuh"

namespace ac {

__global__ void select_kernel(int D, const float *__restrict__ q_cent, const float *__restrict__ q_mean_norm,
                              const int32_t *__restrict__ q_count, int kq_cap, const float *__restrict__ k_cent,
                              const int32_t *__restrict__ k_count, int kk_cap, const int32_t *__restrict__ nq,
                              const int32_t *__restrict__ nk, int kq_fixed, int kk_fixed,
                              const uint8_t *__restrict__ dense, double top_p, int n2,
                              int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_cnt) {
    extern __shared__ __align__(16) unsigned char smraw[];
    double *sp = reinterpret_cast<double *>(smraw);          // [n2] p (sort key)
    int *sb = reinterpret_cast<int *>(sp + n2);             // [n2] b
    double *sw = reinterpret_cast<double *>(sb + n2);        // [kk_cap] weights
    unsigned char *keep = reinterpret_cast<unsigned char *>(sw + kk_cap);  // [kk_cap]
    __shared__ double mu[128];
    __shared__ double red[32];
    __shared__ int ired[33];
    __shared__ double sW;

    const int h = blockIdx.y, a = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int nqh = nq ? nq[h] : kq_fixed;
    const int nkh = nk ? nk[h] : kk_fixed;
    int32_t *out = sel_idx + ((size_t)h * kq_cap + a) * kk_cap;
    if (a >= kq_cap) return;
    if (a >= nqh || (dense && dense[h]) || q_count[(size_t)h * kq_cap + a] == 0) {
        if (tid == 0) sel_cnt[(size_t)h * kq_cap + a] = 0;
        return;
    }
    const float *kc = k_cent + (size_t)h * kk_cap * D;
    const int32_t *kn = k_count + (size_t)h * kk_cap;
    for (int t = tid; t < D; t += nt) mu[t] = (double)q_cent[((size_t)h * kq_cap + a) * D + t];
    const double rbar = (double)q_mean_norm[(size_t)h * kq_cap + a];
    const double scale = 1.0 / sqrt((double)D);
    __syncthreads();

    // scores and their maximum over non-empty key clusters
    double m = -INFINITY;
    for (int b = tid; b < nkh; b += nt) {
        double s = -INFINITY;
        if (kn[b] > 0) {
            const float *c = kc + (size_t)b * D;
            double dot = 0.0;
            for (int t = 0; t < D; t++) dot = dadd(dot, dmul(mu[t], (double)c[t]));
            s = dmul(dmul(rbar, dot), scale);
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
            keep[sb[r]] = 1;
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
    if (tid == 0) sel_cnt[(size_t)h * kq_cap + a] = ired[32];
}

void k_select(int H, int D, const float *q_cent, const float *q_mean_norm, const int32_t *q_count, int kq_cap,
              const float *k_cent, const int32_t *k_count, int kk_cap, const int32_t *nq, const int32_t *nk,
              int kq_fixed, int kk_fixed, const uint8_t *dense, double top_p, int32_t *sel_idx, int32_t *sel_cnt,
              cudaStream_t st) {
    int n2 = 1;
    while (n2 < kk_cap) n2 <<= 1;
    size_t smem = (size_t)n2 * (sizeof(double) + sizeof(int)) + (size_t)kk_cap * (sizeof(double) + 1);
    static size_t smem_set = 0;
    if (smem > 48 * 1024 && smem > smem_set) {
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        smem_set = smem;
    }
    dim3 g(kq_cap, H);
    select_kernel<<<g, 256, smem, st>>>(D, q_cent, q_mean_norm, q_count, kq_cap, k_cent, k_count, kk_cap, nq, nk,
                                        kq_fixed, kk_fixed, dense, top_p, n2, sel_idx, sel_cnt); note_launch();
}

}  // namespace ac
