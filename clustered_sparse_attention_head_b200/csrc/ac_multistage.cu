// Device-side control of Algorithm 1 (MultiStageClustering, AdaCluster §3.2.2):
// per-head stage decisions, the tau rules of the first stage, and the removal
// of tokens within tau of their centre from the remaining set U.
//
// Readings of the algorithm (the paper leaves these open):
//  - U starts as all tokens; stage t clusters U into m_t clusters with
//    m_0 = m0 and m_t = min(|U|, ceil(m0 |U| / N)) for t >= 1.  N is the
//    number of tokens clustered (nrows, the first nrows of each head's N).
//  - |C| >= N_max is tested before a stage; then F is set and the loop stops.
//  - A token of U leaves U when its distance to its centre is < tau.
//  - tau (MEAN_X / MEDIAN_RADIUS_X) is fixed from the first stage.
#include "ac_kernels.cuh"
#include "ac_multistage.cuh"

namespace ac {

// Both U buffers start as the identity, so every entry is a valid token id
// (entries past |U| are never used as members, but row gathers read them).
__global__ void ms_init_kernel(int H, int N, int nrows, MsHead *__restrict__ st, int32_t *__restrict__ U,
                               int32_t *__restrict__ U2) {
    int h = blockIdx.y;
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < N) {
        U[(size_t)h * N + i] = i;
        U2[(size_t)h * N + i] = i;
    }
    if (i == 0) {
        MsHead s;
        s.nc = 0;
        s.nu = nrows;
        s.stage = 0;
        s.flag = 0;
        s.mt = 0;
        s.done = 0;
        s.same = 0;
        s.rep_src = 0;
        s.rep_n = 0;
        s.pad = 0;
        s.tau = 0.0;
        st[h] = s;
    }
}

// Decide the next stage of every head; writes the pass descriptors and a
// summary {active heads, max |U|, max m_t, max |C|, capacity error, -, -,
// heads that repeat} for the host.
//
// A stage that removed no token is a fixed point: the next stage has the same
// U (same order), hence the same m_t and the same starting rows, runs the same
// k-means and removes nothing again, so every stage until |C| >= N_max
// repeats it and F is set.  The head then skips them: its centres are copied
// forward (k_ms_repeat), which gives what running them gives, bit for bit.
__global__ void ms_control_kernel(int H, int N, int m0, int nmax, int cap, MsHead *__restrict__ st,
                                  HeadSeg *__restrict__ seg, int32_t *__restrict__ info, int *status) {
    __shared__ int act, mnu, mmt, mnc, err, nrep;
    if (threadIdx.x == 0) { act = 0; mnu = 0; mmt = 0; mnc = 0; err = 0; nrep = 0; }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        MsHead s = st[h];
        HeadSeg g;
        g.nrows = 0;
        g.k = 0;
        g.cent_off = s.nc;
        g.pad = 0;
        if (!s.done) {
            if (s.nu <= 0) {
                s.done = 1;
            } else if (s.nc >= nmax) {
                s.flag = 1;
                s.done = 1;
            } else if (s.same && s.stage >= 1) {
                const int m = s.mt;  // the repeated stage's m_t (|U| is unchanged)
                const int r = (nmax - s.nc + m - 1) / m;
                if (s.nc + r * m > cap) {
                    atomicExch(&err, 1);
                    set_status(status, ST_CAPACITY);
                    s.done = 1;
                } else {
                    s.rep_src = s.nc - m;
                    s.rep_n = r;
                    s.nc += r * m;
                    s.stage += r;
                    s.flag = 1;
                    s.done = 1;
                    atomicAdd(&nrep, 1);
                }
            } else {
                int mt;
                if (s.stage == 0) mt = m0;
                else {
                    long long num = (long long)m0 * s.nu;
                    long long c = (num + N - 1) / N;
                    mt = (int)(c < s.nu ? c : s.nu);
                }
                if (mt > s.nu) mt = s.nu;
                if (s.nc + mt > cap) {
                    atomicExch(&err, 1);
                    set_status(status, ST_CAPACITY);
                    s.done = 1;
                } else {
                    s.mt = mt;
                    g.nrows = s.nu;
                    g.k = mt;
                    atomicAdd(&act, 1);
                    atomicMax(&mnu, s.nu);
                    atomicMax(&mmt, mt);
                }
            }
        }
        atomicMax(&mnc, s.nc + (g.nrows > 0 ? s.mt : 0));
        st[h] = s;
        seg[h] = g;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        info[0] = act;
        info[1] = mnu;
        info[2] = mmt;
        info[3] = mnc;
        info[4] = err;
        info[7] = nrep;
    }
}

__global__ void ms_repeat_kernel(int D, MsHead *__restrict__ st, float *__restrict__ cent, int cap) {
    const int h = blockIdx.x;
    const MsHead s = st[h];
    if (s.rep_n <= 0) return;
    const int m = s.mt;
    const float *src = cent + ((size_t)h * cap + s.rep_src) * D;
    for (int e = threadIdx.x; e < s.rep_n * m * D; e += blockDim.x) {
        const int i = e / (m * D), r = e - i * (m * D);
        cent[((size_t)h * cap + s.rep_src + (size_t)(i + 1) * m) * D + r] = src[r];
    }
    __syncthreads();
    if (threadIdx.x == 0) st[h].rep_n = 0;
}

// tau of the first stage (one CTA per head; positions = tokens at stage 0).
//  ABS: tau = x.
//  MEAN_X: x * (sequential sum of distances in token order) / |U|.
//  MEDIAN_RADIUS_X: x * lower median over non-empty clusters of the
//  sequential (token-order) mean member distance.
__global__ void ms_tau_kernel(int N, int rule, double x, const HeadSeg *__restrict__ seg,
                              const double *__restrict__ dist, const int32_t *__restrict__ perm,
                              const int32_t *__restrict__ off, int cap, MsHead *__restrict__ st) {
    extern __shared__ double rad[];  // [n2]
    __shared__ int nrad;
    int h = blockIdx.x;
    HeadSeg g = seg[h];
    if (g.nrows <= 0 || st[h].stage != 0) return;
    const double *dh = dist + (size_t)h * N;
    if (rule == 0) {
        if (threadIdx.x == 0) st[h].tau = x;
        return;
    }
    if (rule == 1) {
        if (threadIdx.x == 0) {
            double s = 0.0;
            for (int i = 0; i < g.nrows; i++) s = dadd(s, dh[i]);
            st[h].tau = dmul(x, ddiv(s, (double)g.nrows));
        }
        return;
    }
    int n2 = 1;
    while (n2 < g.k) n2 <<= 1;
    if (threadIdx.x == 0) nrad = 0;
    __syncthreads();
    const int32_t *o = off + (size_t)h * (cap + 1);
    for (int j = threadIdx.x; j < n2; j += blockDim.x) rad[j] = INFINITY;
    __syncthreads();
    for (int j = threadIdx.x; j < g.k; j += blockDim.x) {
        int b = o[j], e = o[j + 1];
        if (e > b) {
            double s = 0.0;
            for (int r = b; r < e; r++) s = dadd(s, dh[perm[(size_t)h * N + r]]);
            rad[j] = ddiv(s, (double)(e - b));
            atomicAdd(&nrad, 1);
        }
    }
    __syncthreads();
    for (int k = 2; k <= n2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n2; i += blockDim.x) {
                int l = i ^ j;
                if (l > i) {
                    double a = rad[i], b = rad[l];
                    bool up = (i & k) == 0;
                    if (up ? (a > b) : (a < b)) { rad[i] = b; rad[l] = a; }
                }
            }
            __syncthreads();
        }
    }
    if (threadIdx.x == 0) st[h].tau = dmul(x, rad[(nrad - 1) / 2]);
}

// Keep the positions of U whose distance is not < tau (order preserved), then
// advance the head's stage: |C| += m_t.  One CTA per head.
__global__ void ms_remove_kernel(int N, const HeadSeg *__restrict__ seg, const double *__restrict__ dist,
                                 const int32_t *__restrict__ U, int32_t *__restrict__ Unext, MsHead *__restrict__ st) {
    __shared__ int wsum[32];
    __shared__ int base;
    int h = blockIdx.x;
    HeadSeg g = seg[h];
    if (g.nrows <= 0) return;
    const double tau = st[h].tau;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
    if (tid == 0) base = 0;
    __syncthreads();
    for (int p0 = 0; p0 < g.nrows; p0 += blockDim.x) {
        int pos = p0 + tid;
        int keep = (pos < g.nrows) && !(dist[(size_t)h * N + pos] < tau);
        unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) wsum[w] = __popc(bal);
        __syncthreads();
        int before = base;
        for (int u = 0; u < w; u++) before += wsum[u];
        if (keep) Unext[(size_t)h * N + before + __popc(bal & ((1u << lane) - 1u))] = U[(size_t)h * N + pos];
        __syncthreads();
        if (tid == 0) {
            int t = 0;
            for (int u = 0; u < nw; u++) t += wsum[u];
            base += t;
        }
        __syncthreads();
    }
    if (tid == 0) {
        MsHead s = st[h];
        s.same = base == g.nrows ? 1 : 0;
        s.nu = base;
        s.nc += s.mt;
        s.stage += 1;
        st[h] = s;
    }
}

// Final pass over all tokens with every centre of C; also publishes
// nclusters and the flag F.
__global__ void ms_final_kernel(int H, int nrows, const MsHead *__restrict__ st, HeadSeg *__restrict__ seg,
                                int32_t *__restrict__ ncl, uint8_t *__restrict__ flag, int32_t *__restrict__ info) {
    __shared__ int mnc, mst;
    if (threadIdx.x == 0) {
        mnc = 0;
        mst = 0;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        MsHead s = st[h];
        HeadSeg g;
        g.nrows = s.nc > 0 ? nrows : 0;
        g.k = s.nc;
        g.cent_off = 0;
        g.pad = 0;
        seg[h] = g;
        if (ncl) ncl[h] = s.nc;
        if (flag) flag[h] = (uint8_t)s.flag;
        atomicMax(&mnc, s.nc);
        atomicMax(&mst, s.stage);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        info[5] = mnc;
        info[6] = mst;
    }
}

__global__ void seg_uniform_kernel(int H, int nrows, int k, HeadSeg *__restrict__ seg, int32_t *__restrict__ ncl,
                                   uint8_t *__restrict__ flag) {
    int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    HeadSeg g;
    g.nrows = nrows;
    g.k = k;
    g.cent_off = 0;
    g.pad = 0;
    seg[h] = g;
    if (ncl) ncl[h] = k;
    if (flag) flag[h] = 0;
}

// Per-head pass descriptors from device cluster counts (nk may be NULL), less
// `sub` groups that the pass does not cluster (the text-key group).  A count
// outside [0, cap] (caller memory) is clamped and records ST_INVALID: the
// sort and every pass over the descriptors size their tables by cap.
__global__ void seg_from_counts_kernel(int H, int nrows, const int32_t *__restrict__ ncl, int kfix, int sub, int cap,
                                       HeadSeg *__restrict__ seg, int *status) {
    int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    HeadSeg g;
    g.nrows = nrows;
    g.k = clamp_count((ncl ? ncl[h] : kfix) - sub, cap - sub, status);
    g.cent_off = 0;
    g.pad = 0;
    seg[h] = g;
}

// ---------------------------------------------------------------------------
// Single-cluster stages on chip.  Once a head's stage size m_t is 1 it stays 1
// (m_t = min(|U|, ceil(m0 |U| / N)) cannot grow while |U| shrinks), so every
// remaining stage of the head clusters U into one cluster.  Such a stage is
// complete after one k-means round: every row goes to cluster 0, so the first
// update gives the centre every later round repeats.  One CTA per head runs all
// of the head's remaining stages back to back, with the arithmetic and order
// of the host-driven stage:
//   init   c = working vector of U's first row (kept if iters = 0, or on the
//          sphere when the member sum is zero);
//   update s_t = sum over U in list (token) order of w_i[t], in double;
//          EUCLID c_t = s_t / |U|; SPHERE c_t = s_t / sqrt(sum_t s_t^2);
//   d_i    = sqrt(sum over t in order of (w_i[t] - c_t)^2) with c as stored (fp32);
//   U     <- the rows with !(d_i < tau), order kept; |C| += 1.
// The control of every stage is ms_control_kernel's: |U| = 0 ends the head,
// |C| >= N_max sets F and ends it, |C| + 1 > capacity records ST_CAPACITY.
// The working vectors of the rows in U when the kernel starts are computed once
// into wc (double, [H, wrows, D], row = position in that first list), and U is
// replaced by positions into wc as the stages shrink it.
template <typename T, int D>
__global__ void __launch_bounds__(256) ms_single_kernel(const T *__restrict__ x, int N, int nrows, int m0, int nmax,
                                                        int cap_c, int iters, const double *__restrict__ norm,
                                                        int mode, int32_t *__restrict__ Ua, int32_t *__restrict__ Ub,
                                                        double *__restrict__ wc, int wrows, MsHead *__restrict__ st,
                                                        float *__restrict__ cent, int cap, int *status) {
    __shared__ double ssum[D];
    __shared__ float cs[D];
    __shared__ double snr;
    __shared__ int wsum[8];
    __shared__ int base;
    const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    MsHead s = st[h];  // every thread keeps the same copy; thread 0 writes it back
    if (s.done || s.nu <= 0) return;
    if (s.nu > wrows) {  // cannot happen when m_t = 1 (|U| <= N / m0); left to the host loop
        return;
    }
    int32_t *U = Ua + (size_t)h * N, *P = Ub + (size_t)h * N;
    const T *xh = x + (size_t)h * N * D;
    const double *nh = norm + (size_t)h * N;
    double *wh = wc + (size_t)h * wrows * D;
    // working vectors of U, in list order; positions replace tokens from here on
    for (int e = tid; e < s.nu * D; e += blockDim.x) {
        const int r = e / D, t = e - r * D;
        const int tok = U[r];
        wh[e] = work_val(xh + (size_t)tok * D, t, mode, nh[tok]);
    }
    for (int r = tid; r < s.nu; r += blockDim.x) P[r] = r;
    int32_t *Pn = U;  // the other buffer
    __syncthreads();
    for (;;) {
        // ---- control (every thread takes the same decision)
        if (s.nu <= 0) { s.done = 1; break; }
        if (s.nc >= nmax) { s.flag = 1; s.done = 1; break; }
        const long long num = (long long)m0 * s.nu;
        int mt = (int)((num + nrows - 1) / nrows);
        if (mt > s.nu) mt = s.nu;
        if (mt != 1) break;  // not a single-cluster stage: back to the host loop
        if (s.nc + 1 > cap_c) {
            if (tid == 0) set_status(status, ST_CAPACITY);
            s.done = 1;
            break;
        }
        // ---- centre: init, then (iters >= 1) the update over U in list order
        const int p0 = P[0];
        if (tid < D) {
            cs[tid] = (float)wh[(size_t)p0 * D + tid];
            if (iters > 0) {
                double acc = 0.0;
                int i = 0;
                for (; i + 8 <= s.nu; i += 8) {
                    double v[8];
#pragma unroll
                    for (int u = 0; u < 8; u++) v[u] = wh[(size_t)P[i + u] * D + tid];
#pragma unroll
                    for (int u = 0; u < 8; u++) acc = dadd(acc, v[u]);
                }
                for (; i < s.nu; i++) acc = dadd(acc, wh[(size_t)P[i] * D + tid]);
                ssum[tid] = acc;
            }
        }
        __syncthreads();
        if (iters > 0) {
            if (mode == MODE_EUCLID) {
                if (tid < D) cs[tid] = (float)ddiv(ssum[tid], (double)s.nu);
            } else {
                if (tid == 0) {
                    double ss = 0.0;
                    for (int u = 0; u < D; u++) ss = dadd(ss, dmul(ssum[u], ssum[u]));
                    snr = sqrt(ss);
                }
                __syncthreads();
                if (tid < D && snr > 0.0) cs[tid] = (float)ddiv(ssum[tid], snr);
            }
        }
        __syncthreads();
        if (tid < D) cent[((size_t)h * cap + s.nc) * D + tid] = cs[tid];
        // ---- distances to the centre and ordered compaction of the rows kept
        if (tid == 0) base = 0;
        __syncthreads();
        for (int q0 = 0; q0 < s.nu; q0 += blockDim.x) {
            const int i = q0 + tid;
            int keep = 0, pi = 0;
            if (i < s.nu) {
                pi = P[i];
                const double2 *row = reinterpret_cast<const double2 *>(wh + (size_t)pi * D);
                double acc = 0.0;
#pragma unroll 4
                for (int t2 = 0; t2 < D / 2; t2++) {
                    const double2 v = row[t2];
                    const double d0 = dsub(v.x, (double)cs[2 * t2]);
                    acc = dadd(acc, dmul(d0, d0));
                    const double d1 = dsub(v.y, (double)cs[2 * t2 + 1]);
                    acc = dadd(acc, dmul(d1, d1));
                }
                keep = !(sqrt(acc) < s.tau);
            }
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            if (lane == 0) wsum[w] = __popc(bal);
            __syncthreads();
            int before = base;
            for (int u = 0; u < w; u++) before += wsum[u];
            if (keep) Pn[before + __popc(bal & ((1u << lane) - 1u))] = pi;
            __syncthreads();
            if (tid == 0) {
                int tt = 0;
                for (int u = 0; u < (int)(blockDim.x >> 5); u++) tt += wsum[u];
                base += tt;
            }
            __syncthreads();
        }
        const bool same = base == s.nu;
        s.nu = base;
        s.nc += 1;
        s.stage += 1;
        if (same && s.nc < nmax) {
            // no row left U: every later stage repeats this one (same U, same
            // centre) until |C| >= N_max; their centres are this one's
            const int r = nmax - s.nc;
            for (int e = tid; e < r * D; e += blockDim.x)
                cent[((size_t)h * cap + s.nc) * D + e] = cs[e % D];
            s.nc += r;
            s.stage += r;
        }
        int32_t *tmp = P;
        P = Pn;
        Pn = tmp;
        __syncthreads();  // this stage's reads of base and P are done before the next stage writes them
    }
    if (tid == 0) st[h] = s;
}

int k_ms_single(const void *x, int dtype, int H, int N, int D, int nrows, int m0, int nmax, int cap_c, int iters,
                const double *norm, int mode, int32_t *U, int32_t *U2, double *wc, int wrows, MsHead *st,
                float *cent, int cap, int *status, cudaStream_t s) {
#define AC_MS_SINGLE(T, DD)                                                                                     \
    ms_single_kernel<T, DD><<<H, 256, 0, s>>>(static_cast<const T *>(x), N, nrows, m0, nmax, cap_c, iters, norm, \
                                              mode, U, U2, wc, wrows, st, cent, cap, status)
    if (dtype == DT_BF16) {
        if (D == 64) AC_MS_SINGLE(__nv_bfloat16, 64);
        else AC_MS_SINGLE(__nv_bfloat16, 128);
    } else {
        if (D == 64) AC_MS_SINGLE(float, 64);
        else AC_MS_SINGLE(float, 128);
    }
#undef AC_MS_SINGLE
    note_launch();
    return 0;
}

void k_ms_repeat(int H, int D, MsHead *st, float *cent, int cap, cudaStream_t s) {
    ms_repeat_kernel<<<H, 256, 0, s>>>(D, st, cent, cap);
    note_launch();
}

// One CTA per head.  A centre is a duplicate when an earlier one has the same
// bits in every element; a 32-bit hash of each centre (in shared memory)
// screens the pairs, and equal hashes are compared element by element.
__global__ void dedup_cent_kernel(int D, const HeadSeg *__restrict__ seg, const float *__restrict__ cent, int cap,
                                  float *__restrict__ cu, int32_t *__restrict__ cmap, HeadSeg *__restrict__ segu) {
    extern __shared__ uint32_t hsh[];  // [cap] hashes, then [cap] first-copy flags
    uint32_t *first = hsh + cap;
    __shared__ int wsum[32];
    const int h = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const HeadSeg g = seg[h];
    const int k = g.k;
    const uint32_t *c = reinterpret_cast<const uint32_t *>(cent + (size_t)h * cap * D);
    for (int j = tid; j < k; j += nt) {
        uint32_t x = 2166136261u;
        for (int t = 0; t < D; t++) x = (x ^ c[(size_t)j * D + t]) * 16777619u;
        hsh[j] = x;
    }
    __syncthreads();
    for (int j = tid; j < k; j += nt) {
        uint32_t f = 1u;
        for (int i = 0; i < j && f; i++) {
            if (hsh[i] != hsh[j]) continue;
            bool eq = true;
            for (int t = 0; t < D && eq; t++) eq = c[(size_t)i * D + t] == c[(size_t)j * D + t];
            if (eq) f = 0u;
        }
        first[j] = f;
    }
    __syncthreads();
    // ordered compaction of the first copies (block-wide exclusive scan)
    int base = 0;
    for (int j0 = 0; j0 < k; j0 += nt) {
        const int j = j0 + tid;
        const int f = j < k ? (int)first[j] : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        const int lane = tid & 31, w = tid >> 5;
        if (lane == 0) wsum[w] = __popc(bal);
        __syncthreads();
        int before = base;
        for (int u = 0; u < w; u++) before += wsum[u];
        if (f) {
            const int u = before + __popc(bal & ((1u << lane) - 1u));
            cmap[(size_t)h * cap + u] = j;
            for (int t = 0; t < D; t++)
                cu[((size_t)h * cap + u) * D + t] = cent[((size_t)h * cap + j) * D + t];
        }
        __syncthreads();
        for (int u = 0; u < nt / 32; u++) base += wsum[u];
        __syncthreads();
    }
    if (tid == 0) {
        HeadSeg o = g;
        o.k = base;
        o.cent_off = 0;
        segu[h] = o;
    }
}

__global__ void map_ids_kernel(int N, const HeadSeg *__restrict__ seg, const int32_t *__restrict__ cmap, int cap,
                               int32_t *__restrict__ assign) {
    const int h = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= seg[h].nrows) return;
    const int a = assign[(size_t)h * N + i];
    if (a >= 0 && a < cap) assign[(size_t)h * N + i] = cmap[(size_t)h * cap + a];
}

void k_dedup_cent(int H, int D, const HeadSeg *seg, const float *cent, int cap, float *cu, int32_t *cmap,
                  HeadSeg *segu, cudaStream_t s) {
    const size_t smem = (size_t)2 * cap * sizeof(uint32_t);
    if (smem > 48 * 1024) cudaFuncSetAttribute(dedup_cent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dedup_cent_kernel<<<H, 256, smem, s>>>(D, seg, cent, cap, cu, cmap, segu);
    note_launch();
}

void k_map_ids(int H, int N, const HeadSeg *seg, const int32_t *cmap, int cap, int32_t *assign, cudaStream_t s) {
    map_ids_kernel<<<dim3((N + 255) / 256, H), 256, 0, s>>>(N, seg, cmap, cap, assign);
    note_launch();
}

void k_ms_init(int H, int N, int nrows, MsHead *st, int32_t *U, int32_t *U2, cudaStream_t s) {
    dim3 g((N + 255) / 256, H);
    ms_init_kernel<<<g, 256, 0, s>>>(H, N, nrows, st, U, U2); note_launch();
}
void k_ms_control(int H, int N, int m0, int nmax, int cap, MsHead *st, HeadSeg *seg, int32_t *info, int *status,
                  cudaStream_t s) {
    ms_control_kernel<<<1, 256, 0, s>>>(H, N, m0, nmax, cap, st, seg, info, status); note_launch();
}
void k_ms_tau(int H, int N, int rule, double x, const HeadSeg *seg, const double *dist, const int32_t *perm,
              const int32_t *off, int cap, int kmax, MsHead *st, cudaStream_t s) {
    int n2 = 1;
    while (n2 < kmax) n2 <<= 1;
    size_t smem = (size_t)n2 * sizeof(double);
    // the attribute belongs to the current device: set it on every call that needs it
    if (smem > 48 * 1024) cudaFuncSetAttribute(ms_tau_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    ms_tau_kernel<<<H, 256, smem, s>>>(N, rule, x, seg, dist, perm, off, cap, st); note_launch();
}
void k_ms_remove(int H, int N, const HeadSeg *seg, const double *dist, const int32_t *U, int32_t *Unext, MsHead *st,
                 cudaStream_t s) {
    ms_remove_kernel<<<H, 1024, 0, s>>>(N, seg, dist, U, Unext, st); note_launch();
}
void k_ms_final(int H, int nrows, const MsHead *st, HeadSeg *seg, int32_t *ncl, uint8_t *flag, int32_t *info,
                cudaStream_t s) {
    ms_final_kernel<<<1, 256, 0, s>>>(H, nrows, st, seg, ncl, flag, info); note_launch();
}
void k_seg_uniform(int H, int nrows, int k, HeadSeg *seg, int32_t *ncl, uint8_t *flag, cudaStream_t s) {
    seg_uniform_kernel<<<(H + 127) / 128, 128, 0, s>>>(H, nrows, k, seg, ncl, flag); note_launch();
}
void k_seg_from_counts(int H, int nrows, const int32_t *ncl, int kfix, int cap, HeadSeg *seg, int *status,
                       cudaStream_t s, int sub) {
    seg_from_counts_kernel<<<(H + 127) / 128, 128, 0, s>>>(H, nrows, ncl, kfix, sub, cap, seg, status); note_launch();
}

// The text-key group after key clustering: rows [nrows, N) of every head get
// id = the head's cluster count (seg.k of the final pass), its count is N -
// nrows, and the head's cluster count grows by one.
__global__ void text_group_kernel(int H, int N, int nrows, const HeadSeg *__restrict__ seg, int32_t *__restrict__ assign,
                                  int32_t *__restrict__ count, int cap, int32_t *__restrict__ ncl) {
    const int h = blockIdx.y;
    const int id = seg[h].k;
    const int i = nrows + blockIdx.x * blockDim.x + threadIdx.x;
    if (i < N) assign[(size_t)h * N + i] = id;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (count) count[(size_t)h * cap + id] = N - nrows;
        ncl[h] = id + 1;
    }
}
void k_text_group(int H, int N, int nrows, const HeadSeg *seg, int32_t *assign, int32_t *count, int cap,
                  int32_t *ncl, cudaStream_t s) {
    const int T = N - nrows;
    text_group_kernel<<<dim3((T + 255) / 256, H), 256, 0, s>>>(H, N, nrows, seg, assign, count, cap, ncl);
    note_launch();
}

}  // namespace ac
