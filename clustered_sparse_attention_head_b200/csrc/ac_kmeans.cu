// k-means kernels of AdaCluster ("AdaCluster: Adaptive Query-Key Clustering for
// Sparse Attention in Video Generation"): spherical k-means on normalised
// queries (§3.1) and Euclidean k-means on keys (§3.2.1), used per stage by
// Algorithm 1 (§3.2.2).
//
// Decisions (which centroid is closest) are made in double precision with the
// same operation order as a plain sequential loop, so that they are exact up
// to the input values: a fp32 screening pass finds the best two candidates of
// every row and a rigorous rounding bound; only rows whose top-2 gap lies
// within that bound are re-scored exactly (a warp per row).  Centroid sums are
// per-cluster double sums in token order over the cluster-sorted permutation,
// which makes the update deterministic.
#include "ac_kernels.cuh"

namespace ac {

// ---------------------------------------------------------------- row norms
// norm[h,i] = sqrt(sum_t x_t^2) (double, sequential).  With check_finite,
// a NaN/Inf element records ST_NONFINITE.
template <typename T, int D>
__global__ void __launch_bounds__(256)
    row_norm_kernel(const T *__restrict__ x, int N, double *__restrict__ norm, int check, int *status) {
    // One thread per row: 16-byte vector loads, squares summed sequentially in
    // double in element order (the order of a plain loop).
    constexpr int PER = 16 / sizeof(T);   // elements per vector
    constexpr int NV = D / PER;           // vectors per row
    constexpr int CH = NV < 8 ? NV : 8;   // vectors loaded ahead of the sum
    const int h = blockIdx.y, r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= N) return;
    const uint4 *row = reinterpret_cast<const uint4 *>(x + ((size_t)h * N + r) * D);
    double ss = 0.0;
    bool bad = false;
#pragma unroll
    for (int c0 = 0; c0 < NV; c0 += CH) {
        uint4 v[CH];
#pragma unroll
        for (int i = 0; i < CH; i++) v[i] = __ldg(row + c0 + i);
#pragma unroll
        for (int i = 0; i < CH; i++) {
            const T *e = reinterpret_cast<const T *>(&v[i]);
#pragma unroll
            for (int u = 0; u < PER; u++) {
                const float f = to_f(e[u]);
                if (check && !isfinite(f)) bad = true;
                ss = dadd(ss, dmul((double)f, (double)f));
            }
        }
    }
    if (bad) set_status(status, ST_NONFINITE);
    norm[(size_t)h * N + r] = sqrt(ss);
}


// ------------------------------------------------------------------- init
// Centroid j of the pass = working vector of listed row floor(j * nrows / k).
template <typename T>
__global__ void init_cent_kernel(const T *__restrict__ x, int N, int D, const int32_t *__restrict__ rows,
                                 const double *__restrict__ norm, const HeadSeg *__restrict__ seg, int mode,
                                 float *__restrict__ cent, int cap) {
    int h = blockIdx.y, j = blockIdx.x;
    HeadSeg s = seg[h];
    if (s.nrows <= 0 || j >= s.k) return;
    int r = (int)(((int64_t)j * s.nrows) / s.k);
    int tok = rows ? rows[(size_t)h * N + r] : r;
    const T *xi = x + ((size_t)h * N + tok) * D;
    double nrm = norm[(size_t)h * N + tok];
    float *c = cent + ((size_t)h * cap + s.cent_off + j) * D;
    for (int t = threadIdx.x; t < D; t += blockDim.x) c[t] = (float)work_val(xi, t, mode, nrm);
}

// ||c_j||^2 as fp32 (from double) and max_j ||c_j|| (rounded up) per head.
__global__ void cent_prep_kernel(const float *__restrict__ cent, int cap, int D, const HeadSeg *__restrict__ seg,
                                 float *__restrict__ cn2, float *__restrict__ cmax) {
    int h = blockIdx.x;
    HeadSeg s = seg[h];
    __shared__ float red[32];
    float mx = 0.f;
    for (int j = threadIdx.x; j < s.k; j += blockDim.x) {
        const float *c = cent + ((size_t)h * cap + s.cent_off + j) * D;
        double ss = 0.0;
        for (int t = 0; t < D; t++) ss += (double)c[t] * (double)c[t];
        cn2[(size_t)h * cap + j] = (float)ss;
        float nr = (float)(sqrt(ss) * (1.0 + 1e-6));
        mx = fmaxf(mx, nr);
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) m = fmaxf(m, red[w]);
        cmax[h] = m;
    }
}

// ---------------------------------------------------------- fp32 screening
// CTA tile: 128 rows x 64 centroids per step, 256 threads, thread = 8 rows x 4
// centroids.  Screening score (smaller is closer):
//   EUCLID: ||c||^2 - 2 x.c      SPHERE: -(x.mu)   (x unnormalised: the argmax
//   of x_hat.mu equals that of x.mu since ||x|| > 0; zero rows tie everywhere).
// Each score is within E of its exact value, E = (D+8) 2^-23 (2||x|| Cmax +
// Cmax^2) for EUCLID and (D+8) 2^-23 ||x|| Cmax for SPHERE (twice the standard
// bound for a length-D fp32 dot product, plus the final combination), plus an
// absolute 2^-100 for underflow.  A row whose best two scores are more than 2E
// apart has a certain winner; the others go to the exact pass.
constexpr int SCR_ROWS = 128, SCR_COLS = 64, SCR_XS = SCR_ROWS + 4, SCR_CS = SCR_COLS + 4;

template <typename T, int D>
__global__ void __launch_bounds__(256) assign_screen_kernel(
    const T *__restrict__ x, int N, const int32_t *__restrict__ rows, const HeadSeg *__restrict__ seg,
    const float *__restrict__ cent, int cap, const float *__restrict__ cn2, const float *__restrict__ cmax, int mode,
    int32_t *__restrict__ assign, int32_t *__restrict__ amb_list, int32_t *__restrict__ amb_count) {
    extern __shared__ __align__(16) float smf[];
    float *Xs = smf;                 // [D][SCR_XS]
    float *Cs = smf + D * SCR_XS;    // [D][SCR_CS]
    int h = blockIdx.y;
    HeadSeg s = seg[h];
    int r0 = blockIdx.x * SCR_ROWS;
    if (r0 >= s.nrows || s.k <= 0) return;
    const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
    const float *ch = cent + ((size_t)h * cap + s.cent_off) * D;
    const float *cn = cn2 + (size_t)h * cap;

    for (int idx = tid; idx < SCR_ROWS * D; idx += 256) {
        int rr = idx / D, t = idx - rr * D;
        int pos = r0 + rr;
        float v = 0.f;
        if (pos < s.nrows) {
            int tok = rows ? rows[(size_t)h * N + pos] : pos;
            v = to_f(x[((size_t)h * N + tok) * D + t]);
        }
        Xs[t * SCR_XS + rr] = v;
    }

    __syncthreads();
    float xn_row = 0.f;
    if (tid < SCR_ROWS) {
        float xx = 0.f;
        for (int t = 0; t < D; t++) xx = fmaf(Xs[t * SCR_XS + tid], Xs[t * SCR_XS + tid], xx);
        xn_row = sqrtf(xx) * 1.001f;
    }

    float b1[8], b2[8];
    int i1[8];
#pragma unroll
    for (int a = 0; a < 8; a++) { b1[a] = INFINITY; b2[a] = INFINITY; i1[a] = 0; }

    for (int j0 = 0; j0 < s.k; j0 += SCR_COLS) {
        __syncthreads();
        for (int idx = tid; idx < SCR_COLS * D; idx += 256) {
            int jj = idx / D, t = idx - jj * D;
            int j = j0 + jj;
            Cs[t * SCR_CS + jj] = (j < s.k) ? ch[(size_t)j * D + t] : 0.f;
        }
        __syncthreads();
        float acc[8][4];
#pragma unroll
        for (int a = 0; a < 8; a++)
#pragma unroll
            for (int b = 0; b < 4; b++) acc[a][b] = 0.f;
#pragma unroll 4
        for (int t = 0; t < D; t++) {
            float4 xa = *reinterpret_cast<const float4 *>(&Xs[t * SCR_XS + tr * 8]);
            float4 xb = *reinterpret_cast<const float4 *>(&Xs[t * SCR_XS + tr * 8 + 4]);
            float4 cc = *reinterpret_cast<const float4 *>(&Cs[t * SCR_CS + tc * 4]);
            float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            float cv[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
            for (int a = 0; a < 8; a++)
#pragma unroll
                for (int b = 0; b < 4; b++) acc[a][b] = fmaf(xv[a], cv[b], acc[a][b]);
        }
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int j = j0 + tc * 4 + b;
            if (j < s.k) {
                float c2 = (mode == MODE_EUCLID) ? cn[j] : 0.f;
#pragma unroll
                for (int a = 0; a < 8; a++) {
                    float sc = (mode == MODE_EUCLID) ? (c2 - 2.f * acc[a][b]) : -acc[a][b];
                    if (sc < b1[a]) { b2[a] = b1[a]; b1[a] = sc; i1[a] = j; }
                    else if (sc < b2[a]) b2[a] = sc;
                }
            }
        }
    }
    __syncthreads();
    // reduce the 16 column groups of every row (buffers overwrite the X tile)
    float *R1 = smf;                        // [128][16]
    float *R2 = smf + SCR_ROWS * 16;        // [128][16]
    int *RI = reinterpret_cast<int *>(smf + 2 * SCR_ROWS * 16);
#pragma unroll
    for (int a = 0; a < 8; a++) {
        int rr = tr * 8 + a;
        R1[rr * 16 + tc] = b1[a];
        R2[rr * 16 + tc] = b2[a];
        RI[rr * 16 + tc] = i1[a];
    }
    __syncthreads();
    if (tid < SCR_ROWS) {
        int rr = tid, pos = r0 + rr;
        if (pos < s.nrows) {
            float B1 = INFINITY, B2 = INFINITY;
            int I1 = 0x7fffffff;
            for (int g = 0; g < 16; g++) {
                float v1 = R1[rr * 16 + g], v2 = R2[rr * 16 + g];
                int iv = RI[rr * 16 + g];
                if (v1 < B1 || (v1 == B1 && iv < I1)) {
                    B2 = fminf(B2, B1);
                    B1 = v1;
                    I1 = iv;
                } else {
                    B2 = fminf(B2, v1);
                }
                B2 = fminf(B2, v2);
            }
            float xn = xn_row;
            float cm = cmax[h];
            // + 2^-100: absolute slack for subnormal products, where the
            // relative bound fails
            float E = (float)(D + 8) * 1.1920929e-7f * ((mode == MODE_EUCLID) ? (2.f * xn * cm + cm * cm) : (xn * cm)) +
                      0x1p-100f;
            if (s.k > 1 && !(B2 - B1 > 2.f * E)) {
                int slot = atomicAdd(&amb_count[h], 1);
                amb_list[(size_t)h * N + slot] = pos;
            } else {
                assign[(size_t)h * N + pos] = I1;
            }
        }
    }
}

// ------------------------------------------------------------- exact pass
// One warp per ambiguous row: every centroid is scored in double with the
// sequential order of a plain loop (EUCLID: sum (x-c)^2; SPHERE: sum x_hat*mu),
// and the best score wins, ties to the lowest id.
template <typename T, int D>
__global__ void __launch_bounds__(256) assign_exact_kernel(
    const T *__restrict__ x, int N, const int32_t *__restrict__ rows, const HeadSeg *__restrict__ seg,
    const float *__restrict__ cent, int cap, const double *__restrict__ norm, int mode,
    const int32_t *__restrict__ amb_list, const int32_t *__restrict__ amb_count, const int2 *__restrict__ amb_cand,
    int32_t *__restrict__ assign, bool vec) {
    __shared__ double xs[8][D];
    int h = blockIdx.y;
    HeadSeg s = seg[h];
    int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int na = amb_count[h];
    const float *ch = cent + ((size_t)h * cap + s.cent_off) * D;
    for (int a = blockIdx.x * 8 + warp; a < na; a += gridDim.x * 8) {
        int pos = amb_list[(size_t)h * N + a];
        int tok = rows ? rows[(size_t)h * N + pos] : pos;
        const T *xi = x + ((size_t)h * N + tok) * D;
        double nrm = norm[(size_t)h * N + tok];
        __syncwarp();
        for (int t = lane; t < D; t += 32) xs[warp][t] = work_val(xi, t, mode, nrm);
        __syncwarp();
        double best = (mode == MODE_EUCLID) ? INFINITY : -INFINITY;
        int bj = 0x7fffffff;
        // shortlisted rows: only the two candidates the screen left open (a
        // candidate outside [0, k) means a full scan)
        int2 cand = amb_cand ? amb_cand[(size_t)h * N + a] : make_int2(-1, -1);
        if (cand.x >= s.k || cand.y >= s.k || cand.y < 0) cand = make_int2(-1, -1);
        const int jcount = cand.x >= 0 ? 2 : s.k;
        for (int q = lane; q < jcount; q += 32) {
            const int j = cand.x >= 0 ? (q == 0 ? cand.x : cand.y) : q;
            const float *c = ch + (size_t)j * D;
            double acc = 0.0;
            // partial unrolling: a fully unrolled loop hoists all D loads into
            // registers and spills; the summation order is unchanged
            // (the centroid read 16 bytes at a time when its base is 16-byte
            // aligned: rows of D floats keep that alignment)
            if (mode == MODE_EUCLID) {
                if (vec) {
                    const float4 *c4 = reinterpret_cast<const float4 *>(c);
#pragma unroll 4
                    for (int t4 = 0; t4 < D / 4; t4++) {
                        const float4 f = __ldg(c4 + t4);
                        const float cf[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const double df = dsub(xs[warp][4 * t4 + e], (double)cf[e]);
                            acc = dadd(acc, dmul(df, df));
                        }
                    }
                } else {
#pragma unroll 16
                    for (int t = 0; t < D; t++) {
                        double df = dsub(xs[warp][t], (double)c[t]);
                        acc = dadd(acc, dmul(df, df));
                    }
                }
                if (acc < best) { best = acc; bj = j; }
            } else {
                if (vec) {
                    const float4 *c4 = reinterpret_cast<const float4 *>(c);
#pragma unroll 4
                    for (int t4 = 0; t4 < D / 4; t4++) {
                        const float4 f = __ldg(c4 + t4);
                        const float cf[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                        for (int e = 0; e < 4; e++) acc = dadd(acc, dmul(xs[warp][4 * t4 + e], (double)cf[e]));
                    }
                } else {
#pragma unroll 16
                    for (int t = 0; t < D; t++) acc = dadd(acc, dmul(xs[warp][t], (double)c[t]));
                }
                if (acc > best) { best = acc; bj = j; }
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            double ob = __shfl_xor_sync(0xffffffffu, best, o);
            int oj = __shfl_xor_sync(0xffffffffu, bj, o);
            bool better = (mode == MODE_EUCLID) ? (ob < best) : (ob > best);
            if (better || (ob == best && oj < bj)) { best = ob; bj = oj; }
        }
        // no score compared as better than the start (every score NaN): the
        // lowest candidate, so the id is always one of the pass's clusters
        if (bj == 0x7fffffff) bj = cand.x >= 0 ? min(cand.x, cand.y) : 0;
        if (lane == 0) assign[(size_t)h * N + pos] = bj;
    }
}

// ------------------------------------------------------------- distances
// dist[h,pos] = ||x' - c_assign||_2 in double (x' = working vector).
template <typename T, int D>
__global__ void dist_kernel(const T *__restrict__ x, int N, const int32_t *__restrict__ rows,
                            const HeadSeg *__restrict__ seg, const float *__restrict__ cent, int cap,
                            const double *__restrict__ norm, int mode, const int32_t *__restrict__ assign,
                            double *__restrict__ dist, bool vec) {
    int h = blockIdx.y;
    HeadSeg s = seg[h];
    int pos = blockIdx.x * blockDim.x + threadIdx.x;
    if (pos >= s.nrows) return;
    int tok = rows ? rows[(size_t)h * N + pos] : pos;
    const T *xi = x + ((size_t)h * N + tok) * D;
    double nrm = norm[(size_t)h * N + tok];
    // ids are in [0, k) by construction; clamped so that no id can read
    // outside the centroid block
    const int a = min(max(assign[(size_t)h * N + pos], 0), max(s.k - 1, 0));
    const float *c = cent + ((size_t)h * cap + s.cent_off + a) * D;
    double acc = 0.0;
    if (!vec) {  // a base not 16-byte aligned: element by element
        for (int t = 0; t < D; t++) {
            const double df = dsub(work_val(xi, t, mode, nrm), (double)c[t]);
            acc = dadd(acc, dmul(df, df));
        }
        dist[(size_t)h * N + pos] = sqrt(acc);
        return;
    }
    // the row and its centroid read 16 bytes at a time (both bases 16-byte
    // aligned, rows of 128 or 256 bytes); the squares are still summed element
    // by element in order
    constexpr int V = 16 / (int)sizeof(T);  // row elements per load
    const uint4 *xv = reinterpret_cast<const uint4 *>(xi);
    const float4 *cv = reinterpret_cast<const float4 *>(c);
#pragma unroll 2
    for (int u = 0; u < D / V; u++) {
        const uint4 w = __ldg(xv + u);
        const T *xs = reinterpret_cast<const T *>(&w);
        float cf[V];
#pragma unroll
        for (int i = 0; i < V / 4; i++) {
            const float4 f = __ldg(cv + u * (V / 4) + i);
            cf[4 * i] = f.x;
            cf[4 * i + 1] = f.y;
            cf[4 * i + 2] = f.z;
            cf[4 * i + 3] = f.w;
        }
#pragma unroll
        for (int e = 0; e < V; e++) {
            const double df = dsub(work_val(xs, e, mode, nrm), (double)cf[e]);
            acc = dadd(acc, dmul(df, df));
        }
    }
    dist[(size_t)h * N + pos] = sqrt(acc);
}

// ----------------------------------------------------------------- update
// Cluster j of head h (grid x = j, y = h): members are perm[off[j] .. off[j+1])
// in token order; element t of their working vectors is summed in double in
// that order.  EUCLID: c = sum / count.  SPHERE: mu = sum / ||sum||.  Empty
// clusters (or a zero sum) keep their centroid.
//
// The member rows are staged through shared memory: chunks of R rows are
// copied by cp.async as 16-byte pieces (every thread copies four pieces, so a
// CTA keeps two chunks in flight while it sums a third), and thread t adds
// element t of the chunk's rows in order.  The token ids of a chunk are read
// one chunk before its copy is issued, so the copy never waits for them.  On
// the sphere the working value x/||x|| is the correctly rounded quotient,
// computed from y = RN(1/||x||) (one per row) with Markstein's correction
// (q = RN(x y), r = x - ||x|| q exactly by FMA, RN(q + r y) = RN(x / ||x||);
// Markstein 1990, see Muller et al., Handbook of Floating-Point Arithmetic,
// on division by FMA), the value plain division gives.
namespace {
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int NPEND> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(NPEND) : "memory");
}
}  // namespace

// 8 KB chunks, three stages: about 25 KB of shared memory, eight CTAs (clusters) per SM
constexpr int UPD_THREADS = 128, UPD_STAGES = 3, UPD_CHUNK_BYTES = 8192;
constexpr int UPD_PIECES_PER_THREAD = UPD_CHUNK_BYTES / 16 / UPD_THREADS;

template <typename T, int D>
__global__ void __launch_bounds__(UPD_THREADS) update2_kernel(const T *__restrict__ x, int N,
                                                             const HeadSeg *__restrict__ seg,
                                                             const int32_t *__restrict__ perm,
                                                             const int32_t *__restrict__ off, int cap,
                                                             const double *__restrict__ norm, int mode,
                                                             float *__restrict__ cent,
                                                             const int32_t *__restrict__ order) {
    constexpr int ROW_BYTES = D * (int)sizeof(T);
    constexpr int R = UPD_CHUNK_BYTES / ROW_BYTES;   // rows per chunk
    constexpr int PIECES = ROW_BYTES / 16;           // 16-byte pieces per row
    static_assert(R * PIECES == UPD_PIECES_PER_THREAD * UPD_THREADS, "four pieces per thread");
    static_assert(R <= UPD_THREADS && D <= UPD_THREADS, "one thread per row / element");
    extern __shared__ __align__(16) unsigned char upd_smem[];
    T *rows = reinterpret_cast<T *>(upd_smem);                                           // [S][R][D]
    // per staged row (||x||, RN(1/||x||)), read by the summing threads as one 16-byte pair
    double2 *nry = reinterpret_cast<double2 *>(upd_smem + UPD_STAGES * UPD_CHUNK_BYTES);  // [S][R]
    __shared__ double ssum[D];
    __shared__ double snr;
    // grid (head, rank): with an order the rank-th largest cluster of the head
    const int h = blockIdx.x, tid = threadIdx.x;
    const int j = order ? order[(size_t)h * cap + blockIdx.y] : (int)blockIdx.y;
    const HeadSeg s = seg[h];
    if (s.nrows <= 0 || j < 0 || j >= s.k) return;
    const int32_t *o = off + (size_t)h * (cap + 1);
    const int b = o[j], e = o[j + 1];
    if (e <= b) return;
    const int n = e - b, nchunks = (n + R - 1) / R;
    const int32_t *ph = perm + (size_t)h * N + b;
    const T *xh = x + (size_t)h * N * D;
    const double *nh = norm + (size_t)h * N;
    const bool sphere = mode == MODE_SPHERE;
    // token ids of this thread's pieces of the next chunk to copy (and, on the
    // sphere, of row tid, whose norm it copies); -1 past the chunk's end
    int tk[UPD_PIECES_PER_THREAD], tkn = -1;
    auto load_tokens = [&](int c) {
        const int r0 = c * R, nr = c < nchunks ? min(R, n - r0) : 0;
#pragma unroll
        for (int k = 0; k < UPD_PIECES_PER_THREAD; k++) {
            const int r = (tid + k * UPD_THREADS) / PIECES;
            tk[k] = r < nr ? ph[r0 + r] : -1;
        }
        tkn = (sphere && tid < nr) ? ph[r0 + tid] : -1;
    };
    // copy chunk c (tokens in tk) into stage c % S: one commit group per chunk, also when empty
    auto issue = [&](int c) {
        unsigned char *dst = reinterpret_cast<unsigned char *>(rows) + (size_t)(c % UPD_STAGES) * UPD_CHUNK_BYTES;
#pragma unroll
        for (int k = 0; k < UPD_PIECES_PER_THREAD; k++) {
            const int pc = tid + k * UPD_THREADS, r = pc / PIECES, q = pc - r * PIECES;
            if (tk[k] >= 0)
                cp_async16(dst + r * ROW_BYTES + q * 16,
                           reinterpret_cast<const unsigned char *>(xh + (size_t)tk[k] * D) + q * 16);
        }
        if (tkn >= 0) cp_async8(&nry[(c % UPD_STAGES) * R + tid].x, nh + tkn);
        cp_async_commit();
    };
#pragma unroll
    for (int c = 0; c < UPD_STAGES - 1; c++) {
        load_tokens(c);
        issue(c);
    }
    load_tokens(UPD_STAGES - 1);
    double acc = 0.0;
    for (int c = 0; c < nchunks; c++) {
        cp_async_wait<UPD_STAGES - 2>();
        __syncthreads();  // chunk c has landed for every thread; stage (c - 1) % S is free
        const int st = c % UPD_STAGES, nr = min(R, n - c * R);
        if (sphere) {
            // y = RN(1/||x||) once per row, 0 for a zero row
            if (tid < nr) {
                const double v = nry[st * R + tid].x;
                nry[st * R + tid].y = v > 0.0 ? __drcp_rn(v) : 0.0;
            }
            __syncthreads();
        }
        issue(c + UPD_STAGES - 1);
        load_tokens(c + UPD_STAGES);
        if (tid < D) {
            const T *rs = rows + (size_t)st * R * D + tid;
            if (sphere) {
                const double2 *ny_s = nry + st * R;
                // a zero row (||x|| = 0) has every element +-0 and y = 0, so q0,
                // rr and q are all +0, which is what a zero row adds
#pragma unroll 8
                for (int r = 0; r < nr; r++) {
                    const double v = (double)to_f(rs[r * D]);
                    const double2 ny = ny_s[r];
                    const double q0 = dmul(v, ny.y);
                    const double rr = __fma_rn(-ny.x, q0, v);
                    acc = dadd(acc, __fma_rn(rr, ny.y, q0));
                }
            } else {
#pragma unroll 8
                for (int r = 0; r < nr; r++) acc = dadd(acc, (double)to_f(rs[r * D]));
            }
        }
    }
    cp_async_wait<0>();
    float *c = cent + ((size_t)h * cap + s.cent_off + j) * D;
    if (!sphere) {
        if (tid < D) c[tid] = (float)ddiv(acc, (double)n);
        return;
    }
    if (tid < D) ssum[tid] = acc;
    __syncthreads();
    if (tid == 0) {
        double ss = 0.0;
        for (int u = 0; u < D; u++) ss = dadd(ss, dmul(ssum[u], ssum[u]));
        snr = sqrt(ss);
    }
    __syncthreads();
    if (tid < D && snr > 0.0) c[tid] = (float)ddiv(acc, snr);
}

// Mean ||q|| over the members of each cluster (sequential double sum in
// token order); 0 for empty clusters.
__global__ void mean_norm_kernel(int N, const HeadSeg *__restrict__ seg, const int32_t *__restrict__ perm,
                                 const int32_t *__restrict__ off, int cap, const double *__restrict__ norm,
                                 float *__restrict__ mean_norm) {
    int h = blockIdx.y;
    int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= cap) return;
    HeadSeg s = seg[h];
    float out = 0.f;
    if (j < s.k) {
        const int32_t *o = off + (size_t)h * (cap + 1);
        int b = o[j], e = o[j + 1];
        double acc = 0.0;
        for (int r = b; r < e; r++) acc = dadd(acc, norm[(size_t)h * N + perm[(size_t)h * N + r]]);
        if (e > b) out = (float)ddiv(acc, (double)(e - b));
    }
    mean_norm[(size_t)h * cap + j] = out;
}

// ------------------------------------------------------------- launchers
template <typename T>
static void launch_row_norm(const void *x, int H, int N, int D, double *norm, int check, int *status,
                            cudaStream_t st) {
    dim3 g((N + 255) / 256, H);
    if (D == 64) row_norm_kernel<T, 64><<<g, 256, 0, st>>>((const T *)x, N, norm, check, status);
    else row_norm_kernel<T, 128><<<g, 256, 0, st>>>((const T *)x, N, norm, check, status);
    note_launch();
}

void k_row_norm(const void *x, int dtype, int H, int N, int D, double *norm, int check, int *status,
                cudaStream_t st) {
    if (dtype == DT_BF16) launch_row_norm<__nv_bfloat16>(x, H, N, D, norm, check, status, st);
    else launch_row_norm<float>(x, H, N, D, norm, check, status, st);
}

void k_init_cent(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const double *norm,
                 const HeadSeg *seg, int kmax, int mode, float *cent, int cap, cudaStream_t st) {
    dim3 g(kmax, H);
    if (dtype == DT_BF16)
        init_cent_kernel<__nv_bfloat16><<<g, 128, 0, st>>>((const __nv_bfloat16 *)x, N, D, rows, norm, seg, mode,
                                                             cent, cap);
    else
        init_cent_kernel<float><<<g, 128, 0, st>>>((const float *)x, N, D, rows, norm, seg, mode, cent, cap);
    note_launch();
}

template <typename T, int D>
static void launch_assign(const void *x, int H, int N, const int32_t *rows, const HeadSeg *seg, int nrows_max,
                          const float *cent, int cap, const float *cn2, const float *cmax, const double *norm,
                          int mode, int32_t *assign, int32_t *amb_list, int32_t *amb_count, cudaStream_t st) {
    size_t smem = (size_t)D * (SCR_XS + SCR_CS) * sizeof(float);
    // the attribute belongs to the current device: set it on every call
    cudaFuncSetAttribute(assign_screen_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 g((nrows_max + SCR_ROWS - 1) / SCR_ROWS, H);
    assign_screen_kernel<T, D><<<g, 256, smem, st>>>((const T *)x, N, rows, seg, cent, cap, cn2, cmax, mode, assign,
                                                      amb_list, amb_count); note_launch();
    dim3 g2(64, H);
    const bool vec = (reinterpret_cast<uintptr_t>(cent) & 15) == 0;
    assign_exact_kernel<T, D><<<g2, 256, 0, st>>>((const T *)x, N, rows, seg, cent, cap, norm, mode, amb_list,
                                                   amb_count, nullptr, assign, vec); note_launch();
}

void k_assign(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const HeadSeg *seg,
              int nrows_max, const float *cent, int cap, float *cn2, float *cmax, const double *norm, int mode,
              int32_t *assign, int32_t *amb_list, int32_t *amb_count, cudaStream_t st) {
    cudaMemsetAsync(amb_count, 0, sizeof(int32_t) * H, st);
    cent_prep_kernel<<<H, 256, 0, st>>>(cent, cap, D, seg, cn2, cmax); note_launch();
    if (dtype == DT_BF16) {
        if (D == 64)
            launch_assign<__nv_bfloat16, 64>(x, H, N, rows, seg, nrows_max, cent, cap, cn2, cmax, norm, mode, assign,
                                             amb_list, amb_count, st);
        else
            launch_assign<__nv_bfloat16, 128>(x, H, N, rows, seg, nrows_max, cent, cap, cn2, cmax, norm, mode,
                                              assign, amb_list, amb_count, st);
    } else {
        if (D == 64)
            launch_assign<float, 64>(x, H, N, rows, seg, nrows_max, cent, cap, cn2, cmax, norm, mode, assign,
                                     amb_list, amb_count, st);
        else
            launch_assign<float, 128>(x, H, N, rows, seg, nrows_max, cent, cap, cn2, cmax, norm, mode, assign,
                                      amb_list, amb_count, st);
    }
}

void k_assign_exact(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const HeadSeg *seg,
                    const float *cent, int cap, const double *norm, int mode, const int32_t *amb_list,
                    const int32_t *amb_count, const int2 *amb_cand, int32_t *assign, cudaStream_t st) {
    dim3 g2(64, H);
    const bool vec = (reinterpret_cast<uintptr_t>(cent) & 15) == 0;
#define AC_EXACT(T, DD)                                                                                          \
    assign_exact_kernel<T, DD><<<g2, 256, 0, st>>>((const T *)x, N, rows, seg, cent, cap, norm, mode, amb_list, \
                                                    amb_count, amb_cand, assign, vec)
    if (dtype == DT_BF16) {
        if (D == 64) AC_EXACT(__nv_bfloat16, 64);
        else AC_EXACT(__nv_bfloat16, 128);
    } else {
        if (D == 64) AC_EXACT(float, 64);
        else AC_EXACT(float, 128);
    }
#undef AC_EXACT
    note_launch();
}

void k_dist(const void *x, int dtype, int H, int N, int D, const int32_t *rows, const HeadSeg *seg,
            int nrows_max, const float *cent, int cap, const double *norm, int mode, const int32_t *assign,
            double *dist, cudaStream_t st) {
    dim3 g((nrows_max + 127) / 128, H);
    const bool vec = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(cent)) & 15) == 0;
#define AC_DIST(T, DD) \
    dist_kernel<T, DD><<<g, 128, 0, st>>>((const T *)x, N, rows, seg, cent, cap, norm, mode, assign, dist, vec)
    if (dtype == DT_BF16) {
        if (D == 64) AC_DIST(__nv_bfloat16, 64);
        else AC_DIST(__nv_bfloat16, 128);
    } else {
        if (D == 64) AC_DIST(float, 64);
        else AC_DIST(float, 128);
    }
#undef AC_DIST
    note_launch();
}

void k_update(const void *x, int dtype, int H, int N, int D, const HeadSeg *seg, int kmax, const int32_t *perm,
              const int32_t *off, int cap, const double *norm, int mode, float *cent, cudaStream_t st,
              const int32_t *order) {
    // blocks start in launch order, x fastest: every head's rank-0 cluster, then rank 1, ...
    dim3 g(H, kmax);
    // staged rows (8 KB chunks, three stages) plus the rows' norms and reciprocals
#define AC_UPD(T, DD)                                                                                             \
    do {                                                                                                          \
        constexpr int R_ = UPD_CHUNK_BYTES / (DD * (int)sizeof(T));                                               \
        constexpr int SM_ = UPD_STAGES * (UPD_CHUNK_BYTES + 2 * R_ * 8);                                          \
        cudaFuncSetAttribute(update2_kernel<T, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM_);             \
        update2_kernel<T, DD><<<g, UPD_THREADS, SM_, st>>>((const T *)x, N, seg, perm, off, cap, norm, mode, cent, order); \
    } while (0)
    if (dtype == DT_BF16) {
        if (D == 64) AC_UPD(__nv_bfloat16, 64);
        else AC_UPD(__nv_bfloat16, 128);
    } else {
        if (D == 64) AC_UPD(float, 64);
        else AC_UPD(float, 128);
    }
#undef AC_UPD
    note_launch();
}

void k_mean_norm(int H, int N, const HeadSeg *seg, const int32_t *perm, const int32_t *off, int cap,
                 const double *norm, float *mean_norm, cudaStream_t st) {
    dim3 g((cap + 127) / 128, H);
    mean_norm_kernel<<<g, 128, 0, st>>>(N, seg, perm, off, cap, norm, mean_norm); note_launch();
}

// ------------------------------------------------------------ convergence
// Fixed-count k-means stops per head once an assignment pass reproduces the
// previous pass: the update of an unchanged assignment gives back the same
// centroids, so every later pass would repeat it exactly and stopping changes
// no result.  kst[4h + 0] = stopped, + 1 = rows changed in this pass, + 2 =
// rounds (assignment + update) run.  A stopped head's pass segment gets 0 rows,
// which every clustering kernel already skips.

// Rows of each active head whose assignment differs from `prev`; then prev = assign.
__global__ void conv_check_kernel(int N, const HeadSeg *__restrict__ seg, const int32_t *__restrict__ assign,
                                  int32_t *__restrict__ prev, int32_t *__restrict__ kst, int first) {
    const int h = blockIdx.y;
    const int nrows = seg[h].nrows;
    if ((int)(blockIdx.x * blockDim.x) >= nrows) return;  // whole CTA
    const int pos = blockIdx.x * blockDim.x + threadIdx.x;
    int diff = 0;
    if (pos < nrows) {
        const size_t i = (size_t)h * N + pos;
        const int32_t a = assign[i];
        diff = (!first && a != prev[i]) ? 1 : 0;
        prev[i] = a;
    }
    const int n = __syncthreads_count(diff);
    if (threadIdx.x == 0 && n) atomicAdd(&kst[4 * h + 1], n);
}

// After pass `it`: stop the heads whose assignment did not change.
__global__ void conv_decide_kernel(int H, HeadSeg *__restrict__ seg, int32_t *__restrict__ kst, int it) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    if (it == 0) kst[4 * h + 0] = 0;
    if (seg[h].nrows > 0) {
        if (it > 0 && kst[4 * h + 1] == 0) {
            kst[4 * h + 0] = 1;
            seg[h].nrows = 0;
        } else {
            kst[4 * h + 2] = it + 1;
        }
    }
    kst[4 * h + 1] = 0;
}

void k_conv_check(int H, int N, const HeadSeg *seg, const int32_t *assign, int32_t *prev, int32_t *kst, int first,
                  cudaStream_t st) {
    conv_check_kernel<<<dim3((N + 255) / 256, H), 256, 0, st>>>(N, seg, assign, prev, kst, first);
    note_launch();
}
void k_conv_decide(int H, HeadSeg *seg, int32_t *kst, int it, cudaStream_t st) {
    conv_decide_kernel<<<(H + 127) / 128, 128, 0, st>>>(H, seg, kst, it);
    note_launch();
}

}  // namespace ac
