// Cluster-sort permutation and gather (Algorithm 3, "K* = K[Index]"):
// a stable counting sort of tokens by cluster id, so every cluster's tokens are
// contiguous and in increasing token order, then a 16-byte vectorised row
// gather into cluster order.
//
// Stable ranks: each warp owns a tile of 256 positions and walks it in order,
// 32 at a time; __match_any_sync groups equal ids within the 32 and a
// shared-memory counter per id gives each position its rank among equal ids
// of the tile.  Tile histograms are then scanned per cluster (over tiles) and
// per head (over clusters) to place every position.
#include "ac_kernels.cuh"

namespace ac {

__global__ void __launch_bounds__(128) rank_hist_kernel(const int32_t *__restrict__ ids, const HeadSeg *__restrict__ seg,
                                                        int N, int cap, int ntiles_max, int32_t *__restrict__ rank,
                                                        int32_t *__restrict__ hist, int *status) {
    // A CTA tile holds SORT_TILE = 1024 positions, 256 per warp.  Each warp
    // ranks its 256 positions in order with per-warp shared counters; the
    // counters are then turned into per-warp prefixes (warp order = position
    // order) so that a rank counts the equal ids earlier in the whole tile.
    extern __shared__ int32_t sh[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const HeadSeg s = seg[h];
    const int tile = blockIdx.x;
    const int base = tile * SORT_TILE + warp * (SORT_TILE / 4);
    if (tile * SORT_TILE >= s.nrows || tile >= ntiles_max) return;  // whole CTA
    int32_t *cnt = sh + warp * cap;
    for (int j = lane; j < s.k; j += 32) cnt[j] = 0;
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
    int rk[8], idv[8];
#pragma unroll
    for (int c = 0; c < 8; c++) {
        const int pos = base + c * 32 + lane;
        bool valid = pos < s.nrows;
        int id = valid ? ids[(size_t)h * N + pos] : -1;
        if (valid && (id < 0 || id >= s.k)) {
            set_status(status, 1);
            id = -1;
            valid = false;
        }
        const unsigned m = __match_any_sync(0xffffffffu, id);
        int r = 0;
        if (valid) r = cnt[id] + __popc(m & lt);
        __syncwarp();
        if (valid && lane == __ffs(m) - 1) cnt[id] += __popc(m);
        __syncwarp();
        rk[c] = r;
        idv[c] = id;
    }
    __syncthreads();
    int32_t *hh = hist + ((size_t)h * ntiles_max + tile) * cap;
    for (int j = threadIdx.x; j < s.k; j += blockDim.x) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < 4; w++) {
            const int v = sh[w * cap + j];
            sh[w * cap + j] = run;
            run += v;
        }
        hh[j] = run;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 8; c++) {
        const int pos = base + c * 32 + lane;
        if (idv[c] >= 0) rank[(size_t)h * N + pos] = rk[c] + cnt[idv[c]];
    }
}

// Per cluster j: exclusive scan over tiles (in place) and the cluster size.
__global__ void scan_tiles_kernel(const HeadSeg *__restrict__ seg, int cap, int ntiles_max,
                                  int32_t *__restrict__ hist, int32_t *__restrict__ cnt) {
    int h = blockIdx.y;
    int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= cap) return;
    HeadSeg s = seg[h];
    int run = 0;
    if (j < s.k && s.nrows > 0) {
        int nt = (s.nrows + SORT_TILE - 1) / SORT_TILE;
        int32_t *p = hist + (size_t)h * ntiles_max * cap + j;
        // eight tiles' counts loaded before they are scanned, so the loads do
        // not wait on one another
        int t = 0;
        for (; t + 8 <= nt; t += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) v[u] = p[(size_t)(t + u) * cap];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                p[(size_t)(t + u) * cap] = run;
                run += v[u];
            }
        }
        for (; t < nt; t++) {
            int v = p[(size_t)t * cap];
            p[(size_t)t * cap] = run;
            run += v;
        }
    }
    cnt[(size_t)h * cap + j] = run;
}

// Size class of a non-empty cluster: 4 per octave (the exponent and the two
// bits below the leading one), 0..127
__device__ __forceinline__ int size_class(int v) {
    const int e = 31 - __clz(v);
    const int m = e >= 2 ? ((v >> (e - 2)) & 3) : 0;
    return min(4 * e + m, 127);
}

// Per head: exclusive scan of cluster sizes -> offsets [cap + 1].  With
// `order`, also the non-empty clusters by size class, largest first (-1 after
// them): a kernel with one CTA per cluster launched over (head, rank) then
// starts every head's largest clusters first.
__global__ void scan_clusters_kernel(const int32_t *__restrict__ cnt, int cap, int32_t *__restrict__ off,
                                     int32_t *__restrict__ order) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    int h = blockIdx.x;
    const int32_t *c = cnt + (size_t)h * cap;
    int32_t *o = off + (size_t)h * (cap + 1);
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int b = 0; b < cap; b += blockDim.x) {
        int j = b + threadIdx.x;
        int v = j < cap ? c[j] : 0;
        int x = v;
        int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        for (int d = 1; d < 32; d <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) warp_tot[w] = x;
        __syncthreads();
        if (w == 0) {
            int nw = blockDim.x >> 5;
            int t = lane < nw ? warp_tot[lane] : 0;
            for (int d = 1; d < 32; d <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, t, d);
                if (lane >= d) t += y;
            }
            if (lane < nw) warp_tot[lane] = t;
        }
        __syncthreads();
        int incl = x + (w > 0 ? warp_tot[w - 1] : 0) + carry;
        if (j < cap) o[j] = incl - v;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) o[cap] = carry;
    if (!order) return;
    __shared__ int32_t cls[128];
    __shared__ int32_t nonempty;
    int32_t *ord = order + (size_t)h * cap;
    for (int i = threadIdx.x; i < 128; i += blockDim.x) cls[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < cap; j += blockDim.x)
        if (c[j] > 0) atomicAdd(&cls[size_class(c[j])], 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int i = 127; i >= 0; i--) {
            const int t = cls[i];
            cls[i] = run;
            run += t;
        }
        nonempty = run;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < cap; j += blockDim.x)
        if (c[j] > 0) ord[atomicAdd(&cls[size_class(c[j])], 1)] = j;
    for (int p = nonempty + threadIdx.x; p < cap; p += blockDim.x) ord[p] = -1;
}

__global__ void scatter_kernel(const int32_t *__restrict__ ids, const int32_t *__restrict__ rows,
                               const HeadSeg *__restrict__ seg, int N, int cap, int ntiles_max,
                               const int32_t *__restrict__ rank, const int32_t *__restrict__ hist,
                               const int32_t *__restrict__ off, int32_t *__restrict__ perm) {
    int h = blockIdx.y;
    HeadSeg s = seg[h];
    int pos = blockIdx.x * blockDim.x + threadIdx.x;
    if (pos >= s.nrows) return;
    int id = ids[(size_t)h * N + pos];
    if (id < 0 || id >= s.k) return;
    int tile = pos / SORT_TILE;
    int p = off[(size_t)h * (cap + 1) + id] + hist[((size_t)h * ntiles_max + tile) * cap + id] +
            rank[(size_t)h * N + pos];
    perm[(size_t)h * N + p] = rows ? rows[(size_t)h * N + pos] : pos;
}

size_t sort_hist_elems(int H, int N, int cap) {
    size_t nt = (size_t)(N + SORT_TILE - 1) / SORT_TILE;
    return (size_t)H * nt * cap;
}

void k_sort(const int32_t *ids, const int32_t *rows, const HeadSeg *seg, int H, int N, int nrows_max, int cap,
            int32_t *rank, int32_t *hist, int32_t *cnt, int32_t *off, int32_t *perm, int *status, cudaStream_t st,
            int32_t *order) {
    int ntiles_max = (N + SORT_TILE - 1) / SORT_TILE;
    int nt = (nrows_max + SORT_TILE - 1) / SORT_TILE;
    size_t smem = (size_t)4 * cap * sizeof(int32_t);
    // the attribute belongs to the current device: set it on every call that needs it
    if (smem > 48 * 1024) cudaFuncSetAttribute(rank_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (nt > 0) {
        dim3 g1(nt, H);
        rank_hist_kernel<<<g1, 128, smem, st>>>(ids, seg, N, cap, ntiles_max, rank, hist, status); note_launch();
    }
    dim3 g2((cap + 127) / 128, H);
    scan_tiles_kernel<<<g2, 128, 0, st>>>(seg, cap, ntiles_max, hist, cnt); note_launch();
    scan_clusters_kernel<<<H, 1024, 0, st>>>(cnt, cap, off, order); note_launch();
    if (nrows_max > 0) {
        dim3 g3((nrows_max + 255) / 256, H);
        scatter_kernel<<<g3, 256, 0, st>>>(ids, rows, seg, N, cap, ntiles_max, rank, hist, off, perm); note_launch();
    }
}

// dst[h, p, :] = src[h, perm[h, p], :], 16 bytes per thread.
__global__ void gather_rows_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                   const int32_t *__restrict__ perm, int N, int vec_per_row) {
    int h = blockIdx.y;
    size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    size_t tot = (size_t)N * vec_per_row;
    if (idx >= tot) return;
    int p = (int)(idx / vec_per_row), v = (int)(idx - (size_t)p * vec_per_row);
    int tok = perm[(size_t)h * N + p];
    dst[((size_t)h * N + p) * vec_per_row + v] = src[((size_t)h * N + tok) * vec_per_row + v];
}

void k_gather_rows(const void *src, void *dst, const int32_t *perm, int H, int N, int row_bytes, cudaStream_t st) {
    int vpr = row_bytes / 16;
    size_t tot = (size_t)N * vpr;
    dim3 g((unsigned)((tot + 255) / 256), H);
    gather_rows_kernel<<<g, 256, 0, st>>>((const uint4 *)src, (uint4 *)dst, perm, N, vpr); note_launch();
}

}  // namespace ac
