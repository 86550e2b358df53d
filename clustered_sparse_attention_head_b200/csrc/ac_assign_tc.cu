// Tensor-core screening pass of the k-means assignment (AdaCluster §3.1 and
// §3.2.1: queries to the centroid of largest q_hat.mu, keys to the closest
// centroid) for bf16 inputs on sm_100a.
//
// Each fp32 centroid is split into two bf16 parts, c = c_hi + c_lo + r with
// |r| <= 2^-18 |c| elementwise, and the CTA computes X (C_hi + C_lo)^T for a
// 128-row tile of X against 128-centroid chunks with tcgen05.mma (both parts
// accumulate into one fp32 TMEM tile; bf16 x bf16 products are exact).  The
// four epilogue warps (one row per thread) read the tile from TMEM and keep
// each row's three smallest scores, shifted by a per-row constant:
//   EUCLID: ||c||^2 - 2 x.c + ||x||^2     SPHERE: ||x|| - x.mu
// (smaller is closer).  Each score travels as a packed key, its low mantissa
// bits replaced by the column index, so a min/max network on keys alone
// tracks the indices too; the packing adds at most 2^(kb-22) |key| to the
// error of a score (kb index bits).
// Error bound of a dot product: |x.r| <= 2^-18 ||x|| ||c|| plus fp32
// accumulation of 2d exact products, <= 2d 2^-23 ||x|| ||c||; the pass uses
// E_dot = 2^-13 ||x|| Cmax (>= 2x that bound for d <= 128), plus an absolute
// 2^-100 for fp32 underflow.  A row whose best two keys are within 2E plus the
// packing bounds goes to the exact double pass (assign_exact_kernel), so the
// final decision equals the exact one.
//
// Warp 0 issues TMA (X tile once, then C_hi/C_lo chunks), warp 1 issues the
// MMAs into two TMEM accumulators (double buffer; whole warp, one elected
// lane), warps 2-5 run the epilogue.  The epilogue keeps four independent
// running top-3 lists per row (column pairs interleaved four ways, each pair
// merged into a list with two 3-input mins) and merges them at the end: one
// serial list per row made the kernel latency-bound, and separate index
// selects made it bound by the ALU pipe.  All waits are bounded.
#include "ac_kernels.cuh"

namespace ac {

__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float m;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

template <int D> struct TcCfg {
    static constexpr int ROWS = 128, COLS = 128;
    static constexpr int DB = D / 64;                        // 128-byte column blocks
    static constexpr int STAGES = D == 128 ? 1 : 2;
    static constexpr int X_BYTES = ROWS * D * 2;
    static constexpr int C_BYTES = COLS * D * 2;              // one part (hi or lo)
    static constexpr int OFF_X = 0;
    static constexpr int OFF_C = X_BYTES;                      // stage s: hi at +2s*C, lo at +(2s+1)*C
    static constexpr int OFF_BAR = OFF_C + STAGES * 2 * C_BYTES;
    static constexpr int OFF_CN = OFF_BAR + 256;  // ||c||^2 of the head, kpad floats
    // dynamic shared memory for a given kpad (plus 1 KB of alignment slack)
    static constexpr int smem_bytes(int kpad) { return OFF_CN + kpad * 4 + 1024; }
    static constexpr uint32_t TMEM_COLS = 256;
};

struct TcParams {
    int N, cap, kpad;
    const int32_t *rows;
    const HeadSeg *seg;
    const float *cn2, *cmax;
    const double *norm;
    int mode;
    int32_t *assign, *amb_list, *amb_count;
    int2 *amb_cand;
    int *status;
};

template <int D>
__global__ void __launch_bounds__(192, 2)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmChi,
                     const __grid_constant__ CUtensorMap tmClo, const TcParams p) {
    using C = TcCfg<D>;
    const int h = blockIdx.y;
    const HeadSeg s = p.seg[h];
    const int r0 = blockIdx.x * C::ROWS;
    if (r0 >= s.nrows || s.k <= 0) return;  // whole CTA
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *x_full = bars, *c_full = bars + 1, *c_empty = bars + 3, *d_full = bars + 5, *d_empty = bars + 7;
    uint64_t *drain = bars + 9;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 11);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = (s.k + C::COLS - 1) / C::COLS;

    if (threadIdx.x == 0) {
        mbar_init(x_full, 1);
        for (int i = 0; i < 2; i++) {
            mbar_init(c_full + i, 1);
            mbar_init(c_empty + i, 1);
            mbar_init(d_full + i, 1);
            mbar_init(d_empty + i, 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            int issued = -1;
            mbar_arrive_expect_tx(x_full, C::X_BYTES);
            for (int kb = 0; kb < C::DB; kb++)
                tma_load_2d(sm + C::OFF_X + kb * (C::ROWS * 128), &tmX, x_full, kb * 64, h * p.N + r0);
            const int crow0 = h * p.kpad;
            for (int j = 0; j < nch && ok; j++) {
                const int st = j % C::STAGES;
                const int u = j / C::STAGES;
                if (u >= 1 && !mbar_wait(c_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx(c_full + st, 2 * C::C_BYTES);
                unsigned char *hi = sm + C::OFF_C + (2 * st) * C::C_BYTES;
                unsigned char *lo = sm + C::OFF_C + (2 * st + 1) * C::C_BYTES;
                for (int kb = 0; kb < C::DB; kb++) {
                    tma_load_2d(hi + kb * (C::COLS * 128), &tmChi, c_full + st, kb * 64, crow0 + j * C::COLS);
                    tma_load_2d(lo + kb * (C::COLS * 128), &tmClo, c_full + st, kb * 64, crow0 + j * C::COLS);
                }
                issued = j;
            }
            if (!ok) {
                // wait (bounded) for this thread's copies before the CTA leaves
                uint64_t t0 = gtimer();
                while (!mbar_try_wait(x_full, 0) && gtimer() - t0 < 200000000ull) {
                }
                for (int j = issued - C::STAGES + 1; j <= issued; j++) {
                    if (j < 0) continue;
                    t0 = gtimer();
                    while (!mbar_try_wait(c_full + (j % C::STAGES), (j / C::STAGES) & 1) &&
                           gtimer() - t0 < 200000000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // whole warp, identical values in every lane; one elected lane issues
        bool ok = mbar_wait_warp(x_full, 0, abort_flag, p.status);
        constexpr uint32_t idesc = idesc_make(128, C::COLS, 1, false);
        const uint64_t xdesc = sdesc_sw128(smem_u32(sm + C::OFF_X), 16, 1024);
        const uint64_t cdesc = sdesc_sw128(smem_u32(sm + C::OFF_C), 16, 1024);
        for (int j = 0; j < nch && ok; j++) {
            const int st = j % C::STAGES;
            const int b = j & 1;
            if (!mbar_wait_warp(c_full + st, (j / C::STAGES) & 1, abort_flag, p.status)) { ok = false; break; }
            if (j >= 2 && !mbar_wait_warp(d_empty + b, ((j >> 1) - 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t dcol = tmem + b * C::COLS;
            // 16-byte units: hi part of stage st at 2st*C_BYTES, lo part at (2st+1)*C_BYTES
            const uint64_t hdesc = cdesc + (uint64_t)(((2 * st) * C::C_BYTES) >> 4);
            const uint64_t ldesc = cdesc + (uint64_t)(((2 * st + 1) * C::C_BYTES) >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 16; ks++) {
                const uint64_t a = xdesc + (uint64_t)(((ks / 4) * (C::ROWS * 128) + (ks % 4) * 32) >> 4);
                const uint64_t bo = (uint64_t)(((ks / 4) * (C::COLS * 128) + (ks % 4) * 32) >> 4);
                umma_f16_w(dcol, a, hdesc + bo, idesc, ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < D / 16; ks++) {
                const uint64_t a = xdesc + (uint64_t)(((ks / 4) * (C::ROWS * 128) + (ks % 4) * 32) >> 4);
                const uint64_t bo = (uint64_t)(((ks / 4) * (C::COLS * 128) + (ks % 4) * 32) >> 4);
                umma_f16_w(dcol, a, ldesc + bo, idesc, 1u);
            }
            umma_commit_w(c_empty + st);
            umma_commit_w(d_full + b);
        }
        if (!ok) {
            umma_commit_w(drain);
            uint64_t t0 = gtimer();
            while (!mbar_try_wait(drain, 0) && gtimer() - t0 < 200000000ull) {
            }
        }
    } else {
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        // ||c||^2 of this head's centroids (zero-padded to whole chunks) in
        // shared memory; the four epilogue warps share a named barrier
        float *cn_s = reinterpret_cast<float *>(sm + C::OFF_CN);
        const int kpadc = nch * C::COLS;
        // padding columns (zero centroid rows, x.c = 0) get a large finite
        // score, so their keys stay ordered numbers that never win
        for (int i = threadIdx.x - 64; i < kpadc; i += 128)
            cn_s[i] = i >= s.k ? 1e30f : (p.mode == MODE_EUCLID ? p.cn2[(size_t)h * p.cap + i] : 0.f);
        // this thread's row: ||x|| (rounded up) and the per-row shift
        // sigma = ||x||^2 (EUCLID) or ||x|| (SPHERE), which turns the scores
        // into ||x - c||^2 resp. ||x|| (1 - cos), small for the nearest centroids
        const int pos = r0 + row;
        const bool live = pos < s.nrows;
        float xn = 0.f;
        if (live) {
            const int tok = p.rows ? p.rows[(size_t)h * p.N + pos] : pos;
            xn = (float)(p.norm[(size_t)h * p.N + tok] * (1.0 + 1e-6));
        }
        const float sigma = (p.mode == MODE_EUCLID) ? xn * xn : xn;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // Packed keys: the shifted score with its low kb mantissa bits replaced
        // by the column index (kb = bits of the largest column).  min/max of
        // keys then carries the index along, and a key differs from its score
        // by less than 2^(kb-23) of its magnitude.  Four running top-3 lists of
        // keys (column pairs 2m, 2m+1 go to list m mod 4), updated a pair at a
        // time by merging the sorted pair into the sorted triple.
        const int kb = 32 - __clz(kpadc - 1);
        const uint32_t imask = (1u << kb) - 1u;
        float b1[4], b2[4], b3[4];
#pragma unroll
        for (int q = 0; q < 4; q++) b1[q] = b2[q] = b3[q] = INFINITY;
        const float wv = (p.mode == MODE_EUCLID) ? -2.f : -1.f;
        bool ok = true;
        for (int j = 0; j < nch; j++) {
            const int b = j & 1;
            if (!mbar_wait_warp(d_full + b, (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int pc = 0; pc < C::COLS / 32; pc++) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_addr + b * C::COLS + pc * 32, r);
                const int c0 = j * C::COLS + pc * 32;
                // 2^23 + c0: adding the in-group offset gives a float whose low
                // mantissa bits are the column index
                const float cbase = __uint_as_float(0x4B000000u + (uint32_t)c0);
                const float4 *cn4 = reinterpret_cast<const float4 *>(cn_s + c0);
#pragma unroll
                for (int i8 = 0; i8 < 4; i8++) {
                    const float4 ca = cn4[2 * i8], cb = cn4[2 * i8 + 1];
                    const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                    float key[8];
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        // EUCLID: ||c||^2 - 2 x.c + ||x||^2; SPHERE: ||x|| - x.mu
                        const float d = __fadd_rn(fmaf(wv, __uint_as_float(r[8 * i8 + e]), cc[e]), sigma);
                        const float ci = __fadd_rn(cbase, (float)(8 * i8 + e));
                        key[e] = __uint_as_float((__float_as_uint(d) & ~imask) | (__float_as_uint(ci) & imask));
                    }
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const float lo = fminf(key[2 * q], key[2 * q + 1]);
                        const float hi = fmaxf(key[2 * q], key[2 * q + 1]);
                        const float m11 = fmaxf(b1[q], lo), m21 = fmaxf(b2[q], lo), m12 = fmaxf(b1[q], hi);
                        b3[q] = fmin3(b3[q], m21, m12);
                        b2[q] = fmin3(b2[q], m11, hi);
                        b1[q] = fminf(b1[q], lo);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(d_empty + b);
        }
        // merge lists 1-3 into list 0 (keys are distinct, so no ties)
        float B1 = b1[0], B2 = b2[0], B3 = b3[0];
#pragma unroll
        for (int q = 1; q < 4; q++) {
            const float a1 = B1, a2 = B2, a3 = B3;
            B1 = fminf(a1, b1[q]);
            B2 = fmin3(a2, b2[q], fmaxf(a1, b1[q]));
            B3 = fminf(fmin3(a3, b3[q], fmaxf(a2, b1[q])), fmaxf(a1, b2[q]));
        }
        const int i1v = (int)(__float_as_uint(B1) & imask), i2v = (int)(__float_as_uint(B2) & imask);
        if (ok && live) {
            const float cm = p.cmax[h];
            const float edot = 1.220703125e-4f * xn * cm;  // 2^-13 ||x|| Cmax
            // + 2^-100: absolute slack for fp32 underflow (subnormal products and
            // sums in the MMA, subnormal keys), where relative bounds fail
            const float E = ((p.mode == MODE_EUCLID) ? 2.f * edot + 2.384185791e-7f * (cm * cm + 2.f * xn * cm) : edot) +
                            0x1p-100f;
            // a key is within 2^(kb-23) |key| (1 + tiny) of the shifted fp32
            // score, and the shift itself rounds to 2^-24 of it: 2^(kb-22)
            // bounds both.  The bound on exact - key grows with the key, so the
            // second key is the binding competitor of the first.
            const float rho = __uint_as_float((uint32_t)(127 + kb - 22) << 23);
            // A winner outside the pass's clusters (a padding column, which
            // only wins when every real score is NaN, infinite or above the
            // padding score) is never decided here: the exact pass rescans.
            const bool decided = B2 - B1 > 2.f * E + rho * (fabsf(B1) + fabsf(B2)) && i1v < s.k;
            if (s.k > 1 && !decided) {
                // Every centroid other than i1 and i2 has a key >= B3; if even
                // B3 is out of reach of B1, only the two are re-scored.
                const bool two = B3 - B1 > 2.f * E + rho * (fabsf(B1) + fabsf(B3)) && i1v < s.k && i2v < s.k;
                const int slot = atomicAdd(&p.amb_count[h], 1);
                p.amb_list[(size_t)h * p.N + slot] = pos;
                p.amb_cand[(size_t)h * p.N + slot] = two ? make_int2(i1v, i2v) : make_int2(-1, -1);
            } else {
                p.assign[(size_t)h * p.N + pos] = i1v;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Persistent form of the same screen.  One CTA per SM takes items of 256 rows
// (two X tiles) of one head in turn and runs both tiles against each
// centroid chunk, so a chunk is read from L2 once per 256 rows instead of per
// 128; the chunks are double-buffered (d = 128; four stages at d = 64), TMEM
// (both tiles x two accumulators = 512 columns) and the barriers live across
// items, and the next item's X tiles load while the last chunk's epilogue of
// the current item runs.  The decision rule, the packing and the bounds are the
// ones above, so the result is the same.  The per-column score shift (||c||^2,
// or 0 on the sphere, 1e30 for padding) is read from the padded table cnp that
// cent_split_kernel writes, so no table is refilled in shared memory between
// heads.  Warp 0 issues TMA, warp 1 the MMAs, warps 2-9 run the epilogue (tile
// (w - 2) / 4, TMEM lane quarter w % 4).
template <int D> struct Tc2Cfg {
    static constexpr int ROWS = 128, COLS = 128, TILES = 2;
    static constexpr int DB = D / 64;
    static constexpr int CST = D == 128 ? 2 : 4;
    static constexpr int X_BYTES = ROWS * D * 2;
    static constexpr int C_BYTES = COLS * D * 2;               // one part (hi or lo)
    static constexpr int OFF_X = 0;                             // tile t at t * X_BYTES
    static constexpr int OFF_C = TILES * X_BYTES;               // stage s: hi at 2s C_BYTES, lo at (2s+1) C_BYTES
    static constexpr int OFF_BAR = OFF_C + CST * 2 * C_BYTES;
    static constexpr int OFF_ITEMS = OFF_BAR + 512;             // item prefix per head [MAX_H + 1]
    static constexpr int MAX_H = 1024;
    static constexpr int SMEM = OFF_ITEMS + (MAX_H + 1) * 4 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int NTHREADS = 320;
    static constexpr int ITEM_ROWS = TILES * ROWS;
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Tc2Params {
    TcParams p;
    const float *cnp;  // [H, kpad] per-column shift
    int H;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    assign_tc2_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmChi,
                      const __grid_constant__ CUtensorMap tmClo, const Tc2Params q) {
    using C = Tc2Cfg<D>;
    const TcParams &p = q.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *x_full = bars, *x_empty = bars + 1;
    uint64_t *c_full = bars + 2, *c_empty = c_full + C::CST;          // [CST]
    uint64_t *d_full = c_empty + C::CST, *d_empty = d_full + 2;       // [2]
    uint64_t *drain = d_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(drain + 2);
    int *pre = reinterpret_cast<int *>(sm + C::OFF_ITEMS);            // items of heads < h
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(x_full, 1);
        mbar_init(x_empty, 1);
        for (int i = 0; i < C::CST; i++) {
            mbar_init(c_full + i, 1);
            mbar_init(c_empty + i, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(d_full + i, 1);
            mbar_init(d_empty + i, 256);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        // items per head: 256-row blocks of the pass (none when the head is inactive)
        int run = 0;
        for (int h = 0; h < q.H; h++) {
            pre[h] = run;
            const HeadSeg s = p.seg[h];
            run += (s.nrows > 0 && s.k > 0) ? (s.nrows + C::ITEM_ROWS - 1) / C::ITEM_ROWS : 0;
        }
        pre[q.H] = run;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = pre[q.H];
    // head of item i (the items of a head are consecutive)
    auto head_of = [&](int i) -> int {
        int lo = 0, hi = q.H - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pre[mid] <= i) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    };

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            uint32_t g = 0, it = 0;
            int last_chunk = -1;
            for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
                const int h = head_of(i);
                const HeadSeg s = p.seg[h];
                const int r0 = (i - pre[h]) * C::ITEM_ROWS;
                const int nch = (s.k + C::COLS - 1) / C::COLS;
                const int crow0 = h * p.kpad;
                // The first chunks' stages are freed by the previous item's MMAs,
                // so they load before the X tiles, which wait for that item's
                // last MMA (no wait here depends on this item's X tiles).
                const int early = nch < C::CST ? nch : C::CST;
                for (int j = 0; j < nch; j++) {
                    if (j == early) {
                        if (it >= 1 && !mbar_wait(x_empty, (it - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                        mbar_arrive_expect_tx(x_full, C::TILES * C::X_BYTES);
                        for (int t = 0; t < C::TILES; t++)
                            for (int kb = 0; kb < C::DB; kb++)
                                tma_load_2d(sm + C::OFF_X + t * C::X_BYTES + kb * (C::ROWS * 128), &tmX, x_full,
                                            kb * 64, h * p.N + r0 + t * C::ROWS);
                        it++;
                    }
                    const int st = (int)(g % C::CST);
                    const uint32_t u = g / C::CST;
                    if (u >= 1 && !mbar_wait(c_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(c_full + st, 2 * C::C_BYTES);
                    unsigned char *hi = sm + C::OFF_C + (2 * st) * C::C_BYTES;
                    unsigned char *lo = sm + C::OFF_C + (2 * st + 1) * C::C_BYTES;
                    for (int kb = 0; kb < C::DB; kb++) {
                        tma_load_2d(hi + kb * (C::COLS * 128), &tmChi, c_full + st, kb * 64, crow0 + j * C::COLS);
                        tma_load_2d(lo + kb * (C::COLS * 128), &tmClo, c_full + st, kb * 64, crow0 + j * C::COLS);
                    }
                    last_chunk = (int)g;
                    g++;
                }
                if (ok && early == nch) {
                    // every chunk went early: the X tiles follow them
                    if (it >= 1 && !mbar_wait(x_empty, (it - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(x_full, C::TILES * C::X_BYTES);
                    for (int t = 0; t < C::TILES; t++)
                        for (int kb = 0; kb < C::DB; kb++)
                            tma_load_2d(sm + C::OFF_X + t * C::X_BYTES + kb * (C::ROWS * 128), &tmX, x_full,
                                        kb * 64, h * p.N + r0 + t * C::ROWS);
                    it++;
                }
            }
            if (!ok) {
                // wait (bounded) for this thread's copies in flight before the CTA leaves
                uint64_t t0 = gtimer();
                if (it >= 1)
                    while (!mbar_try_wait(x_full, (it - 1) & 1) && gtimer() - t0 < 200000000ull) {
                    }
                for (int j = last_chunk - C::CST + 1; j <= last_chunk; j++) {
                    if (j < 0) continue;
                    t0 = gtimer();
                    while (!mbar_try_wait(c_full + (j % C::CST), (uint32_t)(j / C::CST) & 1) &&
                           gtimer() - t0 < 200000000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // whole warp, identical values in every lane; one elected lane issues
        constexpr uint32_t idesc = idesc_make(128, C::COLS, 1, false);
        const uint64_t xdesc = sdesc_sw128(smem_u32(sm + C::OFF_X), 16, 1024);
        const uint64_t cdesc = sdesc_sw128(smem_u32(sm + C::OFF_C), 16, 1024);
        bool ok = true;
        uint32_t g = 0, dc = 0, it = 0;
        for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
            const int h = head_of(i);
            const HeadSeg s = p.seg[h];
            const int nch = (s.k + C::COLS - 1) / C::COLS;
            if (!mbar_wait_warp(x_full, it & 1, abort_flag, p.status)) { ok = false; break; }
            it++;
            for (int j = 0; j < nch; j++) {
                const int st = (int)(g % C::CST);
                const int b = (int)(dc & 1);
                if (!mbar_wait_warp(c_full + st, (g / C::CST) & 1, abort_flag, p.status)) { ok = false; break; }
                if (dc >= 2 && !mbar_wait_warp(d_empty + b, ((dc >> 1) - 1) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t hdesc = cdesc + (uint64_t)(((2 * st) * C::C_BYTES) >> 4);
                const uint64_t ldesc = cdesc + (uint64_t)(((2 * st + 1) * C::C_BYTES) >> 4);
#pragma unroll
                for (int t = 0; t < C::TILES; t++) {
                    const uint32_t dcol = tmem + (uint32_t)((b * C::TILES + t) * C::COLS);
                    const uint64_t xt = xdesc + (uint64_t)((t * C::X_BYTES) >> 4);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ks++) {
                        const uint64_t a = xt + (uint64_t)(((ks / 4) * (C::ROWS * 128) + (ks % 4) * 32) >> 4);
                        const uint64_t bo = (uint64_t)(((ks / 4) * (C::COLS * 128) + (ks % 4) * 32) >> 4);
                        umma_f16_w(dcol, a, hdesc + bo, idesc, ks > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < D / 16; ks++) {
                        const uint64_t a = xt + (uint64_t)(((ks / 4) * (C::ROWS * 128) + (ks % 4) * 32) >> 4);
                        const uint64_t bo = (uint64_t)(((ks / 4) * (C::COLS * 128) + (ks % 4) * 32) >> 4);
                        umma_f16_w(dcol, a, ldesc + bo, idesc, 1u);
                    }
                }
                umma_commit_w(c_empty + st);
                umma_commit_w(d_full + b);
                g++;
                dc++;
            }
            if (!ok) break;
            umma_commit_w(x_empty);  // the item's X tiles are no longer read
        }
        if (!ok) {
            umma_commit_w(drain);
            uint64_t t0 = gtimer();
            while (!mbar_try_wait(drain, 0) && gtimer() - t0 < 200000000ull) {
            }
        }
    } else {
        const int et = (warp - 2) >> 2;  // tile of this epilogue warp
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const float wv = (p.mode == MODE_EUCLID) ? -2.f : -1.f;
        bool ok = true;
        uint32_t dc = 0;
        for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
            const int h = head_of(i);
            const HeadSeg s = p.seg[h];
            const int nch = (s.k + C::COLS - 1) / C::COLS;
            const int kpadc = nch * C::COLS;
            const int kb = 32 - __clz(kpadc - 1);
            const uint32_t imask = (1u << kb) - 1u;
            const int pos = (i - pre[h]) * C::ITEM_ROWS + et * C::ROWS + row;
            const bool live = pos < s.nrows;
            float xn = 0.f;
            if (live) {
                const int tok = p.rows ? p.rows[(size_t)h * p.N + pos] : pos;
                xn = (float)(p.norm[(size_t)h * p.N + tok] * (1.0 + 1e-6));
            }
            const float sigma = (p.mode == MODE_EUCLID) ? xn * xn : xn;
            const float *cnh = q.cnp + (size_t)h * p.kpad;
            float b1[4], b2[4], b3[4];
#pragma unroll
            for (int r = 0; r < 4; r++) b1[r] = b2[r] = b3[r] = INFINITY;
            for (int j = 0; j < nch; j++) {
                const int b = (int)(dc & 1);
                if (!mbar_wait_warp(d_full + b, (dc >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int pc = 0; pc < C::COLS / 32; pc++) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_addr + (uint32_t)((b * C::TILES + et) * C::COLS + pc * 32), r);
                    const int c0 = j * C::COLS + pc * 32;
                    const float4 *cn4 = reinterpret_cast<const float4 *>(cnh + c0);
#pragma unroll
                    for (int i8 = 0; i8 < 4; i8++) {
                        const float4 ca = __ldg(cn4 + 2 * i8), cb = __ldg(cn4 + 2 * i8 + 1);
                        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                        float key[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            const float d = __fadd_rn(fmaf(wv, __uint_as_float(r[8 * i8 + e]), cc[e]), sigma);
                            // the column index (< kpadc <= 2^kb) in the low kb bits
                            key[e] = __uint_as_float((__float_as_uint(d) & ~imask) | (uint32_t)(c0 + 8 * i8 + e));
                        }
#pragma unroll
                        for (int r4 = 0; r4 < 4; r4++) {
                            const float lo = fminf(key[2 * r4], key[2 * r4 + 1]);
                            const float hi = fmaxf(key[2 * r4], key[2 * r4 + 1]);
                            const float m11 = fmaxf(b1[r4], lo), m21 = fmaxf(b2[r4], lo), m12 = fmaxf(b1[r4], hi);
                            b3[r4] = fmin3(b3[r4], m21, m12);
                            b2[r4] = fmin3(b2[r4], m11, hi);
                            b1[r4] = fminf(b1[r4], lo);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(d_empty + b);
                dc++;
            }
            if (!ok) break;
            float B1 = b1[0], B2 = b2[0], B3 = b3[0];
#pragma unroll
            for (int r4 = 1; r4 < 4; r4++) {
                const float a1 = B1, a2 = B2, a3 = B3;
                B1 = fminf(a1, b1[r4]);
                B2 = fmin3(a2, b2[r4], fmaxf(a1, b1[r4]));
                B3 = fminf(fmin3(a3, b3[r4], fmaxf(a2, b1[r4])), fmaxf(a1, b2[r4]));
            }
            const int i1v = (int)(__float_as_uint(B1) & imask), i2v = (int)(__float_as_uint(B2) & imask);
            if (live) {
                const float cm = p.cmax[h];
                const float edot = 1.220703125e-4f * xn * cm;  // 2^-13 ||x|| Cmax
                const float E = ((p.mode == MODE_EUCLID) ? 2.f * edot + 2.384185791e-7f * (cm * cm + 2.f * xn * cm)
                                                          : edot) +
                                0x1p-100f;
                const float rho = __uint_as_float((uint32_t)(127 + kb - 22) << 23);
                const bool decided = B2 - B1 > 2.f * E + rho * (fabsf(B1) + fabsf(B2)) && i1v < s.k;
                if (s.k > 1 && !decided) {
                    const bool two = B3 - B1 > 2.f * E + rho * (fabsf(B1) + fabsf(B3)) && i1v < s.k && i2v < s.k;
                    const int slot = atomicAdd(&p.amb_count[h], 1);
                    p.amb_list[(size_t)h * p.N + slot] = pos;
                    p.amb_cand[(size_t)h * p.N + slot] = two ? make_int2(i1v, i2v) : make_int2(-1, -1);
                } else {
                    p.assign[(size_t)h * p.N + pos] = i1v;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// C_hi / C_lo (bf16, [H, kpad, D], zero rows beyond k), ||c||^2 (fp32 of a
// double sum) and max ||c|| (rounded up) for the centroids of the pass.
template <int D>
__global__ void cent_split_kernel(const float *__restrict__ cent, int cap, int kpad, const HeadSeg *__restrict__ seg,
                                  __nv_bfloat16 *__restrict__ chi, __nv_bfloat16 *__restrict__ clo,
                                  float *__restrict__ cn2, float *__restrict__ cnp, int mode) {
    // one warp per centroid row: coalesced split, ||c||^2 from a double sum
    const int h = blockIdx.y;
    const HeadSeg s = seg[h];
    const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (j >= kpad) return;
    __nv_bfloat16 *ph = chi + ((size_t)h * kpad + j) * D;
    __nv_bfloat16 *pl = clo + ((size_t)h * kpad + j) * D;
    double ss = 0.0;
    for (int t = lane; t < D; t += 32) {
        float v = 0.f;
        if (j < s.k) v = cent[((size_t)h * cap + s.cent_off + j) * D + t];
        const __nv_bfloat16 vh = __float2bfloat16_rn(v);
        ph[t] = vh;
        pl[t] = __float2bfloat16_rn(v - __bfloat162float(vh));
        ss += (double)v * (double)v;
    }
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0 && j < s.k) cn2[(size_t)h * cap + j] = (float)ss;
    // the column shift of the persistent screen: ||c||^2 (EUCLID) or 0 (SPHERE)
    // for the pass's centroids, a large finite score for the padding columns
    if (cnp && lane == 0) cnp[(size_t)h * kpad + j] = j >= s.k ? 1e30f : (mode == MODE_EUCLID ? (float)ss : 0.f);
}

// max_j ||c_j|| (rounded up) per head, from the ||c||^2 just written.
__global__ void cent_max_kernel(int cap, const HeadSeg *__restrict__ seg, const float *__restrict__ cn2,
                                float *__restrict__ cmax) {
    __shared__ float red[32];
    const int h = blockIdx.x;
    const HeadSeg s = seg[h];
    float mx = 0.f;
    for (int j = threadIdx.x; j < s.k; j += blockDim.x) mx = fmaxf(mx, cn2[(size_t)h * cap + j]);
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) m = fmaxf(m, red[w]);
        cmax[h] = (float)(sqrt((double)m) * (1.0 + 1e-5));
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int bf16_map(EncodeTiledFn enc, CUtensorMap *m, const void *base, int rows, int cols, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? 0
               : -1;
}

template <int D>
static int launch_tc(const void *xc, int H, int N, const int32_t *rows, const HeadSeg *seg, int nrows_max,
                     const float *cent, int cap, int kpad, void *chi, void *clo, float *cn2, float *cmax,
                     const double *norm, int mode, int32_t *assign, int32_t *amb_list, int32_t *amb_count,
                     int2 *amb_cand, int *status, void *encode_fn, float *cnp, int num_sms, cudaStream_t st) {
    using C = TcCfg<D>;
    using C2 = Tc2Cfg<D>;
    // the persistent screen whenever its item table holds every head
    const bool persistent = cnp && H <= C2::MAX_H && num_sms > 0;
    EncodeTiledFn enc = (EncodeTiledFn)encode_fn;
    cent_split_kernel<D><<<dim3(kpad / 8, H), 256, 0, st>>>(cent, cap, kpad, seg, (__nv_bfloat16 *)chi,
                                                            (__nv_bfloat16 *)clo, cn2, persistent ? cnp : nullptr, mode);
    note_launch();
    cent_max_kernel<<<H, 256, 0, st>>>(cap, seg, cn2, cmax);
    note_launch();
    CUtensorMap mx, mh, ml;
    if (bf16_map(enc, &mx, xc, H * N, D, C::ROWS) || bf16_map(enc, &mh, chi, H * kpad, D, C::COLS) ||
        bf16_map(enc, &ml, clo, H * kpad, D, C::COLS))
        return -1;
    if (kpad > 8192) return -1;
    if (persistent) {
        if (cudaFuncSetAttribute(assign_tc2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C2::SMEM) !=
            cudaSuccess)
            return -1;
        Tc2Params q;
        q.p.N = N;
        q.p.cap = cap;
        q.p.kpad = kpad;
        q.p.rows = rows;
        q.p.seg = seg;
        q.p.cn2 = cn2;
        q.p.cmax = cmax;
        q.p.norm = norm;
        q.p.mode = mode;
        q.p.assign = assign;
        q.p.amb_list = amb_list;
        q.p.amb_count = amb_count;
        q.p.amb_cand = amb_cand;
        q.p.status = status;
        q.cnp = cnp;
        q.H = H;
        const long long items = (long long)H * ((nrows_max + C2::ITEM_ROWS - 1) / C2::ITEM_ROWS);
        const int grid = (int)(items < num_sms ? (items > 0 ? items : 1) : num_sms);
        assign_tc2_kernel<D><<<grid, C2::NTHREADS, C2::SMEM, st>>>(mx, mh, ml, q);
        note_launch();
        return 0;
    }
    // the attribute belongs to the current device: set it on every call
    cudaFuncSetAttribute(assign_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::smem_bytes(8192));
    TcParams p;
    p.N = N;
    p.cap = cap;
    p.kpad = kpad;
    p.rows = rows;
    p.seg = seg;
    p.cn2 = cn2;
    p.cmax = cmax;
    p.norm = norm;
    p.mode = mode;
    p.assign = assign;
    p.amb_list = amb_list;
    p.amb_count = amb_count;
    p.amb_cand = amb_cand;
    p.status = status;
    dim3 g((nrows_max + C::ROWS - 1) / C::ROWS, H);
    assign_tc_kernel<D><<<g, 192, C::smem_bytes(kpad), st>>>(mx, mh, ml, p);
    note_launch();
    return 0;
}

int k_assign_tc(const void *xc, int H, int N, int D, const int32_t *rows, const HeadSeg *seg, int nrows_max,
                const float *cent, int cap, int kpad, void *chi, void *clo, float *cn2, float *cmax,
                const double *norm, int mode, int32_t *assign, int32_t *amb_list, int32_t *amb_count, int2 *amb_cand,
                int *status, void *encode_fn, float *cnp, int num_sms, cudaStream_t st) {
    if (D == 64)
        return launch_tc<64>(xc, H, N, rows, seg, nrows_max, cent, cap, kpad, chi, clo, cn2, cmax, norm, mode, assign,
                             amb_list, amb_count, amb_cand, status, encode_fn, cnp, num_sms, st);
    return launch_tc<128>(xc, H, N, rows, seg, nrows_max, cent, cap, kpad, chi, clo, cn2, cmax, norm, mode, assign,
                          amb_list, amb_count, amb_cand, status, encode_fn, cnp, num_sms, st);
}

}  // namespace ac
