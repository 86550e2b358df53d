// Block-sparse exact softmax attention over selected key clusters (AdaCluster,
// Algorithm 3's sparse attention; its dense branch for dense heads) on sm_100a tensor cores.
//
// Inputs are gathered into cluster order (ac_sort.cu): the rows of query
// cluster a are contiguous in Qg, the keys/values of key cluster b contiguous
// in Kg/Vg.  A work item is one tile of up to 128 query rows of one query
// cluster (or of a dense head); it walks the key rows of every selected key
// cluster in chunks of up to BN rows.
//
// Per CTA (persistent, one per SM): warp 0 issues TMA loads (Q tile once per
// item, K/V chunks into a 2-stage ring, 32-row boxes so a short cluster tail
// costs only the rows it needs); lane 0 of warp 1 issues tcgen05.mma:
// S = Q K^T into one of two TMEM buffers, O += P V into a TMEM accumulator;
// warps 2-5 (one thread per query row = TMEM lane) run the online softmax
// from TMEM, write P (bf16, or tf32 for fp32 inputs) to shared memory in the
// 128-byte-swizzled K-major layout, and do the epilogue (O / l, scatter rows
// back to token order).  The running max is only moved (and O rescaled in
// TMEM) when it grows by more than 2^8, so most chunks skip the rescale.
// Every mbarrier wait is bounded; on expiry the CTA records ST_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include "ac_kernels.cuh"

namespace ac {

template <typename T, int D> struct AttnCfg {
    static constexpr int ELT = sizeof(T);
    static constexpr int BM = 128;
    static constexpr int BN = (ELT == 4 && D == 128) ? 64 : 128;
    static constexpr int EPR = 128 / ELT;          // elements per 128-byte swizzle row
    static constexpr int DB = D / EPR;             // 128-byte column blocks of a Q/K/V row
    static constexpr int KSTEP = 32 / ELT;         // K of one MMA instruction
    static constexpr int BOX = 32;                 // rows per K/V TMA box
    static constexpr int NPB = ELT == 2 ? 2 : 1;   // P buffers (double-buffered for bf16)
    static constexpr int SM_WARPS = 4;             // softmax warps: one per TMEM lane quarter
    static constexpr int NTHREADS = (2 + SM_WARPS) * 32;
    static constexpr int Q_BYTES = BM * D * ELT;
    static constexpr int KV_BYTES = BN * D * ELT;  // one stage of K (or of V)
    static constexpr int P_BYTES = BM * BN * ELT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;
    static constexpr int OFF_P = OFF_V + 2 * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + NPB * P_BYTES;
    // + alignment slack; at least 116 KB so that two CTAs never share an SM
    // (each allocates all 512 TMEM columns)
    static constexpr int SMEM_RAW = OFF_BAR + 256 + 1024;
    static constexpr int SMEM = SMEM_RAW > 116 * 1024 ? SMEM_RAW : 116 * 1024;
    static constexpr int FMT = (ELT == 2) ? 1 : 2;     // bf16 / tf32
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int TM_S0 = 0, TM_S1 = BN, TM_O = 2 * BN;
    static_assert(TM_O + D <= (int)TMEM_COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct AttnParams {
    int H, N;
    const int32_t *qperm;
    int kk_cap, kq_cap;
    const int2 *runs;      // per (head, query cluster): ascending key-row runs
    const int2 *run_info;  // per (head, query cluster): {runs, chunks}
    const AttnItem *items;
    const int32_t *n_items;
    void *out;
    float *lse;
    int *status;
    float scale_log2;
};

// Walks the key chunks of one work item: the rows of every key run (selected
// key clusters, neighbours merged; all rows [0, N) for a dense head) in pieces
// of <= BN.
struct ChunkIter {
    const int2 *seg;
    int nsel, si, cur, end, bn, dense_n;
    int2 nxt;
    __device__ void init(const AttnParams &p, const AttnItem &it) {
        if (it.a < 0) {
            seg = nullptr;
            nsel = 1;
        } else {
            seg = p.runs + ((size_t)it.h * p.kq_cap + it.a) * p.kk_cap;
            nsel = p.run_info[(size_t)it.h * p.kq_cap + it.a].x;
        }
        si = -1;
        cur = end = 0;
        dense_n = p.N;
        nxt = (seg && nsel > 0) ? seg[0] : make_int2(0, p.N);
    }
    __device__ bool next(int &start, int &len) {
        while (cur >= end) {
            if (++si >= nsel) return false;
            cur = nxt.x;
            end = nxt.y;
            if (seg && si + 1 < nsel) nxt = seg[si + 1];  // one segment ahead
        }
        start = cur;
        len = min(bn, end - cur);
        cur += len;
        return true;
    }
    __device__ int count(const AttnParams &p, const AttnItem &it) {
        init(p, it);
        int n = 0, s, l;
        while (next(s, l)) n++;
        init(p, it);
        return n;
    }
};

__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status) {
    bool ok = mbar_wait(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain own copies / MMAs).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    uint64_t t0 = gtimer();
    while (!mbar_try_wait(bar, parity)) {
        if (gtimer() - t0 > 200000000ull) break;
    }
}

// 2^x on the FMA pipe: x = n + f with n = rint(x) (magic-constant add),
// f in [-1/2, 1/2]; 2^f by a cubic fitted (relative-error minimax on
// Chebyshev nodes) to |rel err| < 7.5e-5, well below the bf16/tf32 rounding
// P goes through; then n is added to the exponent.  x is clamped at -125.
__device__ __forceinline__ float ex2_poly(float x) {
    x = fmaxf(x, -125.f);
    const float t = x + 12582912.0f;                  // 1.5 * 2^23: t - 1.5*2^23 = rint(x)
    const int n = __float_as_int(t) - 0x4B400000;
    const float f = x - (t - 12582912.0f);
    float p = fmaf(0.0551716648042202f, f, 0.2426111251115799f);
    p = fmaf(p, f, 0.6932609677314758f);
    p = fmaf(p, f, 0.9999280571937561f);
    return __int_as_float(__float_as_int(p) + (n << 23));
}

template <typename T, int D>
__global__ void __launch_bounds__(AttnCfg<T, D>::NTHREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = AttnCfg<T, D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_full = bars + 0, *q_empty = bars + 1;
    uint64_t *k_full = bars + 2, *v_full = bars + 4, *k_empty = bars + 6, *v_empty = bars + 20;
    uint64_t *s_full = bars + 8, *s_empty = bars + 10;
    uint64_t *p_full = bars + 12, *pv_done = bars + 14, *o_free = bars + 16, *drain = bars + 17;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 18);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 19);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t NSM = C::SM_WARPS * 32;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; i++) {
            mbar_init(k_full + i, 1);
            mbar_init(v_full + i, 1);
            mbar_init(k_empty + i, 1);
            mbar_init(v_empty + i, 1);
            mbar_init(s_full + i, 1);
            mbar_init(s_empty + i, NSM);
            mbar_init(p_full + i, NSM);
            mbar_init(pv_done + i, 1);
        }
        mbar_init(o_free, NSM);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = *p.n_items;

    if (warp == 0) {
        // ------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t g = 0, qi = 0;
            int last_kv[2] = {-1, -1};
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const AttnItem it = p.items[item];
                ChunkIter ci;
                ci.bn = C::BN;
                if (ci.count(p, it) == 0) continue;
                if (qi >= 1 && !mbar_wait(q_empty, (qi - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx(q_full, C::Q_BYTES);
                const int qrow = it.h * p.N + it.q_start;
                for (int kb = 0; kb < C::DB; kb++)
                    tma_load_2d(sm + C::OFF_Q + kb * (C::BM * 128), &tmQ, q_full, kb * C::EPR, qrow);
                qi++;
                int start, len;
                while (ci.next(start, len)) {
                    const int st = g & 1;
                    const uint32_t u = g >> 1;
                    // K of stage st is free once S of its previous chunk is done,
                    // V once that chunk's P.V is done
                    if (u >= 1 && !mbar_wait(k_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    const int nb = (len + C::BOX - 1) / C::BOX;
                    const uint32_t bytes = (uint32_t)nb * C::BOX * 128 * C::DB;
                    const int krow = it.h * p.N + start;
                    mbar_arrive_expect_tx(k_full + st, bytes);
                    for (int kb = 0; kb < C::DB; kb++)
                        for (int b = 0; b < nb; b++)
                            tma_load_2d(sm + C::OFF_K + st * C::KV_BYTES + kb * (C::BN * 128) + b * (C::BOX * 128),
                                        &tmK, k_full + st, kb * C::EPR, krow + b * C::BOX);
                    if (u >= 1 && !mbar_wait(v_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(v_full + st, bytes);
                    for (int kb = 0; kb < C::DB; kb++)
                        for (int b = 0; b < nb; b++)
                            tma_load_2d(sm + C::OFF_V + st * C::KV_BYTES + kb * (C::BN * 128) + b * (C::BOX * 128),
                                        &tmV, v_full + st, kb * C::EPR, krow + b * C::BOX);
                    last_kv[st] = (int)u;
                    g++;
                }
            }
            if (!ok) {
                if (qi >= 1) drain_wait(q_full, (qi - 1) & 1);
                for (int st = 0; st < 2; st++)
                    if (last_kv[st] >= 0) {
                        drain_wait(k_full + st, last_kv[st] & 1);
                        drain_wait(v_full + st, last_kv[st] & 1);
                    }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_o = idesc_make(128, D, C::FMT, true);
            uint32_t g = 0, qi = 0;
            bool ok = true;
            // O += P_gp V_gp; P from buffer gp % NPB, V from stage gp % 2
            auto issue_pv = [&](uint32_t gp, int lenp, bool first) -> bool {
                const int pb = gp % C::NPB;
                if (!mbar_wait(p_full + pb, (gp / C::NPB) & 1, abort_flag, p.status)) return false;
                if (!mbar_wait(v_full + (gp & 1), (gp >> 1) & 1, abort_flag, p.status)) return false;
                if (first && qi >= 2 && !mbar_wait(o_free, (qi - 2) & 1, abort_flag, p.status)) return false;
                tc_fence_after();
                const int np = (lenp + 31) & ~31;
                const uint32_t vbase = smem_u32(sm + C::OFF_V + (gp & 1) * C::KV_BYTES);
                const uint32_t pbase = smem_u32(sm + C::OFF_P + pb * C::P_BYTES);
                for (int ks = 0; ks < np / C::KSTEP; ks++) {
                    const int kofs = ks * C::KSTEP;
                    const uint64_t a = sdesc_sw128(pbase + (kofs / C::EPR) * (C::BM * 128) + (kofs % C::EPR) * C::ELT,
                                                   16, 1024);
                    // V is MN-major (d contiguous): 128-byte blocks along d at
                    // LBO; 8-row (bf16) or 4-row (tf32, 32-byte atoms) K groups at SBO
                    const uint64_t b = sdesc_make(vbase + kofs * 128, C::BN * 128, C::ELT == 2 ? 1024 : 512,
                                                  C::ELT == 2 ? 2u : 1u);
                    if (C::FMT == 1) umma_f16(tmem + C::TM_O, a, b, idesc_o, (!first || ks > 0) ? 1u : 0u);
                    else umma_tf32(tmem + C::TM_O, a, b, idesc_o, (!first || ks > 0) ? 1u : 0u);
                }
                umma_commit(pv_done + pb);
                umma_commit(v_empty + (gp & 1));
                return true;
            };
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const AttnItem it = p.items[item];
                ChunkIter ci;
                ci.bn = C::BN;
                const int nch = ci.count(p, it);
                if (nch == 0) continue;
                if (!mbar_wait(q_full, qi & 1, abort_flag, p.status)) { ok = false; break; }
                qi++;
                int start, len, c = 0, prev_len = 0;
                while (ci.next(start, len)) {
                    const int st = g & 1;
                    const uint32_t u = g >> 1;
                    if (!mbar_wait(k_full + st, u & 1, abort_flag, p.status)) { ok = false; break; }
                    if (u >= 1 && !mbar_wait(s_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const int ncol = (len + 31) & ~31;
                    const uint32_t idesc_s = idesc_make(128, ncol, C::FMT, false);
                    const uint32_t qbase = smem_u32(sm + C::OFF_Q);
                    const uint32_t kbase = smem_u32(sm + C::OFF_K + st * C::KV_BYTES);
                    const uint32_t dS = tmem + (st ? C::TM_S1 : C::TM_S0);
                    for (int ks = 0; ks < D / C::KSTEP; ks++) {
                        const int kofs = ks * C::KSTEP;
                        const uint32_t boff = (kofs % C::EPR) * C::ELT;
                        const uint64_t a = sdesc_sw128(qbase + (kofs / C::EPR) * (C::BM * 128) + boff, 16, 1024);
                        const uint64_t b = sdesc_sw128(kbase + (kofs / C::EPR) * (C::BN * 128) + boff, 16, 1024);
                        if (C::FMT == 1) umma_f16(dS, a, b, idesc_s, ks > 0 ? 1u : 0u);
                        else umma_tf32(dS, a, b, idesc_s, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(s_full + st);
                    umma_commit(k_empty + st);
                    if (c == nch - 1) umma_commit(q_empty);
                    if (c > 0 && !issue_pv(g - 1, prev_len, c == 1)) { ok = false; break; }
                    prev_len = len;
                    c++;
                    g++;
                }
                if (!ok) break;
                if (!issue_pv(g - 1, prev_len, nch == 1)) { ok = false; break; }
            }
            if (!ok) {
                umma_commit(drain);
                drain_wait(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        // One thread per query row (= TMEM lane).  Each chunk's scores come out
        // of TMEM in one wide load; the S buffer is released right away, P goes
        // to the buffer whose previous P.V has completed.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        uint32_t g = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const AttnItem it = p.items[item];
            ChunkIter ci;
            ci.bn = C::BN;
            const int nch = ci.count(p, it);
            float m_ref = -INFINITY, l = 0.f;
            int start, len, c = 0;
            while (nch > 0 && ci.next(start, len)) {
                const int st = g & 1;
                const uint32_t u = g >> 1;
                if (!wait_all(s_full + st, u & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[C::BN];
                if (C::BN == 128) tmem_ld128(tmem + lane_addr + (st ? C::TM_S1 : C::TM_S0), *reinterpret_cast<uint32_t (*)[128]>(sr));
                else tmem_ld64(tmem + lane_addr + (st ? C::TM_S1 : C::TM_S0), *reinterpret_cast<uint32_t (*)[64]>(sr));
                tc_fence_before();
                mbar_arrive(s_empty + st);
                // columns past the chunk's keys (rounded up to 32) do not count
                if (len < C::BN) {
#pragma unroll
                    for (int i = 0; i < C::BN; i++)
                        if (i >= len) sr[i] = __float_as_uint(-INFINITY);
                }
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < C::BN; i++) mx = fmaxf(mx, __uint_as_float(sr[i]));
                const float m_new = mx * p.scale_log2;
                if (c == 0) m_ref = m_new;
                // Move the reference max (and rescale O) only when it grew by
                // more than 2^8.  The TMEM accesses are warp-collective, so the
                // decision is per warp; rows that did not grow use f = 1.
                if (c > 0 && __any_sync(0xffffffffu, m_new > m_ref + 8.f)) {
                    const uint32_t gq = g - 1;
                    if (!wait_all(pv_done + gq % C::NPB, (gq / C::NPB) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const float m_to = fmaxf(m_ref, m_new);
                    const float f = ex2_approx(m_ref - m_to);
                    l *= f;
#pragma unroll
                    for (int pc = 0; pc < D / 32; pc++) {
                        uint32_t r[32];
                        const uint32_t oa = tmem + lane_addr + C::TM_O + pc * 32;
                        tmem_ld32(oa, r);
#pragma unroll
                        for (int i = 0; i < 32; i++) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                        tmem_st32(oa, r);
                    }
                    tmem_st_wait();
                    m_ref = m_to;
                }
                // P buffer g % NPB is free once the P.V of its previous use is done
                const int pb = g % C::NPB;
                const uint32_t pu = g / C::NPB;
                if (pu >= 1 && !wait_all(pv_done + pb, (pu - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                unsigned char *prow = sm + C::OFF_P + pb * C::P_BYTES + row * 128;
                const int npc = (len + 31) >> 5;
#pragma unroll
                for (int pc = 0; pc < C::BN / 32; pc++) {
                    if (pc < npc) {
                        float pv[32];
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const float x = fmaf(__uint_as_float(sr[pc * 32 + i]), p.scale_log2, -m_ref);
                            pv[i] = (i & 3) == 3 ? ex2_poly(x) : ex2_approx(x);
                            l += pv[i];
                        }
                        if (C::ELT == 2) {
                            const int kb = (pc * 32) / C::EPR;
                            const int ch0 = ((pc * 32) % C::EPR) / 8;
#pragma unroll
                            for (int q4 = 0; q4 < 4; q4++) {
                                uint32_t w[4];
#pragma unroll
                                for (int e2 = 0; e2 < 4; e2++) {
                                    __nv_bfloat162 b2 = __floats2bfloat162_rn(pv[q4 * 8 + e2 * 2], pv[q4 * 8 + e2 * 2 + 1]);
                                    w[e2] = *reinterpret_cast<uint32_t *>(&b2);
                                }
                                const int chunk = (ch0 + q4) ^ (row & 7);
                                *reinterpret_cast<uint4 *>(prow + kb * (C::BM * 128) + chunk * 16) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        } else {
                            const int kb = pc;
#pragma unroll
                            for (int q4 = 0; q4 < 8; q4++) {
                                uint32_t w[4];
#pragma unroll
                                for (int e2 = 0; e2 < 4; e2++) {
                                    uint32_t tf;
                                    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(tf) : "f"(pv[q4 * 4 + e2]));
                                    w[e2] = tf;
                                }
                                const int chunk = q4 ^ (row & 7);
                                *reinterpret_cast<uint4 *>(prow + kb * (C::BM * 128) + chunk * 16) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                    }
                }
                tc_fence_before();          // orders a rescale's tcgen05.st before the P.V
                fence_proxy_async_smem();   // P (generic stores) visible to the MMA
                mbar_arrive(p_full + pb);
                c++;
                g++;
            }
            if (!ok) break;
            // epilogue: out row = O / l, scattered back to token order
            const bool valid = row < it.q_len;
            int tok = 0;
            if (valid) tok = p.qperm[(size_t)it.h * p.N + it.q_start + row];
            const size_t orow = ((size_t)it.h * p.N + tok) * D;
            if (nch > 0) {
                const uint32_t gq = g - 1;
                if (!wait_all(pv_done + gq % C::NPB, (gq / C::NPB) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                const float inv = 1.f / l;
#pragma unroll
                for (int pc = 0; pc < D / 32; pc++) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_addr + C::TM_O + pc * 32, r);
                    if (valid) {
                        if (C::ELT == 2) {
                            uint32_t w[16];
#pragma unroll
                            for (int i = 0; i < 16; i++) {
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * inv,
                                                                          __uint_as_float(r[2 * i + 1]) * inv);
                                w[i] = *reinterpret_cast<uint32_t *>(&b2);
                            }
                            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.out) + orow + pc * 32);
#pragma unroll
                            for (int i = 0; i < 4; i++) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + orow + pc * 32);
#pragma unroll
                            for (int i = 0; i < 8; i++)
                                dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                                     __uint_as_float(r[4 * i + 2]) * inv,
                                                     __uint_as_float(r[4 * i + 3]) * inv);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(o_free);
                if (valid && p.lse) p.lse[(size_t)it.h * p.N + tok] = (m_ref + __log2f(l)) * 0.69314718055994531f;
            } else if (valid) {
                for (int t = 0; t < D; t++) {
                    if (C::ELT == 2) reinterpret_cast<__nv_bfloat16 *>(p.out)[orow + t] = __float2bfloat16(0.f);
                    else reinterpret_cast<float *>(p.out)[orow + t] = 0.f;
                }
                if (p.lse) p.lse[(size_t)it.h * p.N + tok] = -INFINITY;
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

// ------------------------------------------------------------ work items
// Work items are query tiles of 128 rows per non-empty query cluster (or over
// all rows of a dense head).  Three launches: per head, tile counts and their
// exclusive scan plus the head's (query, key) pairs; across heads, the bases;
// per (cluster, head), the items themselves.
__global__ void items_count_kernel(int N, int rpi, int kq_cap, int kk_cap, const int32_t *__restrict__ qoff,
                                   const int32_t *__restrict__ nq, const uint8_t *__restrict__ dense, int kq_fixed,
                                   const int32_t *__restrict__ koff, const int32_t *__restrict__ sel_idx,
                                   const int32_t *__restrict__ sel_cnt, int32_t *__restrict__ tile_off,
                                   int32_t *__restrict__ head_tiles, unsigned long long *__restrict__ head_pairs,
                                   int *status) {
    __shared__ int wsum[32];
    __shared__ int carry;
    __shared__ unsigned long long pacc;
    const int h = blockIdx.x, tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, w = tid >> 5;
    const bool dn = dense && dense[h];
    // counts from caller memory are clamped to the capacities (ST_INVALID if not within)
    const int nqh = dn ? 1 : (nq ? clamp_count(nq[h], kq_cap, tid == 0 ? status : nullptr) : kq_fixed);
    const int32_t *qo = qoff + (size_t)h * (kq_cap + 1);
    const int32_t *ko = koff + (size_t)h * (kk_cap + 1);
    int32_t *to = tile_off + (size_t)h * (kq_cap + 1);
    if (tid == 0) { carry = 0; pacc = 0ull; }
    __syncthreads();
    for (int a0 = 0; a0 < nqh; a0 += nt) {
        const int a = a0 + tid;
        int tiles = 0;
        if (a < nqh) {
            const int qn = dn ? N : qo[a + 1] - qo[a];
            tiles = (qn + rpi - 1) / rpi;
            unsigned long long pr = 0ull;
            if (dn) {
                pr = (unsigned long long)N * (unsigned long long)N;
            } else if (qn > 0) {
                long long keys = 0;
                const int32_t *sl = sel_idx + ((size_t)h * kq_cap + a) * kk_cap;
                const int ns = clamp_count(sel_cnt[(size_t)h * kq_cap + a], kk_cap, status);
                for (int c = 0; c < ns; c++) {
                    const int b = sl[c];
                    if (b >= 0 && b < kk_cap) keys += ko[b + 1] - ko[b];
                }
                pr = (unsigned long long)(keys * qn);
            }
            atomicAdd(&pacc, pr);
        }
        int x = tiles;
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) wsum[w] = x;
        __syncthreads();
        if (w == 0) {
            int t = lane < nt / 32 ? wsum[lane] : 0;
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, d);
                if (lane >= d) t += y;
            }
            if (lane < nt / 32) wsum[lane] = t;
        }
        __syncthreads();
        if (a < nqh) to[a] = carry + x - tiles + (w > 0 ? wsum[w - 1] : 0);
        __syncthreads();
        if (tid == 0) carry += wsum[nt / 32 - 1];
        __syncthreads();
    }
    if (tid == 0) {
        to[nqh] = carry;
        head_tiles[h] = carry;
        head_pairs[h] = pacc;
    }
}

__global__ void items_base_kernel(int H, const int32_t *__restrict__ head_tiles,
                                  const unsigned long long *__restrict__ head_pairs, int32_t *__restrict__ head_base,
                                  int32_t *__restrict__ n_items, int64_t *__restrict__ pairs) {
    if (threadIdx.x != 0) return;
    int base = 0;
    unsigned long long pr = 0ull;
    for (int h = 0; h < H; h++) {
        head_base[h] = base;
        base += head_tiles[h];
        pr += head_pairs[h];
    }
    n_items[0] = base;
    n_items[1] = 0;  // work counter of the dynamically scheduled attention kernel
    if (pairs) *pairs = (int64_t)pr;
}

__global__ void items_write_kernel(int N, int rpi, int kq_cap, const int32_t *__restrict__ qoff, const int32_t *__restrict__ nq,
                                   const uint8_t *__restrict__ dense, int kq_fixed, const int32_t *__restrict__ tile_off,
                                   const int32_t *__restrict__ head_base, AttnItem *__restrict__ items) {
    const int h = blockIdx.y;
    const int a = blockIdx.x * blockDim.x + threadIdx.x;
    const bool dn = dense && dense[h];
    const int nqh = dn ? 1 : (nq ? clamp_count(nq[h], kq_cap, nullptr) : kq_fixed);
    if (a >= nqh) return;
    const int32_t *qo = qoff + (size_t)h * (kq_cap + 1);
    const int qs = dn ? 0 : qo[a];
    const int qn = dn ? N : qo[a + 1] - qs;
    const int base = head_base[h] + tile_off[(size_t)h * (kq_cap + 1) + a];
    for (int t = 0; t * rpi < qn; t++) {
        AttnItem itm;
        itm.h = h;
        itm.a = dn ? -1 : a;
        itm.q_start = qs + t * rpi;
        itm.q_len = min(rpi, qn - t * rpi);
        items[base + t] = itm;
    }
}

// Key runs of query cluster a of head h (one CTA each).  A bit set over the
// key clusters marks the selected ones and the empty ones; each maximal run of
// marked clusters b0..b1 becomes the row range [koff[b0], koff[b1+1]) of the
// gathered K/V, in ascending order.  A run of empty clusters only has no rows
// (the key stream skips it).  Every run's last piece is rounded up to 8 rows
// and every chunk but the last is full, so the chunk count of KeyStream is
// ceil(sum of rows rounded up to 8 / chunk_rows).
constexpr int kRunWords = 8192 / 32;  // key-cluster capacity is at most 8192

__device__ __forceinline__ int run_last(const uint32_t *m, int nw, int b) {
    int w = b >> 5;
    uint32_t z = ~m[w] & (~0u << (b & 31));  // unmarked clusters at or after b
    while (z == 0) {
        if (++w >= nw) return nw * 32 - 1;
        z = ~m[w];
    }
    return w * 32 + __ffs(z) - 2;
}

__global__ void key_runs_kernel(int kq_cap, int kk_cap, const int32_t *__restrict__ koff,
                                const int32_t *__restrict__ sel_idx, const int32_t *__restrict__ sel_cnt,
                                int chunk_rows, int2 *__restrict__ runs, int2 *__restrict__ info) {
    __shared__ uint32_t m[kRunWords];
    __shared__ int pre[kRunWords];
    __shared__ int n_runs;
    __shared__ unsigned long long slot_rows;
    const int h = blockIdx.y, a = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int nw = (kk_cap + 31) >> 5;
    const int32_t *ko = koff + (size_t)h * (kk_cap + 1);
    const int32_t *sl = sel_idx + ((size_t)h * kq_cap + a) * kk_cap;
    const int n = min(sel_cnt[(size_t)h * kq_cap + a], kk_cap);
    int2 *out = runs + ((size_t)h * kq_cap + a) * kk_cap;
    if (n <= 0) {
        if (tid == 0) info[(size_t)h * kq_cap + a] = make_int2(0, 0);
        return;
    }
    for (int w = tid; w < nw; w += nt) {
        uint32_t e = 0;
        for (int i = 0; i < 32; i++) {
            const int b = w * 32 + i;
            if (b < kk_cap && ko[b + 1] == ko[b]) e |= 1u << i;
        }
        m[w] = e;
    }
    if (tid == 0) slot_rows = 0ull;
    __syncthreads();
    for (int c = tid; c < n; c += nt) {
        const int b = sl[c];
        if (b >= 0 && b < kk_cap) atomicOr(&m[b >> 5], 1u << (b & 31));
    }
    __syncthreads();
    // run starts per word, exclusive prefix over words (warp 0, 8 words a lane)
    if (tid < 32) {
        int cnt[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int w = tid * 8 + i;
            int c = 0;
            if (w < nw) {
                const uint32_t prev = w > 0 ? m[w - 1] >> 31 : 0u;
                c = __popc(m[w] & ~((m[w] << 1) | prev));
            }
            cnt[i] = c;
            sum += c;
        }
        int x = sum;
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (tid >= d) x += y;
        }
        int base = x - sum;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int w = tid * 8 + i;
            if (w < kRunWords) pre[w] = base;
            base += cnt[i];
        }
        if (tid == 31) n_runs = x;
    }
    __syncthreads();
    unsigned long long my_rows = 0ull;
    for (int w = tid; w < nw; w += nt) {
        const uint32_t prev = w > 0 ? m[w - 1] >> 31 : 0u;
        uint32_t st = m[w] & ~((m[w] << 1) | prev);
        int k = pre[w];
        while (st) {
            const int b = w * 32 + __ffs(st) - 1;
            st &= st - 1;
            const int e = run_last(m, nw, b);
            const int r0 = ko[b], r1 = ko[e + 1];
            out[k++] = make_int2(r0, r1);
            my_rows += (unsigned long long)((r1 - r0 + 7) & ~7);
        }
    }
    if (my_rows) atomicAdd(&slot_rows, my_rows);
    __syncthreads();
    if (tid == 0)
        info[(size_t)h * kq_cap + a] =
            make_int2(n_runs, (int)((slot_rows + (unsigned long long)chunk_rows - 1) / (unsigned long long)chunk_rows));
}

void k_key_runs(int H, int kq_cap, int kk_cap, const int32_t *koff, const int32_t *sel_idx, const int32_t *sel_cnt,
                int chunk_rows, int2 *runs, int2 *info, cudaStream_t st) {
    key_runs_kernel<<<dim3(kq_cap, H), 128, 0, st>>>(kq_cap, kk_cap, koff, sel_idx, sel_cnt, chunk_rows, runs, info);
    note_launch();
}

// Chunk masks of every (head, query cluster): for chunk c of the key stream
// (CH keys as KeyStream packs the runs) the number of valid rows in each of
// its 8-row groups, 4 bits per group, eight groups per 32-bit word (CH / 64
// words per chunk, group g in word g / 8).  Run
// r occupies stream positions [S_r, S_r + round8(len_r)) with S_r the prefix
// sum of the rounded lengths, and its first len_r positions hold keys (a run
// split at a chunk boundary is split at a multiple of 8, so this holds for
// every piece).  One CTA per (query cluster, head): a block scan gives S, then
// each thread fills chunks with a binary search per group.
constexpr int kMaskMaxRuns = 8192;

template <int CH>
__global__ void chunk_masks_kernel(int kq_cap, int kk_cap, int max_chunks, const int2 *__restrict__ runs,
                                   const int2 *__restrict__ info, uint32_t *__restrict__ masks) {
    constexpr int W = CH / 64;
    __shared__ int s_start[kMaskMaxRuns];
    __shared__ int wsum[32];
    const int h = blockIdx.y, a = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const size_t qa = (size_t)h * kq_cap + a;
    const int2 inf = info[qa];
    const int nr = min(inf.x, kMaskMaxRuns), nch = min(inf.y, max_chunks);
    if (nch <= 0) return;
    const int2 *rr = runs + qa * kk_cap;
    // exclusive scan of the rounded run lengths (runs processed in blocks of nt)
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
        if (w == 0) {
            int t = lane < nt / 32 ? wsum[lane] : 0;
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, d);
                if (lane >= d) t += y;
            }
            if (lane < nt / 32) wsum[lane] = t;
        }
        __syncthreads();
        if (r < nr) s_start[r] = carry + x - len + (w > 0 ? wsum[w - 1] : 0);
        carry += wsum[nt / 32 - 1];
        __syncthreads();
    }
    uint32_t *out = masks + qa * max_chunks * W;
    for (int cw = tid; cw < nch * W; cw += nt) {
        uint32_t gm = 0;
#pragma unroll 1
        for (int g = 0; g < 8; g++) {
            const int pos = cw * 64 + 8 * g;
            // last run with S_r <= pos
            int lo = 0, hi = nr - 1, r = -1;
            while (lo <= hi) {
                const int mid = (lo + hi) >> 1;
                if (s_start[mid] <= pos) { r = mid; lo = mid + 1; }
                else hi = mid - 1;
            }
            if (r >= 0) {
                const int2 v = rr[r];
                const int left = s_start[r] + (v.y - v.x) - pos;
                gm |= (uint32_t)(left <= 0 ? 0 : (left >= 8 ? 8 : left)) << (4 * g);
            }
        }
        out[cw] = gm;
    }
}

int attn_max_chunks(int N, int kk_cap, int chunk) { return (N + 7 * kk_cap + chunk - 1) / chunk + 1; }

void k_chunk_masks(int H, int kq_cap, int kk_cap, int max_chunks, const int2 *runs, const int2 *info,
                   uint32_t *masks, cudaStream_t st) {
    chunk_masks_kernel<ATTN3_CHUNK><<<dim3(kq_cap, H), 256, 0, st>>>(kq_cap, kk_cap, max_chunks, runs, info, masks);
    note_launch();
}

int attn_max_items(int H, int N, int kq_cap) { return H * ((N + 127) / 128 + kq_cap); }

void k_build_items(int H, int N, int rows_per_item, int kq_cap, int kk_cap, const int32_t *qoff, const int32_t *nq,
                   const uint8_t *dense, int kq_fixed, const int32_t *koff, const int32_t *sel_idx,
                   const int32_t *sel_cnt, AttnItem *items, int32_t *n_items, int64_t *pairs, int32_t *scratch,
                   int *status, cudaStream_t st) {
    int32_t *tile_off = scratch;                                      // [H, kq_cap + 1]
    int32_t *head_tiles = tile_off + (size_t)H * (kq_cap + 1);         // [H]
    int32_t *head_base = head_tiles + H;                               // [H]
    unsigned long long *head_pairs =
        reinterpret_cast<unsigned long long *>(head_base + H + ((2 * H + (size_t)H * (kq_cap + 1)) & 1));  // [H]
    items_count_kernel<<<H, 512, 0, st>>>(N, rows_per_item, kq_cap, kk_cap, qoff, nq, dense, kq_fixed, koff, sel_idx, sel_cnt,
                                          tile_off, head_tiles, head_pairs, status);
    note_launch();
    items_base_kernel<<<1, 32, 0, st>>>(H, head_tiles, head_pairs, head_base, n_items, pairs);
    note_launch();
    items_write_kernel<<<dim3((kq_cap + 127) / 128, H), 128, 0, st>>>(N, rows_per_item, kq_cap, qoff, nq, dense, kq_fixed, tile_off,
                                                                      head_base, items);
    note_launch();
}

size_t items_scratch_elems(int H, int kq_cap) { return (size_t)H * (kq_cap + 1) + 2 * (size_t)H + 1 + 2 * (size_t)H; }

// ------------------------------------------------------------ launcher
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int make_map(EncodeTiledFn enc, CUtensorMap *m, const void *base, int elt, int rows, int cols, int box_rows,
                    CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * elt};
    cuuint32_t box[2] = {(cuuint32_t)(128 / elt), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, elt == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                     const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : -1;
}

template <typename T, int D>
static int launch_attn(const void *qg, const void *kg, const void *vg, const AttnParams &p, int max_items,
                       int num_sms, void *encode_fn, cudaStream_t st) {
    using C = AttnCfg<T, D>;
    EncodeTiledFn enc = (EncodeTiledFn)encode_fn;
    CUtensorMap mq, mk, mv;
    const int rows = p.H * p.N;
    if (make_map(enc, &mq, qg, C::ELT, rows, D, C::BM) || make_map(enc, &mk, kg, C::ELT, rows, D, C::BOX) ||
        make_map(enc, &mv, vg, C::ELT, rows, D, C::BOX,
                 C::ELT == 2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B))
        return -1;
    // the attribute belongs to the current device: set it on every call
    cudaFuncSetAttribute(attn_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    int grid = max_items < num_sms ? max_items : num_sms;
    if (grid < 1) grid = 1;
    attn_kernel<T, D><<<grid, C::NTHREADS, C::SMEM, st>>>(mq, mk, mv, p); note_launch();
    return 0;
}

int k_attention(int dtype, int D, int H, int N, const void *qg, const void *kg, const void *vg,
                const int32_t *qperm, int kk_cap, int kq_cap, const int2 *runs, const int2 *run_info,
                const AttnItem *items, const int32_t *n_items, int max_items, void *out, float *lse, int *status,
                int num_sms, void *encode_fn, cudaStream_t st) {
    AttnParams p;
    p.H = H;
    p.N = N;
    p.qperm = qperm;
    p.kk_cap = kk_cap;
    p.kq_cap = kq_cap;
    p.runs = runs;
    p.run_info = run_info;
    p.items = items;
    p.n_items = n_items;
    p.out = out;
    p.lse = lse;
    p.status = status;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    if (dtype == DT_BF16) {
        if (D == 64) return launch_attn<__nv_bfloat16, 64>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
        return launch_attn<__nv_bfloat16, 128>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
    }
    if (D == 64) return launch_attn<float, 64>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
    return launch_attn<float, 128>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
}

}  // namespace ac
