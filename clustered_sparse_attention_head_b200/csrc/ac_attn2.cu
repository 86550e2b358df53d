// Block-sparse exact softmax attention over selected key clusters (AdaCluster,
// Algorithm 3 line 9; line 4 for dense heads), bf16 inputs, two query tiles
// per CTA.
//
// A work item is up to 256 query rows of one query cluster (two 128-row
// tiles) that share one key stream: the rows of every selected key cluster of
// the gathered K/V, in chunks of <= 128 keys (TMA, 32-row boxes, 2-stage ring).
// Per chunk j and tile t the single MMA thread issues S_t(j) = Q_t K_j^T into
// TMEM and, once softmax warpgroup t has written P_t(j) (bf16) back into the
// same TMEM columns, O_t += P_t(j) V_j with the A operand read from TMEM.  The
// issue order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) lets each tile's softmax
// run while the tensor core works on the other tile.
//
// Ordering facts the protocol relies on (tcgen05 operations issued by one
// thread complete in issue order, and a commit covers all earlier ones):
//  - S_t(j+1) is issued after PV_t(j), so it never overwrites P_t(j) early;
//  - the commit after S_t(j) also covers PV_t(j-1), so when S_t(j) is ready
//    the softmax may both overwrite the P_t columns and rescale O_t;
//  - only the epilogue waits for the item's last PV_t (pv_done[t]).
// Every mbarrier wait is bounded; on expiry the CTA records ST_TIMEOUT,
// drains its copies and MMAs, frees TMEM and returns.
#include "ac_kernels.cuh"

namespace ac {

template <int D> struct A2Cfg {
    static constexpr int BM = 128, BN = 128, EPR = 64, DB = D / 64, BOX = 32, KSTEP = 16;
    static constexpr int Q_BYTES = BM * D * 2;     // one query tile
    static constexpr int KV_BYTES = BN * D * 2;    // one stage of K (or of V)
    // K is consumed by S right away; V only after the softmax, so V gets the
    // deeper ring (its loads must start further ahead of their use)
    static constexpr int KST = 2, VST = 3;
    static constexpr int OFF_Q = 0;                // tile 1 at + Q_BYTES
    static constexpr int OFF_K = 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr int SMEM_RAW = OFF_BAR + 256 + 1024;
    // at least 116 KB so that two CTAs never share an SM (each takes all of TMEM)
    static constexpr int SMEM = SMEM_RAW > 116 * 1024 ? SMEM_RAW : 116 * 1024;
    // warps 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA, 9 MMA, 10-11 idle:
    // three full warpgroups, so registers can move between them (setmaxnreg)
    static constexpr int NTHREADS = 384;
    static constexpr int REGS_LAUNCH = 168, REGS_LOW = 56, REGS_HIGH = 224;
    static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= NTHREADS * REGS_LAUNCH, "register split");
    static constexpr uint32_t TMEM_COLS = 512;     // S/P 0, S/P 1, O 0, O 1
    static constexpr int TM_S = 0, TM_O = 256;     // + 128 t
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct A2Params {
    int H, N;
    const int32_t *qperm;
    const int32_t *koff;
    int kk_cap;
    const int32_t *sel_idx;
    const int32_t *sel_cnt;
    int kq_cap;
    const AttnItem *items;
    const int32_t *n_items;
    __nv_bfloat16 *out;
    float *lse;
    int *status;
    float scale_log2;
    const int2 *segtab;  // per (head, query cluster): key rows of each selected cluster
};

namespace {

struct Chunks {
    const int2 *seg;
    int nsel, si, cur, end, dense_n;
    int2 nxt;
    __device__ void init(const A2Params &p, const AttnItem &it) {
        if (it.a < 0) {
            seg = nullptr;
            nsel = 1;
        } else {
            seg = p.segtab + ((size_t)it.h * p.kq_cap + it.a) * p.kk_cap;
            nsel = p.sel_cnt[(size_t)it.h * p.kq_cap + it.a];
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
        len = min(128, end - cur);
        cur += len;
        return true;
    }
    __device__ int count(const A2Params &p, const AttnItem &it) {
        init(p, it);
        int n = 0, s, l;
        while (next(s, l)) n++;
        init(p, it);
        return n;
    }
};

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = gtimer();
    while (!mbar_try_wait(bar, parity) && gtimer() - t0 < 200000000ull) {
    }
}

// O += P V with A (P, bf16) read from TMEM columns a_col.. (two per 32-bit column).
__device__ __forceinline__ void umma_ts_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
        "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
        "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]),
        "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]),
        "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]),
        "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]),
        "r"(r[63])
        : "memory");
}

template <int R> __device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R> __device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

// (a0, a1) * s + c, two lanes of one packed fp32 FMA
__device__ __forceinline__ void fma2(float &o0, float &o1, float a0, float a1, float s, float c) {
    uint64_t a, b, d, e;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(b) : "f"(s));
    asm("mov.b64 %0, {%1, %1};" : "=l"(e) : "f"(c));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(e));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o0), "=f"(o1) : "l"(d));
}

// 2^x on the FMA pipe (see ac_attn.cu for the derivation): magic-constant
// rounding, cubic minimax fit on [-1/2, 1/2] (|rel err| < 7.5e-5), exponent add.
__device__ __forceinline__ float ex2_fma(float x) {
    x = fmaxf(x, -125.f);
    const float t = x + 12582912.0f;
    const int n = __float_as_int(t) - 0x4B400000;
    const float f = x - (t - 12582912.0f);
    float q = fmaf(0.0551716648042202f, f, 0.2426111251115799f);
    q = fmaf(q, f, 0.6932609677314758f);
    q = fmaf(q, f, 0.9999280571937561f);
    return __int_as_float(__float_as_int(q) + (n << 23));
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK128,
                 const __grid_constant__ CUtensorMap tmV128, const A2Params p) {
    using C = A2Cfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_full = bars + 0, *q_empty = bars + 1;
    uint64_t *k_full = bars + 2, *k_empty = bars + 4;             // [KST]
    uint64_t *v_full = bars + 6, *v_empty = bars + 9;             // [VST]
    uint64_t *s_full = bars + 12, *p_full = bars + 14, *pv_done = bars + 16, *o_free = bars + 18;
    uint64_t *drain_bar = bars + 20;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 21);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 22);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < C::KST; i++) {
            mbar_init(k_full + i, 1);
            mbar_init(k_empty + i, 1);
        }
        for (int i = 0; i < C::VST; i++) {
            mbar_init(v_full + i, 1);
            mbar_init(v_empty + i, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(s_full + i, 1);
            mbar_init(p_full + i, 128);
            mbar_init(pv_done + i, 1);
            mbar_init(o_free + i, 128);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmK128);
        prefetch_tmap(&tmV128);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = *p.n_items;

    if (warp >= 8) {
    regs_dec<C::REGS_LOW>();
    if (warp == 8) {
        // ------------------------------------------------------- TMA producer
        if (lane == 0) {
            // K/V rows are re-read by every query item of the head: keep them in
            // L2; query tiles are read once: let them go first
            const uint64_t pol_keep = l2_policy_evict_last(), pol_stream = l2_policy_evict_first();
            uint32_t g = 0, qi = 0;
            int last_k[C::KST], last_v[C::VST];
            for (int i = 0; i < C::KST; i++) last_k[i] = -1;
            for (int i = 0; i < C::VST; i++) last_v[i] = -1;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const AttnItem it = p.items[item];
                Chunks ci;
                if (ci.count(p, it) == 0) continue;
                const int nt = it.q_len > 128 ? 2 : 1;
                if (qi >= 1 && !mbar_wait(q_empty, (qi - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx(q_full, nt * C::Q_BYTES);
                for (int t = 0; t < nt; t++)
                    for (int kb = 0; kb < C::DB; kb++)
                        tma_load_2d_hint(sm + C::OFF_Q + t * C::Q_BYTES + kb * (C::BM * 128), &tmQ, q_full,
                                         kb * C::EPR, it.h * p.N + it.q_start + t * 128, pol_stream);
                qi++;
                int start, len;
                while (ci.next(start, len)) {
                    const int ks = g % C::KST, vs = g % C::VST;
                    const uint32_t ku = g / C::KST, vu = g / C::VST;
                    const int nb = (len + C::BOX - 1) / C::BOX;
                    const uint32_t bytes = (uint32_t)nb * C::BOX * 128 * C::DB;
                    const int krow = it.h * p.N + start;
                    // a full chunk is one 128-row box per column block; a short
                    // one is as many 32-row boxes as it needs
                    if (ku >= 1 && !mbar_wait(k_empty + ks, (ku - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(k_full + ks, bytes);
                    for (int kb = 0; kb < C::DB; kb++) {
                        unsigned char *dst = sm + C::OFF_K + ks * C::KV_BYTES + kb * (C::BN * 128);
                        if (nb == 4) tma_load_2d_hint(dst, &tmK128, k_full + ks, kb * C::EPR, krow, pol_keep);
                        else
                            for (int b = 0; b < nb; b++)
                                tma_load_2d_hint(dst + b * (C::BOX * 128), &tmK, k_full + ks, kb * C::EPR,
                                                 krow + b * C::BOX, pol_keep);
                    }
                    last_k[ks] = (int)ku;
                    if (vu >= 1 && !mbar_wait(v_empty + vs, (vu - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(v_full + vs, bytes);
                    for (int kb = 0; kb < C::DB; kb++) {
                        unsigned char *dst = sm + C::OFF_V + vs * C::KV_BYTES + kb * (C::BN * 128);
                        if (nb == 4) tma_load_2d_hint(dst, &tmV128, v_full + vs, kb * C::EPR, krow, pol_keep);
                        else
                            for (int b = 0; b < nb; b++)
                                tma_load_2d_hint(dst + b * (C::BOX * 128), &tmV, v_full + vs, kb * C::EPR,
                                                 krow + b * C::BOX, pol_keep);
                    }
                    last_v[vs] = (int)vu;
                    g++;
                }
            }
            if (!ok) {
                if (qi >= 1) drain(q_full, (qi - 1) & 1);
                for (int i = 0; i < C::KST; i++)
                    if (last_k[i] >= 0) drain(k_full + i, last_k[i] & 1);
                for (int i = 0; i < C::VST; i++)
                    if (last_v[i] >= 0) drain(v_full + i, last_v[i] & 1);
            }
        }
    } else if (warp == 9) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_o = idesc_make(128, D, 1, true);
            uint32_t g = 0, qi = 0;
            uint32_t pph[2] = {0, 0};  // p_full phases consumed per tile
            uint32_t act[2] = {0, 0};  // items each tile was active in
            bool ok = true;
            // Descriptors are built once; per MMA only the start-address field
            // (16-byte units, bits 0-13) moves by a compile-time offset.  All
            // shared-memory addresses here are < 256 KB, so the field never carries.
            const uint64_t qdesc = sdesc_sw128(smem_u32(sm + C::OFF_Q), 16, 1024);
            const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm + C::OFF_K), 16, 1024);
            const uint64_t vdesc0 = sdesc_make(smem_u32(sm + C::OFF_V), C::BN * 128, 1024, 2u);
            // S_t = Q_t K^T for the chunk in K ring slot ks_ (ncol key columns)
            auto issue_s = [&](int t, int ks_, int ncol) {
                const uint32_t idesc_s = idesc_make(128, ncol, 1, false);
                const uint32_t d = tmem + C::TM_S + t * 128;
                uint64_t a = qdesc + (uint64_t)((t * C::Q_BYTES) >> 4);
                uint64_t b = kdesc0 + (uint64_t)((ks_ * C::KV_BYTES) >> 4);
                for (int kb = 0; kb < C::DB; kb++) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; k4++)
                        umma_f16(d, a + 2 * k4, b + 2 * k4, idesc_s, (kb | k4) ? 1u : 0u);
                    a += (C::BM * 128) >> 4;
                    b += (C::BN * 128) >> 4;
                }
                umma_commit(s_full + t);
            };
            // O_t (+)= P_t V for V ring slot vs_; P_t is bf16 in TMEM over S_t
            auto issue_pv = [&](int t, int vs_, int ncol, bool first) {
                const uint64_t b0 = vdesc0 + (uint64_t)((vs_ * C::KV_BYTES) >> 4);
                const uint32_t d = tmem + C::TM_O + t * 128;
                const uint32_t a0 = tmem + C::TM_S + t * 128;
                const int nk = ncol / C::KSTEP;
#pragma unroll
                for (int ks = 0; ks < C::BN / C::KSTEP; ks++) {
                    if (ks < nk)
                        umma_ts_f16(d, a0 + ks * 8, b0 + (uint64_t)((ks * C::KSTEP * 128) >> 4), idesc_o,
                                    (!first || ks > 0) ? 1u : 0u);
                }
            };
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const AttnItem it = p.items[item];
                Chunks ci;
                const int nch = ci.count(p, it);
                if (nch == 0) continue;
                const int nt = it.q_len > 128 ? 2 : 1;
                if (!mbar_wait(q_full, qi & 1, abort_flag, p.status)) { ok = false; break; }
                qi++;
                int start, len;
                ci.next(start, len);
                int ncol = (len + 31) & ~31;
                // prologue: S_t(0)
                if (!mbar_wait(k_full + g % C::KST, (g / C::KST) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                for (int t = 0; t < nt; t++) issue_s(t, g % C::KST, ncol);
                umma_commit(k_empty + g % C::KST);
                if (nch == 1) umma_commit(q_empty);
                for (int j = 0; j < nch && ok; j++) {
                    const int st = g % C::VST;
                    int nstart = 0, nlen = 0;
                    const bool more = (j + 1 < nch) && ci.next(nstart, nlen);
                    const int ncol_n = (nlen + 31) & ~31;
                    if (!mbar_wait(v_full + st, (g / C::VST) & 1, abort_flag, p.status)) { ok = false; break; }
                    for (int t = 0; t < nt; t++) {
                        // PV_t(j) once softmax t has written P_t(j)
                        if (!mbar_wait(p_full + t, pph[t] & 1, abort_flag, p.status)) { ok = false; break; }
                        pph[t]++;
                        if (j == 0 && act[t] >= 1 && !mbar_wait(o_free + t, (act[t] - 1) & 1, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_pv(t, st, ncol, j == 0);
                        if (j + 1 == nch) umma_commit(pv_done + t);
                        if (t + 1 == nt) umma_commit(v_empty + st);
                        // S_t(j+1) right behind PV_t(j)
                        if (more) {
                            const int sn = (g + 1) % C::KST;
                            if (t == 0 &&
                                !mbar_wait(k_full + sn, ((g + 1) / C::KST) & 1, abort_flag, p.status)) { ok = false; break; }
                            tc_fence_after();
                            issue_s(t, sn, ncol_n);
                            if (t + 1 == nt) {
                                umma_commit(k_empty + sn);
                                if (j + 2 == nch) umma_commit(q_empty);
                            }
                        }
                    }
                    ncol = ncol_n;
                    g++;
                }
                for (int t = 0; t < nt; t++) act[t]++;
            }
            if (!ok) {
                umma_commit(drain_bar);
                drain(drain_bar, 0);
            }
        }
    }
    } else {
        regs_inc<C::REGS_HIGH>();
        // ------------------------------------------------ softmax + epilogue
        // Warpgroup t = tile t; one thread per query row (= TMEM lane).
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_addr + C::TM_S + t * 128;
        const uint32_t o_addr = tmem + lane_addr + C::TM_O + t * 128;
        const float sc = p.scale_log2;
        uint32_t sph = 0, act = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const AttnItem it = p.items[item];
            const int nt = it.q_len > 128 ? 2 : 1;
            if (t >= nt) continue;
            Chunks ci;
            const int nch = ci.count(p, it);
            const int r = t * 128 + row;
            const bool valid = r < it.q_len;
            int tok = 0;
            if (valid) tok = p.qperm[(size_t)it.h * p.N + it.q_start + r];
            __nv_bfloat16 *orow = p.out + ((size_t)it.h * p.N + tok) * D;
            if (nch == 0) {
                if (valid) {
                    for (int k = 0; k < D; k++) orow[k] = __float2bfloat16(0.f);
                    if (p.lse) p.lse[(size_t)it.h * p.N + tok] = -INFINITY;
                }
                continue;
            }
            float m_ref = -INFINITY, l0 = 0.f, l1 = 0.f;
            int start, len;
            for (int j = 0; j < nch; j++) {
                ci.next(start, len);
                if (!wait_warp(s_full + t, sph & 1, abort_flag, p.status)) { ok = false; break; }
                sph++;
                tc_fence_after();
                uint32_t s[128];
                tmem_ld128(s_addr, s);
                if (len < 128) {
#pragma unroll
                    for (int i = 0; i < 128; i++)
                        if (i >= len) s[i] = __float_as_uint(-INFINITY);
                }
                float mx = __uint_as_float(s[0]);
#pragma unroll
                for (int i = 1; i + 1 < 128; i += 2) mx = max3(mx, __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
                mx = fmaxf(mx, __uint_as_float(s[127]));
                const float m_new = mx * sc;
                if (j == 0) m_ref = m_new;
                // Move the reference max (and rescale O_t) only when it grew by
                // more than 2^8; warp-uniform because TMEM access is collective.
                // PV_t(j-1) is complete: the commit of S_t(j) covers it.
                if (j > 0 && __any_sync(0xffffffffu, m_new > m_ref + 8.f)) {
                    const float m_to = fmaxf(m_ref, m_new);
                    const float f = ex2_approx(m_ref - m_to);
                    l0 *= f;
                    l1 *= f;
#pragma unroll
                    for (int pc = 0; pc < D / 32; pc++) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + pc * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                        tmem_st32(o_addr + pc * 32, o);
                    }
                    tmem_st_wait();
                    m_ref = m_to;
                }
                const float nm = -m_ref;
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const int e = hh * 64 + 2 * i;
                        float x0, x1;
                        fma2(x0, x1, __uint_as_float(s[e]), __uint_as_float(s[e + 1]), sc, nm);
                        const float e0 = ex2_approx(x0);
                        const float e1 = (i & 1) ? ex2_fma(x1) : ex2_approx(x1);
                        l0 += e0;
                        l1 += e1;
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
                        pk[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    tmem_st32(s_addr + hh * 32, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full + t);
            }
            if (!ok) break;
            // epilogue: O_t / l, rows scattered back to token order
            if (!wait_warp(pv_done + t, act & 1, abort_flag, p.status)) { ok = false; break; }
            act++;
            tc_fence_after();
            const float lsum = l0 + l1;
            const float inv = 1.f / lsum;
#pragma unroll
            for (int pc = 0; pc < D / 32; pc++) {
                uint32_t o[32];
                tmem_ld32(o_addr + pc * 32, o);
                if (valid) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                        w[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + pc * 32);
#pragma unroll
                    for (int i = 0; i < 4; i++) __stcs(dst + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(o_free + t);
            if (valid && p.lse) p.lse[(size_t)it.h * p.N + tok] = (m_ref + __log2f(lsum)) * 0.69314718055994531f;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn2)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int bf16_map2(EncodeTiledFn2 enc, CUtensorMap *m, const void *base, int rows, int cols, int box_rows) {
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
static int launch2(const void *qg, const void *kg, const void *vg, const A2Params &p, int max_items, int num_sms,
                   void *encode_fn, cudaStream_t st) {
    using C = A2Cfg<D>;
    EncodeTiledFn2 enc = (EncodeTiledFn2)encode_fn;
    CUtensorMap mq, mk, mv, mk128, mv128;
    const int rows = p.H * p.N;
    if (bf16_map2(enc, &mq, qg, rows, D, 128) || bf16_map2(enc, &mk, kg, rows, D, C::BOX) ||
        bf16_map2(enc, &mv, vg, rows, D, C::BOX) || bf16_map2(enc, &mk128, kg, rows, D, 128) ||
        bf16_map2(enc, &mv128, vg, rows, D, 128))
        return -1;
    static int checked = 0;  // 1 = ok, -1 = refused
    if (checked == 0) {
        // the register split assumes the launch budget ptxas gave the kernel;
        // a larger split would make setmaxnreg.inc wait forever, so refuse
        cudaFuncAttributes fa;
        checked = (cudaFuncGetAttributes(&fa, attn2_kernel<D>) == cudaSuccess && fa.numRegs == C::REGS_LAUNCH) ? 1 : -1;
        if (checked == 1)
            cudaFuncSetAttribute(attn2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    }
    if (checked != 1) return -1;
    int grid = max_items < num_sms ? max_items : num_sms;
    if (grid < 1) grid = 1;
    attn2_kernel<D><<<grid, C::NTHREADS, C::SMEM, st>>>(mq, mk, mv, mk128, mv128, p);
    note_launch();
    return 0;
}

int k_attention2(int D, int H, int N, const void *qg, const void *kg, const void *vg, const int32_t *qperm,
                 const int32_t *koff, int kk_cap, const int32_t *sel_idx, int kq_cap, const int32_t *sel_cnt,
                 const int2 *segtab, const AttnItem *items, const int32_t *n_items, int max_items, void *out,
                 float *lse, int *status, int num_sms, void *encode_fn, cudaStream_t st) {
    A2Params p;
    p.segtab = segtab;
    p.H = H;
    p.N = N;
    p.qperm = qperm;
    p.koff = koff;
    p.kk_cap = kk_cap;
    p.sel_idx = sel_idx;
    p.sel_cnt = sel_cnt;
    p.kq_cap = kq_cap;
    p.items = items;
    p.n_items = n_items;
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = status;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    if (D == 64) return launch2<64>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
    return launch2<128>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
}

}  // namespace ac
